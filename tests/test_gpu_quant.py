"""GPU quantiser, double quantisation and dequantisation vs the CPU oracle:
bit-exact on every workload's weight and on adversarial blocks."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    from bit_nf4_quantized_09_b200 import build
    build.build()
    import bit_nf4_quantized_09_b200 as q
    assert torch.cuda.is_available()
    return q


def gpu_quant(q, W: np.ndarray):
    w = q.quantize_nf4(torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda())
    torch.cuda.synchronize()
    return w


def assert_quant_equal(w, ref):
    codes = w.codes.cpu().numpy()
    qa = w.qabsmax.cpu().numpy()
    s2 = w.s2.cpu().numpy()
    mean = w.mean.cpu().numpy()[0]
    assert np.array_equal(codes, ref["codes"]), f"codes differ at {np.flatnonzero(codes != ref['codes'])[:8]}"
    assert np.array_equal(qa, ref["qabsmax"]), f"qabsmax differ at {np.flatnonzero(qa != ref['qabsmax'])[:8]}"
    assert np.array_equal(s2.view(np.uint32), ref["s2"].view(np.uint32))
    assert np.float32(mean).view(np.uint32) == np.float32(ref["mean"]).view(np.uint32)


def assert_dequant_equal(q, ref, N, K):
    w = q.NF4Weight(torch.from_numpy(ref["codes"]).cuda(), torch.from_numpy(ref["qabsmax"]).cuda(),
                    torch.from_numpy(ref["s2"]).cuda(), torch.tensor([ref["mean"]], dtype=torch.float32).cuda(),
                    N, K)
    out = q.dequantize_nf4(w)
    torch.cuda.synchronize()
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    want = oracle.dequant_bf16_bits(ref["codes"], ref["qabsmax"], ref["s2"], ref["mean"], N, K)
    bad = np.flatnonzero(got.reshape(-1) != want.reshape(-1))
    assert bad.size == 0, f"{bad.size} bf16 mismatches, first at {bad[:8]}"


def test_tiny_quantize_and_dequant_bit_exact(q):
    cfg = synth.TINY
    W = synth.weight(cfg).numpy()
    ref = oracle.quantize_nf4(W)
    assert_quant_equal(gpu_quant(q, W), ref)
    assert_dequant_equal(q, ref, cfg.N, cfg.K)


WEIGHTS = [synth.ATTN7B, synth.MLP7B[0], synth.MLP7B[2], synth.L65B[0], synth.L65B[1], synth.L65B[2],
           synth.SWEEP[0]]


@pytest.mark.parametrize("cfg", WEIGHTS, ids=lambda c: c.name)
def test_full_size_weights_bit_exact(q, cfg):
    W = synth.weight(cfg).numpy()
    ref = oracle.quantize_nf4(W)
    assert_quant_equal(gpu_quant(q, W), ref)
    assert_dequant_equal(q, ref, cfg.N, cfg.K)


def adversarial_weight(N=24, K=448, seed=3):
    """Blocks that stress every rule: zeros, -0, one nonzero, subnormals,
    outliers, exact thresholds and their fp32 neighbours, ties, constant
    blocks; N*K/64 = 168 blocks, so the last group of 256 is short."""
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    B = W.reshape(-1, 64)
    B[0] = 0.0
    B[1] = -0.0
    B[2] = 0.0
    B[2, 5] = -0.3
    B[3] *= np.float32(1e-38)            # subnormal block
    B[4, 7] = 1e-45                      # smallest subnormal beside normals
    B[5, 9] = 30.0                       # outlier
    B[6] = 0.125                         # constant block
    _, L = oracle.nf4_levels()
    M = oracle.midpoints(L)
    vals = []
    for m in M:
        vals += [m, np.nextafter(m, np.float32(1)), np.nextafter(m, np.float32(-1))]
    vals += list(L)
    vals = np.array(vals, np.float32)
    row = 7
    while vals.size:
        blk = np.zeros(64, np.float32)
        blk[0] = 1.0
        take = vals[:63]
        blk[1:1 + take.size] = take
        B[row] = blk
        vals = vals[63:]
        row += 1
    # the same thresholds scaled by a non-power-of-two absmax
    c = np.float32(0.0371)
    for i, m in enumerate(M):
        B[row + i // 4, 0] = c
        B[row + i // 4, 1 + (i % 4) * 3] = np.float32(m) * c
        B[row + i // 4, 2 + (i % 4) * 3] = np.nextafter(np.float32(m) * c, np.float32(1))
        B[row + i // 4, 3 + (i % 4) * 3] = np.nextafter(np.float32(m) * c, np.float32(-1))
    return W


def test_adversarial_blocks_bit_exact(q):
    W = adversarial_weight()
    ref = oracle.quantize_nf4(W)
    assert_quant_equal(gpu_quant(q, W), ref)
    assert_dequant_equal(q, ref, *W.shape)


@pytest.mark.parametrize("shape", [(8, 64), (8, 128), (16, 64 * 17), (264, 320), (1000, 512)])
def test_ragged_and_tiny_shapes_bit_exact(q, shape):
    rng = np.random.default_rng(shape[0] * 7 + shape[1])
    W = (rng.standard_normal(shape) * 0.05).astype(np.float32)
    ref = oracle.quantize_nf4(W)
    assert_quant_equal(gpu_quant(q, W), ref)
    assert_dequant_equal(q, ref, *shape)


def test_quantize_is_deterministic(q):
    W = synth.weight(synth.ATTN7B).cuda()
    a = q.quantize_nf4(W)
    b = q.quantize_nf4(W)
    torch.cuda.synchronize()
    for x, y in ((a.codes, b.codes), (a.qabsmax, b.qabsmax), (a.s2, b.s2), (a.mean, b.mean)):
        assert torch.equal(x, y)


def test_e4m3_cvt_matches_oracle_sweep(q):
    """The double quantisation's E4M3 conversion (sm_100 cvt with satfinite)
    against the oracle's nearest-value definition: every fp32 in
    [2^-12, 2^10) with a stride of 16 bit patterns, both signs, plus every
    midpoint between E4M3 values and its fp32 neighbours."""
    lo = np.float32(2.0 ** -12).view(np.uint32)
    hi = np.float32(2.0 ** 10).view(np.uint32)
    bits = np.arange(lo, hi, 16, dtype=np.uint32)
    x = bits.view(np.float32)
    vals = np.array([oracle.e4m3_decode(c) for c in range(0x7F)])
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    extra = np.concatenate([mids, np.nextafter(mids, np.float32(1e9)), np.nextafter(mids, np.float32(0)),
                            np.float32([0.0, 448.0, 449.0, 464.0, 465.0, 1e30, 2.0 ** -10, 2.0 ** -9])])
    x = np.concatenate([x, extra])
    x = np.concatenate([x, -x])
    got = q.e4m3_encode(torch.from_numpy(x).cuda()).cpu().numpy()
    want = oracle.e4m3_encode_array(x)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, (x[bad[:8]], got[bad[:8]], want[bad[:8]])


def near_threshold_weight(nblocks=16384, seed=5):
    """Blocks whose absmax c is random over the whole exponent range (down to
    subnormal c) and whose other 63 values sit within +-3 ulps of c times a
    decision threshold or a level: the places where v = w / c must be
    rounded exactly for the nearest-level decision to be right."""
    rng = np.random.default_rng(seed)
    _, L = oracle.nf4_levels()
    M = oracle.midpoints(L)
    pts = np.concatenate([M, L]).astype(np.float32)
    e = rng.integers(-140, 20, nblocks)
    c = np.ldexp(1.0 + rng.random(nblocks), e).astype(np.float32)
    W = np.empty((nblocks, 64), np.float32)
    W[:, 0] = c * np.where(rng.random(nblocks) < 0.5, 1, -1).astype(np.float32)
    base = (pts[rng.integers(0, pts.size, (nblocks, 63))] * c[:, None]).astype(np.float32)
    bits = base.view(np.int32) + rng.integers(-3, 4, base.shape).astype(np.int32)
    vals = bits.view(np.float32)
    vals = np.where(np.isfinite(vals) & (np.abs(vals) <= c[:, None]), vals, base)
    W[:, 1:] = vals
    return W.reshape(256, -1)


def test_encoder_near_thresholds_bit_exact(q):
    W = near_threshold_weight()
    ref = oracle.quantize_nf4(W)
    assert_quant_equal(gpu_quant(q, W), ref)


# ------------------------------------------------------ bf16-input quantiser

@pytest.mark.parametrize("shape", [(8, 64), (264, 320), (1000, 512), (4096, 4096)])
def test_bf16_input_quantize_bit_exact(q, shape):
    """A bf16 weight quantises to the oracle's result on its exact fp32
    upcast, and to the fp32 entry point's result on that upcast."""
    rng = np.random.default_rng(shape[0] + 3 * shape[1])
    Wb = torch.from_numpy((rng.standard_normal(shape) * 0.03).astype(np.float32)).to(torch.bfloat16)
    up = Wb.float().numpy()
    ref = oracle.quantize_nf4(up)
    got = q.quantize_nf4(Wb.cuda())
    torch.cuda.synchronize()
    assert_quant_equal(got, ref)
    via_fp32 = gpu_quant(q, up)
    for a, b in ((got.codes, via_fp32.codes), (got.qabsmax, via_fp32.qabsmax), (got.s2, via_fp32.s2),
                 (got.mean, via_fp32.mean)):
        assert torch.equal(a, b)


def test_bf16_input_adversarial_blocks(q):
    """The adversarial blocks (zeros, subnormals, outliers, values at the
    thresholds) rounded to bf16: still the oracle's bits on the upcast."""
    Wb = torch.from_numpy(adversarial_weight()).to(torch.bfloat16)
    ref = oracle.quantize_nf4(Wb.float().numpy())
    got = q.quantize_nf4(Wb.cuda())
    torch.cuda.synchronize()
    assert_quant_equal(got, ref)
