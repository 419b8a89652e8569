"""GPU storage without double quantisation and the adapter merge vs the CPU
oracle, through the C ABI.

Bars: quantised codes, fp32 constants and dequantised bf16 bit-exact; the
layer's outputs within max|err|/max|ref| <= 1e-2 of the fp64 oracle; the
merge within one bf16 step of the exact fp64 merge plus the fp32
accumulation error, bit-equal to the exactly rounded merge on at least 99 %
of the entries, and within the 1e-2 bar."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(scope="module")
def q():
    from bit_nf4_quantized_09_b200 import build
    build.build()
    import bit_nf4_quantized_09_b200 as q
    assert torch.cuda.is_available()
    return q


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def check(name, got, ref, tol=TOL):
    e = oracle.rel_err(got, ref)
    print(f"{name}: max|err|/max|ref| = {e:.3e}")
    assert e <= tol, (name, e)


def quantize(q, W: torch.Tensor, nodq: bool):
    w = q.quantize_nf4_nodq(W.cuda()) if nodq else q.quantize_nf4(W.cuda())
    torch.cuda.synchronize()
    return w


def oracle_bits(W: np.ndarray, nodq: bool) -> np.ndarray:
    if nodq:
        z = oracle.quantize_nf4_nodq(W)
        return oracle.dequant_bf16_bits_nodq(z["codes"], z["absmax"], z["N"], z["K"])
    z = oracle.quantize_nf4(W)
    return oracle.dequant_bf16_bits(z["codes"], z["qabsmax"], z["s2"], z["mean"], z["N"], z["K"])


# ------------------------------------------- no double quantisation --------

NODQ_W = [synth.TINY, synth.custom(N=40, K=192, M=1, r=8), synth.ATTN7B, synth.L65B[1]]


@pytest.mark.parametrize("cfg", NODQ_W, ids=lambda c: c.name)
def test_nodq_quantize_and_dequant_bit_exact(q, cfg):
    W = synth.weight(cfg)
    Wn = W.numpy()
    if cfg.N * cfg.K <= 1 << 16:
        Wn = Wn.copy()
        Wn[1, 64:128] = 0.0        # a zero block
        Wn[2, :64] = -Wn[2, :64]
        W = torch.from_numpy(Wn)
    ref = oracle.quantize_nf4_nodq(Wn)
    w = quantize(q, W, True)
    assert np.array_equal(w.codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(w.absmax.cpu().numpy().view(np.uint32), ref["absmax"].view(np.uint32))
    out = q.dequantize_nf4(w)
    torch.cuda.synchronize()
    want = oracle.dequant_bf16_bits_nodq(ref["codes"], ref["absmax"], cfg.N, cfg.K)
    bad = np.flatnonzero(bits(out).reshape(-1) != want.reshape(-1))
    assert bad.size == 0, f"{bad.size} bf16 mismatches, first at {bad[:8]}"


def test_nodq_from_bf16_is_the_fp32_upcast(q):
    cfg = synth.custom(N=1032, K=576, M=1, r=8, outliers=True)
    Wb = synth.weight(cfg).to(torch.bfloat16)
    ref = oracle.quantize_nf4_nodq(Wb.float().numpy())
    w = quantize(q, Wb, True)
    assert np.array_equal(w.codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(w.absmax.cpu().numpy().view(np.uint32), ref["absmax"].view(np.uint32))


def test_nodq_codes_equal_double_quant_codes(q):
    W = synth.weight(synth.TINY).cuda()
    a, b = q.quantize_nf4_nodq(W), q.quantize_nf4(W)
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes)


NODQ_LINEAR = [synth.custom(N=520, K=320, M=100, r=8),      # tiled, split over K
               synth.custom(N=1024, K=1024, M=600, r=64),   # tiled, whole tiles
               synth.custom(N=264, K=1088, M=4, r=16),      # register GEMV
               synth.custom(N=776, K=1024, M=13, r=32)]     # register GEMV, two token tiles


@pytest.mark.parametrize("cfg", NODQ_LINEAR, ids=lambda c: c.name)
def test_nodq_forward_backward(q, cfg):
    W, X, A, B, dY = (synth.weight(cfg), synth.activations(cfg), synth.lora_a(cfg), synth.lora_b(cfg),
                      synth.grad_output(cfg))
    w = quantize(q, W, True)
    Xg, Ag, Bg, dYg = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    Y, sT = q.linear_fwd(Xg, w, Ag, Bg, cfg.alpha)
    dX, dA, dB = q.linear_bwd(dYg, Xg, w, Ag, Bg, cfg.alpha, sT)
    torch.cuda.synchronize()
    What = oracle.bf16_bits_to_f64(oracle_bits(W.numpy(), True))
    Yr, T = oracle.forward(f64(X), What, f64(A), f64(B), cfg.alpha, cfg.r)
    dXr, dAr, dBr = oracle.backward(f64(dY), f64(X), What, f64(A), f64(B), cfg.alpha, cfg.r)
    check("Y", f64(Y), Yr)
    check("sT", f64(sT), (cfg.alpha / cfg.r) * T)
    check("dX", f64(dX), dXr)
    check("dA", f64(dA), dAr)
    check("dB", f64(dB), dBr)


@pytest.mark.parametrize("cfg", [synth.custom(N=1024, K=576, M=24, r=16), synth.custom(N=776, K=2048, M=5, r=8)],
                         ids=lambda c: c.name)
def test_nodq_small_batch_four_token_tiles(q, cfg):
    """A weight without double quantisation through the small-batch kernel:
    24 tokens (four n8 token tiles; forced past its default limit) with K/64
    odd (one constant load per block), and 5 tokens with K/64 a multiple of
    four (one float4 of constants per row and step)."""
    W, X, A, B = synth.weight(cfg), synth.activations(cfg), synth.lora_a(cfg), synth.lora_b(cfg)
    w = quantize(q, W, True)
    old = q.get_option(q.OPT_SMALL_M_MAX)
    try:
        q.set_option(q.OPT_SMALL_M_MAX, 64)
        Y, _ = q.linear_fwd(X.cuda(), w, A.cuda(), B.cuda(), cfg.alpha)
    finally:
        q.set_option(q.OPT_SMALL_M_MAX, old)
    torch.cuda.synchronize()
    What = oracle.bf16_bits_to_f64(oracle_bits(W.numpy(), True))
    Yr, _ = oracle.forward(f64(X), What, f64(A), f64(B), cfg.alpha, cfg.r)
    check("Y", f64(Y), Yr)


# ------------------------------------------------------------ adapter merge --

def bf16_step(x: np.ndarray) -> np.ndarray:
    """Distance between neighbouring bf16 values at |x| (2^-133 below the
    smallest normal)."""
    _, e = np.frexp(np.abs(x))
    step = np.ldexp(1.0, (e - 8).astype(np.int32))
    return np.where(np.abs(x) < 2.0 ** -126, 2.0 ** -133, step)


def check_merge(got_bits, What, A, B, alpha, r):
    exact = oracle.merge_lora(What, A, B, alpha, r)
    got = oracle.bf16_bits_to_f64(got_bits)
    s = alpha / r
    # fp32 accumulation of r exact products, one fma, then one bf16 rounding
    slack = 2.0 ** -20 * (np.abs(What) + abs(s) * (np.abs(B) @ np.abs(A)))
    over = np.abs(got - exact) - (bf16_step(exact) + slack)
    assert np.all(over <= 0), f"{np.count_nonzero(over > 0)} entries outside the bound"
    same = np.mean(got_bits == oracle.f64_to_bf16_bits(exact))
    print(f"merge: {100 * same:.3f} % exactly rounded")
    assert same >= 0.99
    check("merge", got, exact)


MERGE = [(512, 512, 8), (40, 192, 16), (264, 1088, 32), (8, 64, 64), (1032, 576, 16), (4096, 4096, 64)]


@pytest.mark.parametrize("nodq", [False, True], ids=["dq", "nodq"])
@pytest.mark.parametrize("N,K,r", MERGE, ids=lambda v: str(v))
def test_merge_lora(q, N, K, r, nodq):
    cfg = synth.custom(N=N, K=K, M=1, r=r, alpha=2.0 * r, b_std=0.02)
    W, A, B = synth.weight(cfg), synth.lora_a(cfg), synth.lora_b(cfg)
    w = quantize(q, W, nodq)
    out = q.merge_lora(w, A.cuda(), B.cuda(), cfg.alpha)
    torch.cuda.synchronize()
    What = oracle.bf16_bits_to_f64(oracle_bits(W.numpy(), nodq))
    check_merge(bits(out), What, f64(A), f64(B), cfg.alpha, r)


def test_merge_zero_update_is_the_dequantised_weight(q):
    cfg = synth.custom(N=264, K=1088, M=1, r=16)
    W, A = synth.weight(cfg), synth.lora_a(cfg)
    w = quantize(q, W, False)
    out = q.merge_lora(w, A.cuda(), torch.zeros(cfg.N, cfg.r, dtype=torch.bfloat16, device="cuda"), cfg.alpha)
    deq = q.dequantize_nf4(w)
    torch.cuda.synchronize()
    assert np.array_equal(bits(out), bits(deq))
    assert np.array_equal(bits(out), oracle_bits(W.numpy(), False))


def test_merged_weight_gives_the_layer_output(q):
    """The merged bf16 weight used as a plain weight reproduces the layer's
    forward: X W_merged^T against the fp64 oracle's X What^T + s (X A^T) B^T."""
    cfg = synth.custom(N=1024, K=1024, M=64, r=16, alpha=32.0, b_std=0.02)
    W, X, A, B = synth.weight(cfg), synth.activations(cfg), synth.lora_a(cfg), synth.lora_b(cfg)
    w = quantize(q, W, False)
    Wm = q.merge_lora(w, A.cuda(), B.cuda(), cfg.alpha)
    torch.cuda.synchronize()
    What = oracle.bf16_bits_to_f64(oracle_bits(W.numpy(), False))
    Yr, _ = oracle.forward(f64(X), What, f64(A), f64(B), cfg.alpha, cfg.r)
    check("X W_merged^T", f64(X) @ f64(Wm).T, Yr)


def test_merge_deterministic(q):
    cfg = synth.custom(N=1032, K=576, M=1, r=32)
    W, A, B = synth.weight(cfg), synth.lora_a(cfg).cuda(), synth.lora_b(cfg).cuda()
    w = quantize(q, W, True)
    a = q.merge_lora(w, A, B, cfg.alpha)
    b = q.merge_lora(w, A, B, cfg.alpha)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
