"""GPU parity of the two batching forms against the fp64 CPU oracle.

Several adapters over one frozen base ("waylandz LLM book ch.26", 26.7.3;
"agentlenshq" summary, 利用ケース): token row m uses adapter ids[m]. The
oracle is oracle.forward_multi / backward_multi.

Projections that share one input ("ta-paperlens QLoRA explainer", コードで見る
and 落とし穴: adapters on every linear layer, e.g. q/k/v or gate/up): each
projection keeps its own NF4 weight (own mean and s2) and adapter; outputs
side by side. The oracle is oracle.forward_group for the forward and, per
projection, oracle.backward for the gradients (dX is their sum).

Tolerance as for the single layer: max|err| / max|ref| <= 1e-2 per tensor.
Exact checks where the arithmetic makes them exact: the columns of the
rank-r inputs that belong to another adapter are zero, an adapter no row
uses gets zero gradients, and with one adapter the multi call returns the
single-adapter call's bits."""
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


def check(name, got, ref, tol=TOL):
    e = oracle.rel_err(got, ref)
    print(f"{name}: max|err|/max|ref| = {e:.3e}")
    assert e <= tol, (name, e)
    return e


def oracle_what(W: torch.Tensor, dq=True) -> np.ndarray:
    if dq:
        z = oracle.quantize_nf4(W.numpy())
        bits = oracle.dequant_bf16_bits(z["codes"], z["qabsmax"], z["s2"], z["mean"], z["N"], z["K"])
    else:
        z = oracle.quantize_nf4_nodq(W.numpy())
        bits = oracle.dequant_bf16_bits_nodq(z["codes"], z["absmax"], z["N"], z["K"])
    return oracle.bf16_bits_to_f64(bits)


# ------------------------------------------------ several adapters, one base --

def multi_inputs(N, K, M, r, P, seed, unused=(), none_rows=0):
    """P adapters drawn as independent layers of rank r; ids random over the
    used adapters, with `none_rows` rows whose id is -1 (no adapter)."""
    cfgs = [synth.custom(N=N, K=K, M=M, r=r, seed_base=seed + k) for k in range(P)]
    W = synth.weight(cfgs[0])
    X, dY = synth.activations(cfgs[0]), synth.grad_output(cfgs[0])
    As = [synth.lora_a(c) for c in cfgs]
    Bs = [synth.lora_b(c) for c in cfgs]
    used = [k for k in range(P) if k not in unused]
    rng = np.random.default_rng(seed)
    ids = rng.choice(used, size=M).astype(np.int32)
    if none_rows:
        ids[rng.choice(M, none_rows, replace=False)] = -1
    return dict(W=W, X=X, dY=dY, As=As, Bs=Bs, ids=ids, alpha=cfgs[0].alpha)


def run_multi(q, t, P, r, recompute=False):
    w = q.quantize_nf4(t["W"].cuda())
    A = torch.cat(t["As"], dim=0).cuda()          # [P r, K]
    B = torch.cat(t["Bs"], dim=1).contiguous().cuda()  # [N, P r]
    ids = torch.from_numpy(t["ids"]).cuda()
    X, dY = t["X"].cuda(), t["dY"].cuda()
    Y, sT = q.linear_fwd_multi(X, w, A, B, ids, P, t["alpha"])
    dX, dA, dB = q.linear_bwd_multi(dY, X, w, A, B, ids, P, t["alpha"], sT=None if recompute else sT)
    torch.cuda.synchronize()
    return dict(Y=Y, sT=sT, dX=dX, dA=dA, dB=dB, w=w, A=A, B=B, ids=ids)


def compare_multi(q, t, P, r, recompute=False):
    g = run_multi(q, t, P, r, recompute)
    What = oracle_what(t["W"])
    X, dY = f64(t["X"]), f64(t["dY"])
    As = [f64(a) for a in t["As"]]
    Bs = [f64(b) for b in t["Bs"]]
    ids, alpha = t["ids"], t["alpha"]
    # rows with an adapter through the oracle's multi-adapter layer; rows
    # with id -1 use none: the frozen base layer, X W^T and dY W
    on = ids >= 0
    Y = X @ What.T
    dX = dY @ What
    Y[on] = oracle.forward_multi(X[on], What, As, Bs, ids[on], alpha, r)
    dX[on], dAs, dBs = oracle.backward_multi(dY[on], X[on], What, As, Bs, ids[on], alpha, r)
    check("Y", f64(g["Y"]), Y)
    check("dX", f64(g["dX"]), dX)
    check("dA", f64(g["dA"]), np.concatenate(list(dAs), axis=0))
    check("dB", f64(g["dB"]), np.concatenate(list(dBs), axis=1))
    # the rank-r input of row m holds s X_m A_k^T in its own adapter's columns
    # and exact zeros in every other adapter's
    sT = f64(g["sT"])
    s = alpha / r
    for k in range(P):
        cols = slice(k * r, (k + 1) * r)
        own = ids == k
        assert np.all(sT[~own, cols] == 0.0), k
        if own.any():
            check(f"sT[{k}]", sT[own, cols], s * X[own] @ As[k].T)
    return g


MULTI = [  # (N, K, M, r, P)
    (1024, 512, 300, 16, 3),     # tiled path, split tiles
    (512, 768, 1000, 8, 8),      # eight adapters, rank 64 in all
    (520, 320, 257, 64, 4),      # rank 256 in all: four 64-column chunks, ragged N
    (2048, 1024, 5, 16, 4),      # register-fed small-batch kernel
    (264, 640, 40, 32, 2),       # M between the small-batch kernels and the tiled path
]


@pytest.mark.parametrize("shape", MULTI, ids=lambda s: "N{}_K{}_M{}_r{}_P{}".format(*s))
def test_several_adapters_against_oracle(q, shape):
    N, K, M, r, P = shape
    compare_multi(q, multi_inputs(N, K, M, r, P, seed=300 + P), P, r)


def test_unused_adapter_and_rows_without_adapter(q):
    """An adapter no row uses gets exactly zero dA and dB; rows with id -1
    get the frozen base layer only, bit for bit what a call with B = 0
    returns for them."""
    N, K, M, r, P = 1024, 512, 200, 16, 4
    t = multi_inputs(N, K, M, r, P, seed=410, unused=(2,), none_rows=30)
    g = compare_multi(q, t, P, r)
    dA, dB = g["dA"].cpu(), g["dB"].cpu()
    assert torch.count_nonzero(dA[2 * r:3 * r]) == 0
    assert torch.count_nonzero(dB[:, 2 * r:3 * r]) == 0
    Y0, _ = q.linear_fwd_multi(t["X"].cuda(), g["w"], g["A"], torch.zeros_like(g["B"]), g["ids"], P, t["alpha"])
    torch.cuda.synchronize()
    none = torch.from_numpy(t["ids"] == -1)
    assert torch.equal(g["Y"].cpu()[none].view(torch.int16), Y0.cpu()[none].view(torch.int16))


def test_one_adapter_equals_the_single_call(q):
    """P = 1 with every id 0 launches the same kernels on the same operands
    as qlora_linear_fwd/bwd: identical bits."""
    cfg = synth.custom(N=1024, K=1024, M=333, r=32, seed_base=420)
    W, X, A, B, dY = (synth.weight(cfg), synth.activations(cfg), synth.lora_a(cfg), synth.lora_b(cfg),
                      synth.grad_output(cfg))
    w = q.quantize_nf4(W.cuda())
    X, A, B, dY = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    ids = torch.zeros(cfg.M, dtype=torch.int32, device="cuda")
    Y1, sT1 = q.linear_fwd(X, w, A, B, cfg.alpha)
    d1 = q.linear_bwd(dY, X, w, A, B, cfg.alpha, sT1)
    Y2, sT2 = q.linear_fwd_multi(X, w, A, B, ids, 1, cfg.alpha)
    d2 = q.linear_bwd_multi(dY, X, w, A, B, ids, 1, cfg.alpha, sT2)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2) and torch.equal(sT1, sT2)
    for a, b in zip(d1, d2):
        assert torch.equal(a, b)


def test_several_adapters_recompute_and_determinism(q):
    N, K, M, r, P = 768, 512, 400, 16, 3
    t = multi_inputs(N, K, M, r, P, seed=430)
    a = run_multi(q, t, P, r)
    b = run_multi(q, t, P, r, recompute=True)
    for k in ("dX", "dA", "dB"):
        assert torch.equal(a[k], b[k]), k
    c = run_multi(q, t, P, r)
    for k in ("Y", "dX", "dA", "dB"):
        assert torch.equal(a[k], c[k]), k


# --------------------------------------------- projections sharing an input --

def group_inputs(Ns, K, M, r, seed):
    cfgs = [synth.custom(N=n, K=K, M=M, r=r, seed_base=seed + i) for i, n in enumerate(Ns)]
    return dict(Ws=[synth.weight(c) for c in cfgs], As=[synth.lora_a(c) for c in cfgs],
                Bs=[synth.lora_b(c) for c in cfgs], X=synth.activations(cfgs[0]),
                dY=synth.grad_output(synth.custom(N=sum(Ns), K=K, M=M, r=r, seed_base=seed + 9)),
                alpha=cfgs[0].alpha)


def run_group(q, t, K, r, dq=True, recompute=False):
    Ns = [w.shape[0] for w in t["Ws"]]
    if dq:
        group = q.empty_group(Ns, K, "cuda")
        for w, W in zip(group, t["Ws"]):
            q.quantize_nf4(W.cuda(), out=w)
    else:
        codes = torch.empty(sum(Ns) * K // 2, dtype=torch.uint8, device="cuda")
        group, at = [], 0
        for W in t["Ws"]:
            n = W.shape[0]
            w = q.NF4Weight(codes[at:at + n * K // 2], None, None, None, n, K,
                            absmax=torch.empty(n * K // 64, dtype=torch.float32, device="cuda"))
            q.quantize_nf4_nodq(W.cuda(), out=w)
            group.append(w)
            at += n * K // 2
    A = torch.cat(t["As"], dim=0).cuda()
    B = torch.cat(t["Bs"], dim=0).cuda()
    X, dY = t["X"].cuda(), t["dY"].cuda()
    Y, sT = q.linear_fwd_group(X, group, A, B, t["alpha"])
    dX, dA, dB = q.linear_bwd_group(dY, X, group, A, B, t["alpha"], sT=None if recompute else sT)
    torch.cuda.synchronize()
    return dict(Y=Y, sT=sT, dX=dX, dA=dA, dB=dB)


def compare_group(q, t, K, r, dq=True, grads=True):
    g = run_group(q, t, K, r, dq)
    Whats = [oracle_what(W, dq) for W in t["Ws"]]
    As = [f64(a) for a in t["As"]]
    Bs = [f64(b) for b in t["Bs"]]
    X, alpha = f64(t["X"]), t["alpha"]
    check("Y", f64(g["Y"]), oracle.forward_group(X, Whats, As, Bs, alpha, r))
    s = alpha / r
    check("sT", f64(g["sT"]), np.concatenate([s * X @ a.T for a in As], axis=1))
    if grads:
        dY = f64(t["dY"])
        offs = np.cumsum([0] + [w.shape[0] for w in Whats])
        dX = np.zeros_like(X)
        dAs, dBs = [], []
        for i, (Wh, a, b) in enumerate(zip(Whats, As, Bs)):
            dXi, dAi, dBi = oracle.backward(dY[:, offs[i]:offs[i + 1]], X, Wh, a, b, alpha, r)
            dX += dXi
            dAs.append(dAi)
            dBs.append(dBi)
        check("dX", f64(g["dX"]), dX)
        check("dA", f64(g["dA"]), np.concatenate(dAs, axis=0))
        check("dB", f64(g["dB"]), np.concatenate(dBs, axis=0))
    return g


GROUPS = [  # (Ns, K, M, r)
    ([512, 256, 256], 512, 300, 16),       # q/k/v shaped (k, v narrower), split tiles
    ([1024, 1024], 768, 520, 64),          # gate/up shaped, rank 128 in all (two chunks)
    ([520, 264, 776], 320, 257, 8),        # projections that end inside a 256-column tile
    ([4096, 1024, 1024], 1024, 4, 16),     # register-fed small-batch kernel
    ([264, 512], 640, 40, 32),             # between the small-batch kernels and the tiled path
    ([256] * 4, 256, 100, 64),             # four projections, rank 256 in all
]


@pytest.mark.parametrize("shape", GROUPS, ids=lambda s: "N{}_K{}_M{}_r{}".format("-".join(map(str, s[0])), *s[1:]))
def test_projection_group_against_oracle(q, shape):
    Ns, K, M, r = shape
    compare_group(q, group_inputs(Ns, K, M, r, seed=500 + len(Ns) + r), K, r)


def test_projection_group_without_double_quant(q):
    t = group_inputs([512, 264], 448, 130, 16, seed=560)
    compare_group(q, t, 448, 16, dq=False)
    t = group_inputs([1024, 512], 512, 7, 16, seed=561)
    compare_group(q, t, 512, 16, dq=False, grads=False)


def test_projection_group_recompute_and_determinism(q):
    t = group_inputs([512, 256, 256], 512, 300, 16, seed=570)
    a = run_group(q, t, 512, 16)
    b = run_group(q, t, 512, 16, recompute=True)
    for k in ("dX", "dA", "dB"):
        assert torch.equal(a[k], b[k]), k
    c = run_group(q, t, 512, 16)
    for k in ("Y", "dX", "dA", "dB"):
        assert torch.equal(a[k], c[k]), k


def test_llama7b_gate_up_group_full_size(q):
    """The LLaMA-7B MLP's gate and up projections (11008 x 4096 each, r = 64)
    as one group over 4096 tokens; Y and dX on 32 sampled tokens, dA and dB
    in full."""
    Ns, K, M, r = [11008, 11008], 4096, 4096, 64
    t = group_inputs(Ns, K, M, r, seed=580)
    g = run_group(q, t, K, r)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 30, replace=False)]))
    Whats = [oracle_what(W) for W in t["Ws"]]
    As = [f64(a) for a in t["As"]]
    Bs = [f64(b) for b in t["Bs"]]
    X, dY, alpha = f64(t["X"]), f64(t["dY"]), t["alpha"]
    check("Y[rows]", f64(g["Y"])[rows], oracle.forward_group(X[rows], Whats, As, Bs, alpha, r))
    s = alpha / r
    dXs = np.zeros((len(rows), K))
    for i in range(2):
        dXs += oracle.backward(dY[rows][:, i * Ns[0]:(i + 1) * Ns[0]], X[rows], Whats[i], As[i], Bs[i], alpha, r)[0]
    check("dX[rows]", f64(g["dX"])[rows], dXs)
    dA = np.concatenate([s * (dY[:, i * Ns[0]:(i + 1) * Ns[0]] @ Bs[i]).T @ X for i in range(2)], axis=0)
    dB = np.concatenate([s * dY[:, i * Ns[0]:(i + 1) * Ns[0]].T @ (X @ As[i].T) for i in range(2)], axis=0)
    check("dA", f64(g["dA"]), dA)
    check("dB", f64(g["dB"]), dB)
