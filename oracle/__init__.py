"""CPU oracle for the frozen-NF4 QLoRA linear layer.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are its only users. The product (the CUDA library and its
binding) never imports it, and it never imports the product.

Two halves:
  * quantisation (NF4 levels, blockwise absmax, nearest-level codes, nibble
    packing, double quantisation, dequantisation to bf16) in plain C
    (nf4_oracle.c), reached through ctypes;
  * forward and backward of the layer in fp64 with numpy matmuls as the only
    library step ([p2] "26.2.4 スケーリング係数アルファ": y = W x + (alpha/r) B (A x);
    gradients by the chain rule, none for the frozen W, [p1] "勾配は実際どこへ行くのか").
Beside them: storage without double quantisation, the adapter merge with its
one-step fp64 -> bf16 rounding, a batch whose rows use different adapters over
one base, and projections that share their input.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def lib():
    """Load (building first if needed) the C oracle."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_normal_icdf.restype = ctypes.c_double
        L.oracle_normal_icdf.argtypes = [ctypes.c_double]
        L.oracle_nf4_levels.argtypes = [_f64p, _f32p]
        L.oracle_midpoints.argtypes = [_f32p, ctypes.c_int, _f32p]
        L.oracle_encode_blocks.argtypes = [_f32p, _i64, ctypes.c_int, _f32p, ctypes.c_int,
                                           ctypes.c_uint8, _f32p, _u8p]
        L.oracle_pack_nibbles.argtypes = [_u8p, _i64, _u8p]
        L.oracle_unpack_nibbles.argtypes = [_u8p, _i64, _u8p]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode_array.argtypes = [_f32p, _i64, _u8p]
        L.oracle_dq_mean.restype = ctypes.c_float
        L.oracle_dq_mean.argtypes = [_f32p, _i64, _f64p]
        L.oracle_double_quant.argtypes = [_f32p, _i64, _u8p, _f32p, _f32p]
        L.oracle_dq_constant.restype = ctypes.c_float
        L.oracle_dq_constant.argtypes = [ctypes.c_uint8, ctypes.c_float, ctypes.c_float]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_dequant_bf16.argtypes = [_u8p, _u8p, _f32p, ctypes.c_float, _i64, _i64, _u16p]
        L.oracle_quantize_nf4.restype = ctypes.c_int
        L.oracle_quantize_nf4.argtypes = [_f32p, _i64, _i64, _u8p, _u8p, _f32p, _f32p, _f32p]
        L.oracle_storage_bytes.restype = ctypes.c_int64
        L.oracle_storage_bytes.argtypes = [_i64, _i64, ctypes.c_int]
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_quantize_nf4_nodq.restype = ctypes.c_int
        L.oracle_quantize_nf4_nodq.argtypes = [_f32p, _i64, _i64, _u8p, _f32p]
        L.oracle_dequant_f32_nodq.argtypes = [_u8p, _f32p, _i64, _i64, _f32p]
        L.oracle_dequant_bf16_nodq.argtypes = [_u8p, _f32p, _i64, _i64, _u16p]
        L.oracle_f64_to_bf16.restype = ctypes.c_uint16
        L.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        L.oracle_f64_to_bf16_array.argtypes = [_f64p, _i64, _u16p]
        _lib = L
    return _lib


def _p(a: np.ndarray, t):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(t)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


# ---------------------------------------------------------------- levels ----

def normal_icdf(p: float) -> float:
    return lib().oracle_normal_icdf(float(p))


def nf4_levels() -> tuple[np.ndarray, np.ndarray]:
    """(fp64 levels, fp32 levels), 16 each, sorted ascending."""
    l64 = np.zeros(16, np.float64)
    l32 = np.zeros(16, np.float32)
    lib().oracle_nf4_levels(_p(l64, _f64p), _p(l32, _f32p))
    return l64, l32


def midpoints(levels) -> np.ndarray:
    L = _f32(levels)
    m = np.zeros(len(L) - 1, np.float32)
    lib().oracle_midpoints(_p(L, _f32p), len(L), _p(m, _f32p))
    return m


# ---------------------------------------------------------------- encode ----

def encode_blocks(w, block: int = 64, levels=None, zero_code: int = 7):
    """Blockwise absmax + nearest-level codes (unpacked, one per byte).

    w is any fp32 array whose size is a multiple of `block`; returns
    (absmax[nblocks] fp32, codes[w.size] uint8)."""
    w = _f32(w).reshape(-1)
    if levels is None:
        levels = nf4_levels()[1]
    L = _f32(levels)
    nb = w.size // block
    absmax = np.zeros(nb, np.float32)
    codes = np.zeros(w.size, np.uint8)
    lib().oracle_encode_blocks(_p(w, _f32p), nb, block, _p(L, _f32p), len(L), zero_code,
                               _p(absmax, _f32p), _p(codes, _u8p))
    return absmax, codes


def pack_nibbles(codes) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(codes, np.uint8).reshape(-1))
    out = np.zeros(c.size // 2, np.uint8)
    lib().oracle_pack_nibbles(_p(c, _u8p), c.size, _p(out, _u8p))
    return out


def unpack_nibbles(packed) -> np.ndarray:
    p = np.ascontiguousarray(np.asarray(packed, np.uint8).reshape(-1))
    out = np.zeros(p.size * 2, np.uint8)
    lib().oracle_unpack_nibbles(_p(p, _u8p), out.size, _p(out, _u8p))
    return out


# ------------------------------------------------------------------ E4M3 ----

def e4m3_decode(q: int) -> float:
    return lib().oracle_e4m3_decode(int(q) & 0xFF)


def e4m3_encode(x: float) -> int:
    return int(lib().oracle_e4m3_encode(float(x)))


def e4m3_encode_array(x) -> np.ndarray:
    x = _f32(x).reshape(-1)
    q = np.zeros(x.size, np.uint8)
    lib().oracle_e4m3_encode_array(_p(x, _f32p), x.size, _p(q, _u8p))
    return q


# --------------------------------------------------------- double quant ----

def dq_mean(c) -> tuple[float, float]:
    """(fp32 mean, fp64 tree sum) of the first-level constants."""
    c = _f32(c).reshape(-1)
    s = ctypes.c_double(0.0)
    m = lib().oracle_dq_mean(_p(c, _f32p), c.size, ctypes.byref(s))
    return float(np.float32(m)), s.value


def double_quant(c):
    """(qabsmax uint8[nb], s2 fp32[ng], mean fp32) of fp32 constants c[nb]."""
    c = _f32(c).reshape(-1)
    nb = c.size
    ng = (nb + 255) // 256
    q = np.zeros(nb, np.uint8)
    s2 = np.zeros(ng, np.float32)
    mean = np.zeros(1, np.float32)
    lib().oracle_double_quant(_p(c, _f32p), nb, _p(q, _u8p), _p(s2, _f32p), _p(mean, _f32p))
    return q, s2, mean[0]


def dq_constant(q: int, s2: float, mean: float) -> float:
    return float(np.float32(lib().oracle_dq_constant(int(q), float(s2), float(mean))))


def f32_to_bf16_bits(x: float) -> int:
    return int(lib().oracle_f32_to_bf16(float(x)))


# ------------------------------------------------------- whole quantiser ----

def quantize_nf4(W):
    """fp32 W [N, K] -> dict(codes packed uint8[N*K/2], qabsmax uint8[nb],
    s2 fp32[ng], mean fp32, absmax fp32[nb])."""
    W = _f32(W)
    N, K = W.shape
    n = N * K
    nb = n // 64
    ng = (nb + 255) // 256
    codes = np.zeros(n // 2, np.uint8)
    q = np.zeros(nb, np.uint8)
    s2 = np.zeros(ng, np.float32)
    mean = np.zeros(1, np.float32)
    absmax = np.zeros(nb, np.float32)
    rc = lib().oracle_quantize_nf4(_p(W, _f32p), N, K, _p(codes, _u8p), _p(q, _u8p),
                                   _p(s2, _f32p), _p(mean, _f32p), _p(absmax, _f32p))
    if rc != 0:
        raise ValueError(f"oracle_quantize_nf4: bad shape {W.shape}")
    return dict(codes=codes, qabsmax=q, s2=s2, mean=np.float32(mean[0]), absmax=absmax,
                N=N, K=K)


def dequant_bf16_bits(codes, qabsmax, s2, mean, N: int, K: int) -> np.ndarray:
    """bf16 bit patterns (uint16 [N, K]) of the dequantised weight."""
    codes = np.ascontiguousarray(np.asarray(codes, np.uint8))
    qabsmax = np.ascontiguousarray(np.asarray(qabsmax, np.uint8))
    s2 = _f32(s2)
    out = np.zeros((N, K), np.uint16)
    lib().oracle_dequant_bf16(_p(codes, _u8p), _p(qabsmax, _u8p), _p(s2, _f32p),
                              float(mean), N, K, _p(out, _u16p))
    return out


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# ------------------------------------- storage without double quantisation --

def quantize_nf4_nodq(W):
    """fp32 W [N, K] -> dict(codes packed uint8[N*K/2], absmax fp32[nb]): the
    blockwise quantiser with each block's fp32 absmax kept as its constant
    ([p1] 二重量子化, 4 + 32/64 = 4.5 bits per weight)."""
    W = _f32(W)
    N, K = W.shape
    codes = np.zeros(N * K // 2, np.uint8)
    absmax = np.zeros(N * K // 64, np.float32)
    rc = lib().oracle_quantize_nf4_nodq(_p(W, _f32p), N, K, _p(codes, _u8p), _p(absmax, _f32p))
    if rc != 0:
        raise ValueError(f"oracle_quantize_nf4_nodq: bad shape {W.shape}")
    return dict(codes=codes, absmax=absmax, N=N, K=K)


def dequant_f32_nodq(codes, absmax, N: int, K: int) -> np.ndarray:
    """fp32 [N, K] restore level[code] * absmax of a weight without double
    quantisation."""
    codes = np.ascontiguousarray(np.asarray(codes, np.uint8))
    absmax = _f32(absmax)
    out = np.zeros((N, K), np.float32)
    lib().oracle_dequant_f32_nodq(_p(codes, _u8p), _p(absmax, _f32p), N, K, _p(out, _f32p))
    return out


def dequant_bf16_bits_nodq(codes, absmax, N: int, K: int) -> np.ndarray:
    """bf16 bit patterns (uint16 [N, K]) of dequant_f32_nodq's values."""
    codes = np.ascontiguousarray(np.asarray(codes, np.uint8))
    absmax = _f32(absmax)
    out = np.zeros((N, K), np.uint16)
    lib().oracle_dequant_bf16_nodq(_p(codes, _u8p), _p(absmax, _f32p), N, K, _p(out, _u16p))
    return out


def f64_to_bf16_bits(x) -> np.ndarray:
    """bf16 bit patterns of fp64 values, each rounded once (nearest, ties to
    even; overflow to infinity)."""
    x = np.ascontiguousarray(np.asarray(x, np.float64))
    out = np.zeros(x.shape, np.uint16)
    lib().oracle_f64_to_bf16_array(_p(x, _f64p), x.size, _p(out, _u16p))
    return out


def storage_bytes(N: int, K: int, double_quant: bool = True) -> int:
    return int(lib().oracle_storage_bytes(N, K, 1 if double_quant else 0))


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def lora_param_count(N: int, K: int, r: int) -> int:
    """Trainable numbers of one adapter pair: B is N x r, A is r x K
    ([p1] 前提: LoRAの低ランク更新, r(d + k))."""
    return r * N + r * K


# ------------------------------------------------------ forward/backward ----
# All inputs are taken exactly (bf16 / fp32 values upcast to fp64) and every
# product and sum below is fp64.

def forward(X, What, A, B, alpha: float, r: int):
    """Y = X What^T + (alpha/r) (X A^T) B^T   and   T = X A^T.

    [p2] 26.2.4: y = W x + (alpha/r) B (A x), with x a row of X; [p1] 勾配は
    実際どこへ行くのか: W is the dequantised weight What."""
    s = alpha / r
    T = X @ A.T
    Y = X @ What.T + s * (T @ B.T)
    return Y, T


def backward(dY, X, What, A, B, alpha: float, r: int):
    """Gradients of <dY, Y> for the forward above, by the chain rule:
         dX = dY What + s (dY B) A,  dA = s (dY B)^T X,  dB = s dY^T (X A^T).
    No gradient for What: the frozen weight ([p1] 勾配は実際どこへ行くのか)."""
    s = alpha / r
    U = dY @ B
    dX = dY @ What + s * (U @ A)
    dA = s * (U.T @ X)
    dB = s * (dY.T @ (X @ A.T))
    return dX, dA, dB


# ------------------------------------------------------------ adapter merge --

def merge_lora(What, A, B, alpha: float, r: int) -> np.ndarray:
    """W_merged = What + (alpha/r) B A in fp64: the adapter folded into the
    weight once, for inference ([p2] 26.2.2, LoRAの学習設定, inference: merge
    once, then use W_merged like the original weight). B is [N, r], A is
    [r, K], What the dequantised [N, K] weight. Merging into the 16-bit weight
    rather than the 4-bit one is [p1] 落とし穴 (an update added to the NF4
    weight and re-quantised is mostly lost)."""
    s = alpha / r
    return What + s * (B @ A)


def merge_lora_bf16_bits(What, A, B, alpha: float, r: int) -> np.ndarray:
    """merge_lora rounded once to bf16 (uint16 bit patterns)."""
    return f64_to_bf16_bits(merge_lora(What, A, B, alpha, r))


# ------------------------------------------------- several adapters, one base --

def forward_multi(X, What, As, Bs, ids, alpha: float, r: int):
    """Y for a batch whose token rows use different adapters over one frozen
    base: row m uses adapter ids[m], Y_m = X_m What^T + (alpha/r) (X_m A_k^T)
    B_k^T with k = ids[m]. [p2] 26.7.3: one base model hosts many adapters and
    switches between them at run time; [p3] 利用ケース: one 4-bit base serves
    several adapters. As: [P, r, K]; Bs: [P, N, r]; ids: int [M] in [0, P).
    Written as the single-adapter forward applied to each adapter's rows."""
    ids = np.asarray(ids)
    if ids.size and (ids.min() < 0 or ids.max() >= len(As)):
        raise ValueError("adapter id out of range")
    Y = np.zeros((X.shape[0], What.shape[0]))
    for k in range(len(As)):
        rows = np.flatnonzero(ids == k)
        if rows.size:
            Y[rows], _ = forward(X[rows], What, As[k], Bs[k], alpha, r)
    return Y


def backward_multi(dY, X, What, As, Bs, ids, alpha: float, r: int):
    """Gradients of <dY, forward_multi>: dX row by row with the row's adapter;
    dA_k and dB_k from the rows that use adapter k only (zero for an adapter no
    row uses)."""
    ids = np.asarray(ids)
    dX = np.zeros_like(X, dtype=np.float64)
    dAs = np.zeros((len(As),) + As[0].shape)
    dBs = np.zeros((len(Bs),) + Bs[0].shape)
    for k in range(len(As)):
        rows = np.flatnonzero(ids == k)
        if rows.size:
            dX[rows], dAs[k], dBs[k] = backward(dY[rows], X[rows], What, As[k], Bs[k], alpha, r)
    return dX, dAs, dBs


# ------------------------------------------ projections that share the input --

def forward_group(X, Whats, As, Bs, alpha: float, r: int):
    """Projections of one input with their own frozen weights and adapters
    (q, k, v of attention, or gate and up of the MLP), outputs side by side:
    [Y_1 | Y_2 | ...], Y_i the layer's forward with (What_i, A_i, B_i)."""
    return np.concatenate([forward(X, Wi, Ai, Bi, alpha, r)[0] for Wi, Ai, Bi in zip(Whats, As, Bs)], axis=1)


def rel_err(got, ref) -> float:
    """max |got - ref| / max |ref| (0 when both are all-zero)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.max(np.abs(ref)) if ref.size else 0.0
    num = np.max(np.abs(got - ref)) if ref.size else 0.0
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)
