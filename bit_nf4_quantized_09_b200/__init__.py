"""Python binding of libqlora_nf4.so, the frozen-NF4 QLoRA linear layer on B200.

Argument marshalling only: every step of the computation runs in the CUDA
library. torch supplies device memory and the current stream. If the library
is missing this module raises on first use; there is no fallback path.

Raw C entry points keep their C names (qlora_quantize_nf4, qlora_linear_fwd,
...) on ``lib()``; the functions below wrap them for torch tensors.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")

QLORA_OK = 0
STATUS = {0: "QLORA_OK", -1: "QLORA_ERR_INVALID_ARG", -2: "QLORA_ERR_BAD_SHAPE", -3: "QLORA_ERR_MISALIGNED",
          -4: "QLORA_ERR_UNSUPPORTED_RANK", -5: "QLORA_ERR_WORKSPACE_TOO_SMALL", -6: "QLORA_ERR_CUDA",
          -7: "QLORA_ERR_DEVICE_TIMEOUT", -8: "QLORA_ERR_UNSUPPORTED_DEVICE", -9: "QLORA_ERR_EXCEEDS_STATIC_SCRATCH"}
OP_QUANTIZE, OP_FWD, OP_BWD = 0, 1, 2
OPT_SMALL_M_MAX, OPT_FAIL_LAUNCHES, OPT_WAIT_TIMEOUT_US, OPT_STALL_PRODUCER, OPT_LAUNCH_COUNT = 1, 2, 3, 4, 5
OPT_SKINNY_MAX_SPLITS = 6
OPT_FUSED_PAIRS = 8
OPT_FUSED_TAIL = 9
KERNEL_FUSED_FWD, KERNEL_FUSED_DX = 1, 2


class QLoraError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}" + (f" ({detail})" if detail else ""))


class Nf4WeightC(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("qabsmax", ctypes.c_void_p), ("s2", ctypes.c_void_p),
                ("mean", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("absmax", ctypes.c_void_p)]


_lib = None
_vp, _i64, _sz, _int, _f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
_wp = ctypes.POINTER(Nf4WeightC)

# name -> (restype, argtypes); names match include/qlora_nf4.h
_SIGNATURES = {
    "qlora_nf4_bytes": (_i64, [_i64, _i64, ctypes.POINTER(_sz), ctypes.POINTER(_sz), ctypes.POINTER(_sz),
                               ctypes.POINTER(_sz)]),
    "qlora_workspace_bytes": (_sz, [_int, _i64, _i64, _i64, _int]),
    "qlora_quantize_nf4": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "qlora_quantize_nf4_noalloc": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp]),
    "qlora_quantize_nf4_bf16": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "qlora_quantize_nf4_nodq": (_int, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "qlora_quantize_nf4_bf16_nodq": (_int, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "qlora_dequantize_nf4": (_int, [_wp, _vp, _vp]),
    "qlora_merge_lora": (_int, [_wp, _vp, _vp, _int, _f32, _vp, _vp]),
    "qlora_linear_fwd": (_int, [_vp, _i64, _wp, _vp, _vp, _int, _f32, _vp, _vp, _vp, _sz, _vp]),
    "qlora_linear_bwd": (_int, [_vp, _vp, _i64, _wp, _vp, _vp, _int, _f32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "qlora_workspace_bytes_multi": (_sz, [_int, _i64, _i64, _i64, _int, _int]),
    "qlora_linear_fwd_multi": (_int, [_vp, _i64, _wp, _vp, _vp, _int, _int, _vp, _f32, _vp, _vp, _vp, _sz, _vp]),
    "qlora_linear_bwd_multi": (_int, [_vp, _vp, _i64, _wp, _vp, _vp, _int, _int, _vp, _f32, _vp, _vp, _vp, _vp,
                                      _vp, _sz, _vp]),
    "qlora_workspace_bytes_group": (_sz, [_int, _i64, ctypes.POINTER(_i64), _int, _i64, _int]),
    "qlora_linear_fwd_group": (_int, [_vp, _i64, _wp, _int, _vp, _vp, _int, _f32, _vp, _vp, _vp, _sz, _vp]),
    "qlora_linear_bwd_group": (_int, [_vp, _vp, _i64, _wp, _int, _vp, _vp, _int, _f32, _vp, _vp, _vp, _vp, _vp,
                                      _sz, _vp]),
    "qlora_nf4_tables": (_int, [ctypes.POINTER(_f32), ctypes.POINTER(_f32)]),
    "qlora_device_status": (_int, [_vp, ctypes.POINTER(_int), _vp]),
    "qlora_status_string": (ctypes.c_char_p, [_int]),
    "qlora_last_error": (ctypes.c_char_p, []),
    "qlora_set_option": (_int, [_int, _i64]),
    "qlora_get_option": (_i64, [_int]),
    "qlora_e4m3_encode": (_int, [_vp, _vp, _i64, _vp]),
    "qlora_profile_next_launch": (_int, [_int, _vp, _vp]),
}


def lib():
    """Load libqlora_nf4.so (built in-tree by bit_nf4_quantized_09_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m bit_nf4_quantized_09_b200.build` "
                              "(no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != QLORA_OK:
        detail = lib().qlora_last_error().decode(errors="replace")
        raise QLoraError(status, where, detail)


_check_device_status = False


def set_check_device_status(on: bool):
    """When on, every forward/backward wrapper call reads its workspace's
    device status word back (a synchronisation) and raises if a bounded wait
    of a pipelined kernel ran out, so an unwritten tile cannot pass silently.
    Off by default: the calls stay asynchronous."""
    global _check_device_status
    _check_device_status = bool(on)


def _after_call(ws: torch.Tensor, where: str, M: int = 1):
    # an empty batch launches nothing and leaves the workspace untouched
    if _check_device_status and M > 0:
        st = device_status(ws)
        if st != QLORA_OK:
            raise QLoraError(st, where, "device status after the call")


try:
    _raw_stream = torch._C._cuda_getCurrentRawStream  # fast path: the handle without a Stream object
except AttributeError:  # pragma: no cover
    _raw_stream = None


def _stream(device=None) -> int:
    if _raw_stream is not None:
        idx = torch.cuda.current_device() if device is None else (device.index if isinstance(device, torch.device)
                                                                  and device.index is not None else
                                                                  torch.cuda.current_device())
        return _raw_stream(idx)
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    assert t.is_contiguous(), "tensors must be contiguous"
    return t.data_ptr()


# ----------------------------------------------------------------- sizes ---

def nf4_bytes(N: int, K: int) -> dict:
    c, q, s, m = _sz(), _sz(), _sz(), _sz()
    total = lib().qlora_nf4_bytes(N, K, ctypes.byref(c), ctypes.byref(q), ctypes.byref(s), ctypes.byref(m))
    if total < 0:
        raise QLoraError(-2, "qlora_nf4_bytes")
    return dict(codes=c.value, qabsmax=q.value, s2=s.value, mean=m.value, total=total)


_ws_cache: dict = {}


def workspace_bytes(op: int, M: int, N: int, K: int, r: int) -> int:
    key = (op, M, N, K, r)
    v = _ws_cache.get(key)
    if v is None:
        v = _ws_cache[key] = int(lib().qlora_workspace_bytes(op, M, N, K, r))
    return v


def nf4_tables():
    """(levels[16], thresholds[15]) as the library computes them, fp32."""
    lv = (_f32 * 16)()
    th = (_f32 * 15)()
    _check(lib().qlora_nf4_tables(lv, th), "qlora_nf4_tables")
    return list(lv), list(th)


def set_option(option: int, value: int):
    _check(lib().qlora_set_option(option, int(value)), "qlora_set_option")


def get_option(option: int) -> int:
    return int(lib().qlora_get_option(option))


# ------------------------------------------------------------ the weight ---

@dataclasses.dataclass
class NF4Weight:
    """A quantised N x K weight: device tensors owned by torch. With double
    quantisation codes, qabsmax, s2 and mean are set and absmax is None;
    without it codes and absmax are set and the other three are None."""
    codes: torch.Tensor             # uint8 [N*K/2]
    qabsmax: torch.Tensor | None    # uint8 [N*K/64]
    s2: torch.Tensor | None         # float32 [ceil(N*K/64/256)]
    mean: torch.Tensor | None       # float32 [1]
    N: int
    K: int
    absmax: torch.Tensor | None = None  # float32 [N*K/64], storage without double quantisation

    @property
    def double_quant(self) -> bool:
        return self.absmax is None

    def c_view(self) -> Nf4WeightC:
        key = tuple(t.data_ptr() if t is not None else 0
                    for t in (self.codes, self.qabsmax, self.s2, self.mean, self.absmax)) + (self.N, self.K)
        cached = self.__dict__.get("_c_view")
        if cached is None or cached[0] != key:
            cached = (key, Nf4WeightC(_ptr(self.codes), _ptr(self.qabsmax), _ptr(self.s2), _ptr(self.mean),
                                      self.N, self.K, _ptr(self.absmax)))
            self.__dict__["_c_view"] = cached
        return cached[1]

    @staticmethod
    def empty(N: int, K: int, device) -> "NF4Weight":
        sz = nf4_bytes(N, K)
        return NF4Weight(torch.empty(sz["codes"], dtype=torch.uint8, device=device),
                         torch.empty(sz["qabsmax"], dtype=torch.uint8, device=device),
                         torch.empty(sz["s2"] // 4, dtype=torch.float32, device=device),
                         torch.empty(1, dtype=torch.float32, device=device), N, K)


def _ws(nbytes: int, device, ws: torch.Tensor | None = None) -> torch.Tensor:
    if ws is not None:
        if ws.numel() < nbytes:
            raise QLoraError(-5, "workspace")
        return ws
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def quantize_nf4(W: torch.Tensor, out: NF4Weight | None = None, ws: torch.Tensor | None = None) -> NF4Weight:
    """NF4 + double quantisation of an fp32 or bf16 [N, K] CUDA tensor (a bf16
    weight gives the bits of its fp32 upcast)."""
    assert W.dtype in (torch.float32, torch.bfloat16) and W.is_cuda and W.dim() == 2
    N, K = W.shape
    w = out if out is not None else NF4Weight.empty(N, K, W.device)
    nbytes = workspace_bytes(OP_QUANTIZE, 0, N, K, 0)
    if nbytes == 0:
        raise QLoraError(-2, "qlora_quantize_nf4", f"shape {tuple(W.shape)}")
    ws = _ws(nbytes, W.device, ws)
    entry = "qlora_quantize_nf4_bf16" if W.dtype == torch.bfloat16 else "qlora_quantize_nf4"
    _check(getattr(lib(), entry)(_ptr(W), N, K, _ptr(w.codes), _ptr(w.qabsmax), _ptr(w.s2), _ptr(w.mean),
                                 _ptr(ws), ws.numel(), _stream(W.device)), entry)
    return w


def quantize_nf4_nodq(W: torch.Tensor, out: NF4Weight | None = None) -> NF4Weight:
    """NF4 without double quantisation (one fp32 absmax per block of 64) of
    an fp32 or bf16 [N, K] CUDA tensor."""
    assert W.dtype in (torch.float32, torch.bfloat16) and W.is_cuda and W.dim() == 2
    N, K = W.shape
    if K <= 0 or K % 64 != 0 or N <= 0:
        raise QLoraError(-2, "qlora_quantize_nf4_nodq", f"shape {tuple(W.shape)}")
    if out is None:
        out = NF4Weight(torch.empty(N * K // 2, dtype=torch.uint8, device=W.device), None, None, None, N, K,
                        absmax=torch.empty(N * K // 64, dtype=torch.float32, device=W.device))
    assert out.absmax is not None and (out.N, out.K) == (N, K)
    entry = "qlora_quantize_nf4_bf16_nodq" if W.dtype == torch.bfloat16 else "qlora_quantize_nf4_nodq"
    _check(getattr(lib(), entry)(_ptr(W), N, K, _ptr(out.codes), _ptr(out.absmax), _stream(W.device)), entry)
    return out


def merge_lora(w: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float,
               out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 [N, K] = deq(W) + (alpha/r) B A: the adapter folded into a 16-bit
    copy of the weight."""
    r = A.shape[0]
    out = out if out is not None else torch.empty(w.N, w.K, dtype=torch.bfloat16, device=w.codes.device)
    v = w.c_view()
    _check(lib().qlora_merge_lora(ctypes.byref(v), _ptr(A), _ptr(B), r, float(alpha), _ptr(out),
                                  _stream(out.device)), "qlora_merge_lora")
    if _check_device_status:
        st = call_status(out.device)
        if st != QLORA_OK:
            raise QLoraError(st, "qlora_merge_lora", "device status after the call")
    return out


def quantize_nf4_noalloc(W: torch.Tensor, out: NF4Weight) -> NF4Weight:
    """Quantise without any workspace: for callers that cannot allocate device
    memory at call time. The library keeps its scratch in one static device
    array (N*K up to 67,108,864 weights); `out` must be allocated beforehand."""
    assert W.dtype == torch.float32 and W.is_cuda and W.dim() == 2 and W.is_contiguous()
    N, K = W.shape
    sz = nf4_bytes(N, K)
    assert out.absmax is None and (out.N, out.K) == (N, K), "out must be an NF4Weight with double quantisation of W's shape"
    assert out.codes.numel() >= sz["codes"] and out.qabsmax.numel() >= sz["qabsmax"], "out is too small"
    assert out.s2.numel() * 4 >= sz["s2"] and out.mean.numel() >= 1, "out is too small"
    _check(lib().qlora_quantize_nf4_noalloc(_ptr(W), N, K, _ptr(out.codes), _ptr(out.qabsmax), _ptr(out.s2),
                                            _ptr(out.mean), _stream(W.device)), "qlora_quantize_nf4_noalloc")
    return out


def dequantize_nf4(w: NF4Weight, out: torch.Tensor | None = None) -> torch.Tensor:
    out = out if out is not None else torch.empty(w.N, w.K, dtype=torch.bfloat16, device=w.codes.device)
    v = w.c_view()
    _check(lib().qlora_dequantize_nf4(ctypes.byref(v), _ptr(out), _stream(out.device)), "qlora_dequantize_nf4")
    return out


def linear_fwd(X: torch.Tensor, w: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float,
               Y: torch.Tensor | None = None, sT: torch.Tensor | None = None, save_sT: bool = True,
               ws: torch.Tensor | None = None):
    """(Y, sT): Y = X deq(W)^T + (alpha/r) (X A^T) B^T, sT = bf16((alpha/r) X A^T)."""
    M, K = X.shape
    r = A.shape[0]
    dev = X.device
    Y = Y if Y is not None else torch.empty(M, w.N, dtype=torch.bfloat16, device=dev)
    if save_sT and sT is None:
        sT = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    ws = _ws(workspace_bytes(OP_FWD, M, w.N, w.K, r), dev, ws)
    v = w.c_view()
    _check(lib().qlora_linear_fwd(_ptr(X), M, ctypes.byref(v), _ptr(A), _ptr(B), r, float(alpha), _ptr(Y),
                                  _ptr(sT) if save_sT else None, _ptr(ws), ws.numel(), _stream(dev)),
           "qlora_linear_fwd")
    _after_call(ws, "qlora_linear_fwd", M)
    return Y, (sT if save_sT else None)


def linear_bwd(dY: torch.Tensor, X: torch.Tensor, w: NF4Weight, A: torch.Tensor, B: torch.Tensor,
               alpha: float, sT: torch.Tensor | None = None, dX: torch.Tensor | None = None,
               dA: torch.Tensor | None = None, dB: torch.Tensor | None = None, ws: torch.Tensor | None = None):
    """(dX, dA, dB) of <dY, Y>: dX bf16 [M, K], dA fp32 [r, K], dB fp32 [N, r]."""
    M, K = X.shape
    r = A.shape[0]
    dev = X.device
    dX = dX if dX is not None else torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dA = dA if dA is not None else torch.empty(r, K, dtype=torch.float32, device=dev)
    dB = dB if dB is not None else torch.empty(w.N, r, dtype=torch.float32, device=dev)
    ws = _ws(workspace_bytes(OP_BWD, M, w.N, w.K, r), dev, ws)
    v = w.c_view()
    _check(lib().qlora_linear_bwd(_ptr(dY), _ptr(X), M, ctypes.byref(v), _ptr(A), _ptr(B), r, float(alpha),
                                  _ptr(sT), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(), _stream(dev)),
           "qlora_linear_bwd")
    _after_call(ws, "qlora_linear_bwd", M)
    return dX, dA, dB


# ------------------------------------------ several adapters over one base ---

def workspace_bytes_multi(op: int, M: int, N: int, K: int, r: int, P: int) -> int:
    return int(lib().qlora_workspace_bytes_multi(op, M, N, K, r, P))


def linear_fwd_multi(X: torch.Tensor, w: NF4Weight, A: torch.Tensor, B: torch.Tensor, ids: torch.Tensor, P: int,
                     alpha: float, Y: torch.Tensor | None = None, sT: torch.Tensor | None = None,
                     save_sT: bool = True, ws: torch.Tensor | None = None):
    """(Y, sT) of a batch whose token row m uses adapter ids[m] (int32; an id
    outside [0, P) uses none). A: bf16 [P r, K] (the A_k stacked); B: bf16
    [N, P r] (the B_k side by side); sT: bf16 [M, P r], zero outside the
    row's own adapter."""
    M, K = X.shape
    R = A.shape[0]
    r = R // P
    assert ids.dtype == torch.int32 and ids.numel() == M and B.shape == (w.N, R)
    dev = X.device
    Y = Y if Y is not None else torch.empty(M, w.N, dtype=torch.bfloat16, device=dev)
    if save_sT and sT is None:
        sT = torch.empty(M, R, dtype=torch.bfloat16, device=dev)
    ws = _ws(workspace_bytes_multi(OP_FWD, M, w.N, w.K, r, P), dev, ws)
    v = w.c_view()
    _check(lib().qlora_linear_fwd_multi(_ptr(X), M, ctypes.byref(v), _ptr(A), _ptr(B), r, P, _ptr(ids),
                                        float(alpha), _ptr(Y), _ptr(sT) if save_sT else None, _ptr(ws), ws.numel(),
                                        _stream(dev)), "qlora_linear_fwd_multi")
    _after_call(ws, "qlora_linear_fwd_multi", M)
    return Y, (sT if save_sT else None)


def linear_bwd_multi(dY: torch.Tensor, X: torch.Tensor, w: NF4Weight, A: torch.Tensor, B: torch.Tensor,
                     ids: torch.Tensor, P: int, alpha: float, sT: torch.Tensor | None = None,
                     dX: torch.Tensor | None = None, dA: torch.Tensor | None = None,
                     dB: torch.Tensor | None = None, ws: torch.Tensor | None = None):
    """(dX, dA fp32 [P r, K], dB fp32 [N, P r]) of linear_fwd_multi: every
    adapter's gradients from the rows that use it."""
    M, K = X.shape
    R = A.shape[0]
    r = R // P
    dev = X.device
    dX = dX if dX is not None else torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dA = dA if dA is not None else torch.empty(R, K, dtype=torch.float32, device=dev)
    dB = dB if dB is not None else torch.empty(w.N, R, dtype=torch.float32, device=dev)
    ws = _ws(workspace_bytes_multi(OP_BWD, M, w.N, w.K, r, P), dev, ws)
    v = w.c_view()
    _check(lib().qlora_linear_bwd_multi(_ptr(dY), _ptr(X), M, ctypes.byref(v), _ptr(A), _ptr(B), r, P, _ptr(ids),
                                        float(alpha), _ptr(sT), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(),
                                        _stream(dev)), "qlora_linear_bwd_multi")
    _after_call(ws, "qlora_linear_bwd_multi", M)
    return dX, dA, dB


# ------------------------------------------ projections sharing one input ---

def empty_group(Ns, K: int, device) -> list:
    """Buffers for the NF4 weights of a group (N_i x K each, double
    quantisation): one codes allocation sliced back to back, as the group
    calls require; each weight is quantised into its own view."""
    szs = [nf4_bytes(n, K) for n in Ns]
    codes = torch.empty(sum(s["codes"] for s in szs), dtype=torch.uint8, device=device)
    out, at = [], 0
    for n, sz in zip(Ns, szs):
        out.append(NF4Weight(codes[at:at + sz["codes"]], torch.empty(sz["qabsmax"], dtype=torch.uint8, device=device),
                             torch.empty(sz["s2"] // 4, dtype=torch.float32, device=device),
                             torch.empty(1, dtype=torch.float32, device=device), n, K))
        at += sz["codes"]
    return out


def _group_view(ws_: list):
    arr = (Nf4WeightC * len(ws_))()
    for i, w in enumerate(ws_):
        arr[i] = w.c_view()
    return arr


def workspace_bytes_group(op: int, M: int, Ns, K: int, r: int) -> int:
    n = (_i64 * len(Ns))(*Ns)
    return int(lib().qlora_workspace_bytes_group(op, M, n, len(Ns), K, r))


def linear_fwd_group(X: torch.Tensor, group: list, A: torch.Tensor, B: torch.Tensor, alpha: float,
                     Y: torch.Tensor | None = None, sT: torch.Tensor | None = None, save_sT: bool = True,
                     ws: torch.Tensor | None = None):
    """(Y, sT) of projections sharing X: Y = [Y_0 | Y_1 | ...] bf16 [M, sum N_i].
    A: bf16 [P r, K] (the A_i stacked); B: bf16 [sum N_i, r] (the B_i stacked);
    sT: bf16 [M, P r]."""
    M, K = X.shape
    P = len(group)
    R = A.shape[0]
    r = R // P
    Ns = [w.N for w in group]
    Nt = sum(Ns)
    dev = X.device
    Y = Y if Y is not None else torch.empty(M, Nt, dtype=torch.bfloat16, device=dev)
    if save_sT and sT is None:
        sT = torch.empty(M, R, dtype=torch.bfloat16, device=dev)
    ws = _ws(workspace_bytes_group(OP_FWD, M, Ns, K, r), dev, ws)
    arr = _group_view(group)
    _check(lib().qlora_linear_fwd_group(_ptr(X), M, arr, P, _ptr(A), _ptr(B), r, float(alpha), _ptr(Y),
                                        _ptr(sT) if save_sT else None, _ptr(ws), ws.numel(), _stream(dev)),
           "qlora_linear_fwd_group")
    _after_call(ws, "qlora_linear_fwd_group", M)
    return Y, (sT if save_sT else None)


def linear_bwd_group(dY: torch.Tensor, X: torch.Tensor, group: list, A: torch.Tensor, B: torch.Tensor,
                     alpha: float, sT: torch.Tensor | None = None, dX: torch.Tensor | None = None,
                     dA: torch.Tensor | None = None, dB: torch.Tensor | None = None, ws: torch.Tensor | None = None):
    """(dX, dA fp32 [P r, K], dB fp32 [sum N_i, r]) of linear_fwd_group."""
    M, K = X.shape
    P = len(group)
    R = A.shape[0]
    r = R // P
    Ns = [w.N for w in group]
    dev = X.device
    dX = dX if dX is not None else torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dA = dA if dA is not None else torch.empty(R, K, dtype=torch.float32, device=dev)
    dB = dB if dB is not None else torch.empty(sum(Ns), r, dtype=torch.float32, device=dev)
    ws = _ws(workspace_bytes_group(OP_BWD, M, Ns, K, r), dev, ws)
    arr = _group_view(group)
    _check(lib().qlora_linear_bwd_group(_ptr(dY), _ptr(X), M, arr, P, _ptr(A), _ptr(B), r, float(alpha), _ptr(sT),
                                        _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(), _stream(dev)),
           "qlora_linear_bwd_group")
    _after_call(ws, "qlora_linear_bwd_group", M)
    return dX, dA, dB


def device_status(ws: torch.Tensor) -> int:
    out = _int(0)
    _check(lib().qlora_device_status(_ptr(ws), ctypes.byref(out), _stream(ws.device)), "qlora_device_status")
    return out.value


def call_status(device=None) -> int:
    """Status word of the calls without a workspace (the adapter merge), read
    and cleared: QLORA_OK, or QLORA_ERR_DEVICE_TIMEOUT after a wait ran out."""
    out = _int(0)
    _check(lib().qlora_device_status(None, ctypes.byref(out), _stream(device)), "qlora_device_status")
    return out.value


def profile_next_launch(kernel: int, start: torch.cuda.Event, stop: torch.cuda.Event):
    """Record start/stop around the next launch of a fused matmul kernel."""
    _check(lib().qlora_profile_next_launch(kernel, start.cuda_event, stop.cuda_event),
           "qlora_profile_next_launch")


def launch_count() -> int:
    return get_option(OPT_LAUNCH_COUNT)


def e4m3_encode(x: torch.Tensor) -> torch.Tensor:
    assert x.dtype == torch.float32 and x.is_cuda
    q = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    _check(lib().qlora_e4m3_encode(_ptr(x), _ptr(q), x.numel(), _stream(x.device)), "qlora_e4m3_encode")
    return q
