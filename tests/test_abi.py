"""The C ABI without a GPU: the library loads, exports every function the
header declares, sizes its buffers as the format says, and rejects bad
arguments on the host before any CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora_nf4.h")


@pytest.fixture(scope="module")
def q():
    from bit_nf4_quantized_09_b200 import build
    build.build()
    import bit_nf4_quantized_09_b200 as q
    return q


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(q):
    L = ctypes.CDLL(q.LIB_PATH)
    names = declared_functions()
    assert len(names) >= 12
    for name in names:
        assert hasattr(L, name), name
    # and the binding knows every one of them under the same name
    assert set(names) == set(q._SIGNATURES)


def test_binding_arity_matches_header(q):
    """Every binding signature has as many arguments as the header's
    prototype, and the weight struct as many fields as qlora_nf4_weight."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    protos = re.findall(r"\b(qlora_\w+)\s*\(([^)]*)\)\s*;", text)
    assert len(protos) == len(q._SIGNATURES)
    for name, params in protos:
        params = params.strip()
        n = 0 if params in ("", "void") else len(params.split(","))
        assert len(q._SIGNATURES[name][1]) == n, name
    struct = re.search(r"typedef struct \{(.*?)\} qlora_nf4_weight;", text, flags=re.S).group(1)
    fields = [f for f in struct.split(";") if f.strip()]
    assert [f[0] for f in q.Nf4WeightC._fields_] == [f.split()[-1] for f in fields]


def test_nf4_bytes_match_oracle_storage(q):
    for N, K in [(512, 512), (4096, 4096), (11008, 4096), (8192, 22016), (8, 64)]:
        sz = q.nf4_bytes(N, K)
        assert sz["codes"] == N * K // 2
        assert sz["qabsmax"] == N * K // 64
        assert sz["s2"] == 4 * ((N * K // 64 + 255) // 256)
        assert sz["mean"] == 4
        assert sz["total"] == oracle.storage_bytes(N, K, True)
    with pytest.raises(q.QLoraError):
        q.nf4_bytes(4, 100)


def test_library_tables_equal_oracle_bit_for_bit(q):
    """The library computes the NF4 levels and thresholds on its own (Newton
    on the normal CDF); the oracle by bisection. Same fp32 bits."""
    lv, th = q.nf4_tables()
    _, L = oracle.nf4_levels()
    M = oracle.midpoints(L)
    assert np.array_equal(np.array(lv, np.float32).view(np.uint32), L.view(np.uint32))
    assert np.array_equal(np.array(th, np.float32).view(np.uint32), M.view(np.uint32))


def test_workspace_sizes(q):
    assert q.workspace_bytes(q.OP_QUANTIZE, 0, 512, 512, 0) >= 512 * 512 // 64 * 4
    assert q.workspace_bytes(q.OP_FWD, 64, 512, 512, 8) > 0
    assert q.workspace_bytes(q.OP_BWD, 4096, 4096, 4096, 16) > q.workspace_bytes(q.OP_FWD, 4096, 4096, 4096, 16)
    assert q.workspace_bytes(q.OP_FWD, 64, 512, 500, 8) == 0      # K % 64
    assert q.workspace_bytes(q.OP_FWD, 64, 512, 512, 12) == 0     # rank
    assert q.workspace_bytes(7, 64, 512, 512, 8) == 0             # op


def _weight(q, N=512, K=512, base=0x10000):
    return q.Nf4WeightC(base, base + 0x100000, base + 0x200000, base + 0x300000, N, K)


def test_host_validation_without_gpu(q):
    L = q.lib()
    w = _weight(q)
    P = 0x7000000  # fake, 16-byte aligned; never dereferenced on these paths
    ws_ok = q.workspace_bytes(q.OP_FWD, 64, 512, 512, 8)
    fwd = lambda **kw: L.qlora_linear_fwd(kw.get("X", P), kw.get("M", 64), ctypes.byref(kw.get("w", w)),
                                          kw.get("A", P), kw.get("B", P), kw.get("r", 8), kw.get("alpha", 16.0),
                                          kw.get("Y", P), None, kw.get("ws", P), kw.get("wsb", 0), None)
    assert fwd(r=12) == -4
    assert fwd(r=0) == -4
    assert fwd(X=None) == -1
    assert fwd(alpha=float("nan")) == -1
    assert fwd(X=P + 2) == -3
    assert fwd(M=-1) == -2
    assert fwd(M=0) == 0                       # empty batch: valid no-op, nothing launched
    assert fwd(w=_weight(q, K=500)) == -2       # K % 64 != 0
    assert fwd(w=_weight(q, N=12)) == -2        # N % 8 != 0
    assert fwd(w=_weight(q, base=0x10004)) == -3
    assert fwd(wsb=ws_ok - 1) == -5
    # quantize
    assert L.qlora_quantize_nf4(P, 512, 500, P, P, P, P, P, 1 << 30, None) == -2
    assert L.qlora_quantize_nf4(P, 0, 512, P, P, P, P, P, 1 << 30, None) == -2
    assert L.qlora_quantize_nf4(None, 512, 512, P, P, P, P, P, 1 << 30, None) == -1
    assert L.qlora_quantize_nf4(P, 512, 512, P, P, P, P, P, 16, None) == -5
    # dequantize
    assert L.qlora_dequantize_nf4(ctypes.byref(w), None, None) == -1
    assert L.qlora_dequantize_nf4(ctypes.byref(w), P + 8, None) == -3
    # backward
    bws = q.workspace_bytes(q.OP_BWD, 64, 512, 512, 8)
    bwd = lambda **kw: L.qlora_linear_bwd(P, P, kw.get("M", 64), ctypes.byref(w), P, P, kw.get("r", 8), 16.0,
                                          None, P, kw.get("dA", P), P, P, kw.get("wsb", bws), None)
    assert bwd(r=24) == -4
    assert bwd(dA=None) == -1
    assert bwd(dA=P + 4) == -3
    assert bwd(wsb=bws - 256) == -5
    # the status reader needs somewhere to put the word, with or without a
    # workspace (NULL reads the library's own word)
    assert L.qlora_device_status(P, None, None) == -1
    assert L.qlora_device_status(None, None, None) == -1


def test_host_validation_storage_without_dq_and_merge(q):
    L = q.lib()
    P = 0x7000000
    # a weight without double quantisation needs only codes and absmax
    nodq = q.Nf4WeightC(P, None, None, None, 512, 512, P + 0x100000)
    bad = q.Nf4WeightC(P, None, None, None, 512, 512, None)   # neither storage complete
    mis = q.Nf4WeightC(P, None, None, None, 512, 512, P + 4)
    assert L.qlora_dequantize_nf4(ctypes.byref(bad), P, None) == -1
    assert L.qlora_dequantize_nf4(ctypes.byref(mis), P, None) == -3
    assert L.qlora_dequantize_nf4(ctypes.byref(nodq), None, None) == -1
    # quantise without double quantisation
    for entry in (L.qlora_quantize_nf4_nodq, L.qlora_quantize_nf4_bf16_nodq):
        assert entry(P, 512, 500, P, P, None) == -2
        assert entry(P, 0, 512, P, P, None) == -2
        assert entry(None, 512, 512, P, P, None) == -1
        assert entry(P, 512, 512, P, None, None) == -1
        assert entry(P, 512, 512, P, P + 4, None) == -3
    # merge
    w = _weight(q)
    merge = lambda **kw: L.qlora_merge_lora(ctypes.byref(kw.get("w", w)), kw.get("A", P), kw.get("B", P),
                                            kw.get("r", 8), kw.get("alpha", 16.0), kw.get("out", P), None)
    assert merge(r=12) == -4
    assert merge(A=None) == -1
    assert merge(out=None) == -1
    assert merge(alpha=float("inf")) == -1
    assert merge(B=P + 2) == -3
    assert merge(w=bad) == -1
    assert merge(w=_weight(q, N=12)) == -2


def test_host_fault_injection(q):
    """An injected launch failure is reported as QLORA_ERR_CUDA with its text,
    and nothing reaches a GPU (none is needed for this test)."""
    L = q.lib()
    w = _weight(q)
    P = 0x7000000
    ws = q.workspace_bytes(q.OP_FWD, 64, 512, 512, 8)
    q.set_option(q.OPT_FAIL_LAUNCHES, 1)
    try:
        s = L.qlora_linear_fwd(P, 64, ctypes.byref(w), P, P, 8, 16.0, P, None, P, ws, None)
        assert s == -6
        assert b"injected" in L.qlora_last_error()
        assert q.get_option(q.OPT_FAIL_LAUNCHES) == 0
    finally:
        q.set_option(q.OPT_FAIL_LAUNCHES, 0)


def test_status_strings_and_options(q):
    L = q.lib()
    for code, name in q.STATUS.items():
        assert L.qlora_status_string(code).decode() == name
    assert L.qlora_status_string(-99).decode() == "QLORA_ERR_UNKNOWN"
    old = q.get_option(q.OPT_WAIT_TIMEOUT_US)
    q.set_option(q.OPT_WAIT_TIMEOUT_US, 5000)
    assert q.get_option(q.OPT_WAIT_TIMEOUT_US) == 5000
    q.set_option(q.OPT_WAIT_TIMEOUT_US, old)
    with pytest.raises(q.QLoraError):
        q.set_option(q.OPT_WAIT_TIMEOUT_US, 0)
    with pytest.raises(q.QLoraError):
        q.set_option(99, 1)


def test_missing_library_fails_loudly():
    """Without the built library every call raises: there is no CPU path.
    Run in a fresh interpreter with the library path pointed elsewhere."""
    import subprocess
    import sys
    code = ("import bit_nf4_quantized_09_b200 as q\n"
            "q.LIB_PATH = '/nonexistent/libqlora_nf4.so'\n"
            "q._lib = None\n"
            "try:\n"
            "    q.nf4_tables()\n"
            "except ImportError as e:\n"
            "    print('raised', 'no CPU fallback' in str(e))\n")
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.stdout.strip() == "raised True", out.stdout + out.stderr


def test_host_validation_several_adapters(q):
    """qlora_linear_{fwd,bwd}_multi: P adapters of rank r (P r <= 256) and a
    per-row id array, checked on the host before any CUDA call."""
    L = q.lib()
    w = _weight(q)
    P = 0x7000000
    ws = q.workspace_bytes_multi(q.OP_FWD, 64, 512, 512, 16, 3)
    assert ws > 0
    assert q.workspace_bytes_multi(q.OP_FWD, 64, 512, 512, 16, 17) == 0   # P r > 256
    assert q.workspace_bytes_multi(q.OP_FWD, 64, 512, 512, 12, 2) == 0    # rank
    assert q.workspace_bytes_multi(q.OP_BWD, 64, 512, 512, 64, 4) > q.workspace_bytes(q.OP_BWD, 64, 512, 512, 64)

    def fwd(**kw):
        return L.qlora_linear_fwd_multi(P, kw.get("M", 64), ctypes.byref(w), P, P, kw.get("r", 16), kw.get("P", 3),
                                        kw.get("ids", P), 16.0, P, None, P, kw.get("wsb", ws), None)
    assert fwd(P=0) == -1
    assert fwd(P=17) == -4
    assert fwd(r=24) == -4
    assert fwd(ids=None) == -1
    assert fwd(ids=P + 2) == -3
    assert fwd(M=0, ids=None) == 0
    assert fwd(wsb=ws - 1) == -5
    bws = q.workspace_bytes_multi(q.OP_BWD, 64, 512, 512, 16, 3)

    def bwd(**kw):
        return L.qlora_linear_bwd_multi(P, P, 64, ctypes.byref(w), P, P, 16, kw.get("P", 3), kw.get("ids", P), 16.0,
                                        None, P, P, P, P, kw.get("wsb", bws), None)
    assert bwd(ids=None) == -1
    assert bwd(P=20) == -4
    assert bwd(wsb=bws - 256) == -5


def test_host_validation_projection_group(q):
    """qlora_linear_{fwd,bwd}_group: up to four weights with one K and one
    storage form whose codes lie back to back in one buffer."""
    L = q.lib()
    P = 0x7000000
    K = 512

    def group(Ns, gap=0, Ks=None, nodq=()):
        arr = (q.Nf4WeightC * len(Ns))()
        at = P
        for i, n in enumerate(Ns):
            k = Ks[i] if Ks else K
            arr[i] = q.Nf4WeightC(at, P + 0x1000000 * (i + 1), P + 0x1100000 * (i + 1), P + 0x1200000 * (i + 1), n, k,
                                  P + 0x1300000 * (i + 1) if i in nodq else None)
            at += n * k // 2 + gap
        return arr
    Ns = [512, 256, 264]
    n_arr = (ctypes.c_int64 * 3)(*Ns)
    ws = L.qlora_workspace_bytes_group(q.OP_FWD, 64, n_arr, 3, K, 16)
    assert ws > 0
    assert L.qlora_workspace_bytes_group(q.OP_FWD, 64, n_arr, 5, K, 16) == 0
    assert L.qlora_workspace_bytes_group(q.OP_FWD, 64, n_arr, 3, K, 12) == 0

    def fwd(arr, nw=3, wsb=ws):
        return L.qlora_linear_fwd_group(P, 64, arr, nw, P, P, 16, 16.0, P, None, P, wsb, None)
    assert fwd(group(Ns), wsb=ws - 1) == -5
    assert fwd(group(Ns, gap=16)) == -1                       # codes not back to back
    assert b"back to back" in L.qlora_last_error()
    assert fwd(group(Ns, Ks=[512, 512, 448])) == -2           # K differs
    assert fwd(group(Ns, nodq=(1,))) == -1                    # storage differs
    assert fwd(group([512, 256, 12])) == -2                   # N % 8
    assert fwd(group(Ns), nw=0) == -1
    assert fwd(group(Ns + [256, 256]), nw=5) == -1            # at most four projections
    bws = L.qlora_workspace_bytes_group(q.OP_BWD, 64, n_arr, 3, K, 16)
    assert L.qlora_linear_bwd_group(P, P, 64, group(Ns, gap=16), 3, P, P, 16, 16.0, None, P, P, P, P, bws,
                                    None) == -1
    assert L.qlora_linear_bwd_group(P, P, 64, group(Ns), 3, P, P, 16, 16.0, None, P, None, P, P, bws, None) == -1
