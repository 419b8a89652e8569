"""The quantiser entry point that allocates nothing, for callers that cannot
allocate device memory when they quantise (plugin interfaces of inference
runtimes that pass only input and output buffers, or latency-critical code
that must not call cudaMalloc mid-step). It keeps its scratch in one static
device array, so these checks run it twice in a row through the C ABI and
compare each result with the ordinary entry point, which takes a workspace
from the caller. Quantised outputs are integer and bit patterns, so the
tolerance is exact equality, as for every quantiser test."""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    from bit_nf4_quantized_09_b200 import build
    build.build()
    import bit_nf4_quantized_09_b200 as q
    assert torch.cuda.is_available()
    q.set_option(q.OPT_FAIL_LAUNCHES, 0)
    return q


def with_workspace(q, W):
    return q.quantize_nf4(W)


def without_allocation(q, W):
    """Raw C-ABI call of qlora_quantize_nf4_noalloc into preallocated outputs."""
    N, K = W.shape
    out = q.NF4Weight.empty(N, K, W.device)
    st = torch.cuda.current_stream().cuda_stream
    rc = q.lib().qlora_quantize_nf4_noalloc(W.data_ptr(), N, K, out.codes.data_ptr(), out.qabsmax.data_ptr(),
                                            out.s2.data_ptr(), out.mean.data_ptr(), st)
    assert rc == 0, q.lib().qlora_last_error()
    return out


def same(a, b):
    for x, y in ((a.codes, b.codes), (a.qabsmax, b.qabsmax), (a.s2, b.s2), (a.mean, b.mean)):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_two_calls_in_a_row_match_the_workspace_entry_point(q):
    # two different weights back to back: the second call reuses the static
    # array the first one filled, and must not see its leftovers
    W1 = synth.weight(synth.ATTN7B).cuda()
    W2 = synth.weight(synth.custom(N=1000, K=832, M=1, r=8, seed_base=93)).cuda()
    a1 = without_allocation(q, W1)
    a2 = without_allocation(q, W2)
    b1 = with_workspace(q, W1)
    b2 = with_workspace(q, W2)
    torch.cuda.synchronize()
    same(a1, b1)
    same(a2, b2)


def test_largest_accepted_size_and_rejection(q):
    # 8192 x 8192 is exactly the limit of 67,108,864 weights
    W = synth.weight(synth.L65B[0]).cuda()
    same(without_allocation(q, W), with_workspace(q, W))
    torch.cuda.synchronize()
    # one row more is rejected before anything is launched
    n0 = q.launch_count()
    big = torch.zeros(8200, 8192, dtype=torch.float32, device="cuda")
    out = q.NF4Weight.empty(8200, 8192, big.device)
    rc = q.lib().qlora_quantize_nf4_noalloc(big.data_ptr(), 8200, 8192, out.codes.data_ptr(),
                                            out.qabsmax.data_ptr(), out.s2.data_ptr(), out.mean.data_ptr(),
                                            torch.cuda.current_stream().cuda_stream)
    assert rc == -9
    assert b"static scratch" in q.lib().qlora_last_error()
    assert q.lib().qlora_status_string(rc) == b"QLORA_ERR_EXCEEDS_STATIC_SCRATCH"
    assert q.launch_count() == n0
    assert np.isfinite(q.dequantize_nf4(without_allocation(q, W)).float().cpu().numpy()).all()


def test_python_wrapper_checks_its_outputs(q):
    """The torch wrapper of the same entry point: it matches the workspace
    entry point, and refuses an output sized for another shape before any
    launch (an undersized output would be written past its end)."""
    W = synth.weight(synth.custom(N=520, K=320, M=1, r=8, seed_base=94)).cuda()
    out = q.NF4Weight.empty(520, 320, W.device)
    same(q.quantize_nf4_noalloc(W, out), with_workspace(q, W))
    torch.cuda.synchronize()
    n0 = q.launch_count()
    with pytest.raises(AssertionError):
        q.quantize_nf4_noalloc(W, q.NF4Weight.empty(512, 320, W.device))
    strided = torch.empty(520, 640, dtype=torch.float32, device=W.device)[:, :320]   # not contiguous
    with pytest.raises(AssertionError):
        q.quantize_nf4_noalloc(strided, q.NF4Weight.empty(520, 320, W.device))
    assert q.launch_count() == n0
