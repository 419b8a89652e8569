"""Failure detection on the GPU without a GPU fault: a pipeline wait that
runs out records QLORA_ERR_DEVICE_TIMEOUT in the workspace status word and
the kernel returns; the context stays usable for the next call."""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    from bit_nf4_quantized_09_b200 import build
    build.build()
    import bit_nf4_quantized_09_b200 as q
    return q


def test_stalled_producer_times_out_and_context_survives(q):
    cfg = synth.custom(N=512, K=512, M=256, r=8)   # M > 64: the tiled fused kernel
    W = synth.weight(cfg).cuda()
    X, A, B = synth.activations(cfg).cuda(), synth.lora_a(cfg).cuda(), synth.lora_b(cfg).cuda()
    w = q.quantize_nf4(W)
    ws = torch.empty(q.workspace_bytes(q.OP_FWD, cfg.M, cfg.N, cfg.K, cfg.r), dtype=torch.uint8, device="cuda")
    Y_ref, _ = q.linear_fwd(X, w, A, B, cfg.alpha, ws=ws)
    assert q.device_status(ws) == 0
    old = q.get_option(q.OPT_WAIT_TIMEOUT_US)
    try:
        q.set_option(q.OPT_WAIT_TIMEOUT_US, 200_000)     # 0.2 s per wait
        q.set_option(q.OPT_STALL_PRODUCER, 1)            # the next tiled GEMM loads nothing
        Y = torch.full_like(Y_ref, 3.0)
        q.set_check_device_status(False)                 # the status is read explicitly here
        q.linear_fwd(X, w, A, B, cfg.alpha, Y=Y, ws=ws)
        assert q.device_status(ws) == -7                 # QLORA_ERR_DEVICE_TIMEOUT
        assert q.get_option(q.OPT_STALL_PRODUCER) == 0   # one-shot
        assert torch.all(Y == 3.0)                       # the aborted kernel wrote nothing
    finally:
        q.set_option(q.OPT_WAIT_TIMEOUT_US, old)
        q.set_option(q.OPT_STALL_PRODUCER, 0)
        q.set_check_device_status(True)
    Y2, _ = q.linear_fwd(X, w, A, B, cfg.alpha, ws=ws)
    assert q.device_status(ws) == 0
    assert torch.equal(Y2, Y_ref)


def test_injected_launch_failure_then_recovery(q):
    cfg = synth.TINY
    w = q.quantize_nf4(synth.weight(cfg).cuda())
    X, A, B = synth.activations(cfg).cuda(), synth.lora_a(cfg).cuda(), synth.lora_b(cfg).cuda()
    q.set_option(q.OPT_FAIL_LAUNCHES, 2)
    with pytest.raises(q.QLoraError) as ei:
        q.linear_fwd(X, w, A, B, cfg.alpha)
    assert ei.value.status == -6
    q.set_option(q.OPT_FAIL_LAUNCHES, 0)
    Y, _ = q.linear_fwd(X, w, A, B, cfg.alpha)
    torch.cuda.synchronize()
    assert torch.isfinite(Y.float()).all()


def test_checked_wrapper_raises_on_a_timed_out_wait(q):
    """With the status check on (as in every GPU test), a forward whose
    pipeline wait runs out raises QLORA_ERR_DEVICE_TIMEOUT from the wrapper."""
    cfg = synth.custom(N=512, K=512, M=256, r=8)
    w = q.quantize_nf4(synth.weight(cfg).cuda())
    X, A, B = synth.activations(cfg).cuda(), synth.lora_a(cfg).cuda(), synth.lora_b(cfg).cuda()
    old = q.get_option(q.OPT_WAIT_TIMEOUT_US)
    try:
        q.set_option(q.OPT_WAIT_TIMEOUT_US, 200_000)
        q.set_option(q.OPT_STALL_PRODUCER, 1)
        with pytest.raises(q.QLoraError) as ei:
            q.linear_fwd(X, w, A, B, cfg.alpha)
        assert ei.value.status == -7
    finally:
        q.set_option(q.OPT_WAIT_TIMEOUT_US, old)
        q.set_option(q.OPT_STALL_PRODUCER, 0)
    Y, _ = q.linear_fwd(X, w, A, B, cfg.alpha)
    torch.cuda.synchronize()
    assert torch.isfinite(Y.float()).all()
