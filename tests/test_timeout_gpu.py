"""The kernels' timeout path, exercised without a fault: a test hook makes
one warp of CTA 0 wait on a barrier that nothing arrives at, with the
abortable-wait limit shortened to a few milliseconds.  The kernel must
record FA_ERR_DEVICE_TIMEOUT, stop its other roles, drain its own copies and
tensor-core work, free its tensor memory and return promptly -- and the
next, normal call on the same stream must be exact.  (Every kernel wait is
bounded: this is the path a lost arrival would take.)
"""
import time

import pytest
import torch

import oracle
from exact_io_aware_86_b200 import api, inputs
from parity import LSE_ABS, check_bf16, check_close, to_np

pytestmark = pytest.mark.gpu

LIMIT_NS = 5_000_000  # 5 ms


def _with_stall(which, fn):
    api.selftest_inject_stall(which, LIMIT_NS)
    try:
        t0 = time.perf_counter()
        fn()
        code = api.device_error()
        return code, time.perf_counter() - t0
    finally:
        api.selftest_inject_stall(api.STALL_NONE, 0)


@pytest.mark.parametrize("causal", [True, False])
def test_prefill_wait_times_out_then_recovers(causal):
    inp = inputs.make_prefill([700, 129, 300], 8, 2, 128, causal, seed=8001)
    q, k, v, cu = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.cu_seqlens))
    api.prefill(q, k, v, cu, causal=causal, scale=inp.scale)  # warm-up (module load)
    assert api.device_error() == api.FA_OK
    code, dt = _with_stall(api.STALL_PREFILL,
                           lambda: api.prefill(q, k, v, cu, causal=causal, scale=inp.scale))
    assert code == api.FA_ERR_DEVICE_TIMEOUT
    assert dt < 1.0, f"the timed-out call took {dt:.3f} s"
    o, lse = api.prefill(q, k, v, cu, causal=causal, scale=inp.scale)
    torch.cuda.synchronize()
    assert api.device_error() == api.FA_OK
    o_ref, lse_ref = oracle.prefill(inp.q, inp.k, inp.v, inp.cu_seqlens, causal, inp.scale)
    check_bf16(to_np(o), o_ref, "O after the timeout")
    check_close(to_np(lse), lse_ref, LSE_ABS, None, "LSE after the timeout")


@pytest.mark.parametrize("softcap", [0.0, 20.0])
def test_prefill_variant_wait_times_out_then_recovers(softcap):
    """The mask-variant instantiations (a band alone; a band with softcap)
    take the same path."""
    inp = inputs.make_prefill([600, 77], 4, 4, 128, True, seed=8002)
    q, k, v, cu = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.cu_seqlens))
    run = lambda: api.prefill(q, k, v, cu, causal=True, scale=inp.scale, window=(100, 0),
                              softcap=softcap)
    run()
    assert api.device_error() == api.FA_OK
    code, dt = _with_stall(api.STALL_PREFILL, run)
    assert code == api.FA_ERR_DEVICE_TIMEOUT and dt < 1.0
    o, lse = run()
    assert api.device_error() == api.FA_OK
    o_ref, lse_ref = oracle.prefill(inp.q, inp.k, inp.v, inp.cu_seqlens, True, inp.scale,
                                    window=(100, 0), softcap=softcap)
    check_bf16(to_np(o), o_ref, "O after the timeout")


@pytest.mark.parametrize("ps,splits", [(16, 0), (16, 1), (5, 3)])
def test_decode_wait_times_out_then_recovers(ps, splits):
    inp = inputs.make_decode([3000, 17, 900, 1], 32, 8, 128, ps, seed=8003 + ps)
    q, kp, vp, bt, sl = (t.cuda() for t in (inp.q, inp.k_pages, inp.v_pages, inp.block_table,
                                             inp.seq_lens))
    run = lambda: api.decode_paged(q, kp, vp, bt, sl, num_splits=splits, scale=inp.scale)
    run()
    assert api.device_error() == api.FA_OK
    code, dt = _with_stall(api.STALL_DECODE, run)
    assert code == api.FA_ERR_DEVICE_TIMEOUT
    assert dt < 1.0, f"the timed-out call took {dt:.3f} s"
    o, lse = run()
    torch.cuda.synchronize()
    assert api.device_error() == api.FA_OK
    o_ref, lse_ref = oracle.decode_paged(inp.q, inp.k_pages, inp.v_pages, inp.block_table,
                                         inp.seq_lens, inp.scale)
    check_bf16(to_np(o), o_ref, "O after the timeout")
    check_close(to_np(lse), lse_ref, LSE_ABS, None, "LSE after the timeout")


def test_stall_hook_rejects_unknown_kernels():
    with pytest.raises(api.FAError) as e:
        api.selftest_inject_stall(7, 0)
    assert e.value.code == api.FA_ERR_INVALID_ARG
