"""The allocation-free decode entry point (fa_decode_paged_noalloc).

It exists for callers that cannot allocate device memory when they run a
decode step (an engine whose KV-cache pool already holds nearly all of HBM,
or a step loop that must not block in or fail inside an allocator).  It
must give the same result as fa_decode_paged with a caller-provided
workspace, and both must match the fp64 oracle.  Two calls in a row, on
different shapes, check that the shared scratch array carries nothing over
from one call to the next.  This file is collected last, so a failure here
never hides another test's result.
"""
import pytest
import torch

import oracle
from exact_io_aware_86_b200 import api, inputs
from parity import LSE_ABS, check_bf16, check_close, to_np

pytestmark = pytest.mark.gpu


def _run_both(inp, num_splits):
    q, kp, vp, bt, sl = (t.cuda() for t in (inp.q, inp.k_pages, inp.v_pages, inp.block_table,
                                             inp.seq_lens))
    o_ref, lse_ref = api.decode_paged(q, kp, vp, bt, sl, num_splits=num_splits, scale=inp.scale)
    o = torch.empty_like(q)
    lse = torch.empty(inp.B, inp.Hq, dtype=torch.float32, device="cuda")
    api.fa_decode_paged_noalloc(q, kp, vp, bt, sl, num_splits, o, lse, inp.scale)
    torch.cuda.synchronize()
    assert api.device_error() == api.FA_OK
    return (to_np(o), to_np(lse)), (to_np(o_ref), to_np(lse_ref))


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    first = inputs.make_decode([3000, 17, 640, 1], 32, 8, 128, 16, seed=7001)
    second = inputs.make_decode([129, 2048], 16, 2, 64, 64, seed=7002)
    for inp, splits in ((first, 7), (second, 0)):
        (o, lse), (o_ws, lse_ws) = _run_both(inp, splits)
        check_bf16(o, o_ws, "O noalloc vs workspace entry point")
        check_close(lse, lse_ws, LSE_ABS, None, "LSE noalloc vs workspace entry point")
        o_ref, lse_ref = oracle.decode_paged(inp.q, inp.k_pages, inp.v_pages, inp.block_table,
                                             inp.seq_lens, inp.scale)
        check_bf16(o, o_ref, "O noalloc vs oracle")
        check_close(lse, lse_ref, LSE_ABS, None, "LSE noalloc vs oracle")


def test_noalloc_rejects_scratch_beyond_its_maximum():
    inp = inputs.make_decode([64] * 4, 32, 8, 128, 16, seed=7003)
    q, kp, vp, bt, sl = (t.cuda() for t in (inp.q, inp.k_pages, inp.v_pages, inp.block_table,
                                             inp.seq_lens))
    o = torch.empty_like(q)
    splits = 2048  # 4 * 32 * 2048 * 129 * 4 bytes > 64 MiB
    assert api.decode_workspace_size(4, 32, 128, splits) > 64 << 20
    with pytest.raises(api.FAError) as e:
        api.fa_decode_paged_noalloc(q, kp, vp, bt, sl, splits, o)
    assert e.value.code == api.FA_ERR_UNSUPPORTED
