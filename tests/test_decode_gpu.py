"""Parity of the paged split-KV decode kernels (split + LSE combine) and the
fp32 debug path with the fp64 oracle, through the C ABI, on seeded inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_86_b200 import api, inputs
from parity import (BF16_MAX_ABS, BF16_MEAN_ABS, F32_ABS, LSE_ABS, check_bf16, check_bf16_plain,
                    check_close, to_np)

pytestmark = pytest.mark.gpu


def to_dev(inp):
    return [t.cuda() for t in (inp.q, inp.k_pages, inp.v_pages, inp.block_table, inp.seq_lens)]


def run_gpu(inp, num_splits):
    q, kp, vp, bt, sl = to_dev(inp)
    o, lse = api.decode_paged(q, kp, vp, bt, sl, num_splits=num_splits, scale=inp.scale)
    torch.cuda.synchronize()
    assert api.device_error() == api.FA_OK
    return to_np(o), to_np(lse)


def reference(inp):
    return oracle.decode_paged(inp.q, inp.k_pages, inp.v_pages, inp.block_table, inp.seq_lens,
                               inp.scale)


def assert_decode_matches(inp, num_splits, plain=False):
    o, lse = run_gpu(inp, num_splits)
    o_ref, lse_ref = reference(inp)
    (check_bf16_plain if plain else check_bf16)(o, o_ref, f"O (splits={num_splits})")
    check_close(lse, lse_ref, LSE_ABS, None, f"LSE (splits={num_splits})")
    return o, lse


CASES = [
    # seq_lens, Hq, Hkv, d, page_size
    ([1, 15, 16, 17, 100, 1000, 0, 333], 32, 8, 128, 16),
    ([1, 15, 16, 17, 100, 1000, 0, 333], 32, 8, 64, 16),
    ([5000, 64, 65], 4, 1, 128, 64),
    ([777, 1, 2048], 8, 8, 128, 32),
    ([4096], 16, 2, 64, 16),
    ([300, 301], 1, 1, 128, 16),
    ([129, 4000, 17], 24, 3, 128, 16),
    # wide groups: MQA 32:1 and GQA 16:1 (several query tiles per kv head),
    # 64:1 (eight tiles), 128:1 (two chunks of eight tiles), 12:1 (a ragged tile)
    ([2000, 33, 0, 517], 32, 1, 128, 16),
    ([1500, 16, 700], 32, 2, 128, 16),
    ([900, 65], 64, 1, 128, 64),
    ([600, 31], 128, 1, 64, 16),
    ([450, 1, 1000], 36, 3, 128, 16),
    # page sizes that are not multiples of 16: the per-token gather, stages
    # that span pages
    ([1, 2, 17, 300, 1031], 32, 8, 128, 1),
    ([5, 16, 33, 777], 8, 2, 128, 3),
    ([8, 9, 640, 2049], 32, 8, 128, 8),
    ([23, 24, 25, 1000], 16, 4, 64, 24),
    ([70, 1234], 32, 1, 128, 5),
]


_case_cache = {}


def case_inputs(case):
    if case not in _case_cache:
        seq_lens, Hq, Hkv, d, ps = CASES[case]
        inp = inputs.make_decode(seq_lens, Hq, Hkv, d, ps, seed=6000 + case)
        _case_cache[case] = (inp, reference(inp))
    return _case_cache[case]


@pytest.mark.parametrize("num_splits", [1, 2, 7, 0])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_small(case, num_splits):
    inp, (o_ref, lse_ref) = case_inputs(case)
    o, lse = run_gpu(inp, num_splits)
    check_bf16(o, o_ref, "O")
    check_close(lse, lse_ref, LSE_ABS, None, "LSE")


def test_split_count_does_not_change_the_result_beyond_rounding():
    inp = inputs.make_decode([3000, 1500, 70], 32, 8, 128, 16, seed=6100)
    outs = [run_gpu(inp, s) for s in (1, 2, 3, 16, 64, 0)]
    for o, lse in outs[1:]:
        check_close(o, outs[0][0], 2 * BF16_MAX_ABS, BF16_MEAN_ABS, "O across splits")
        check_close(lse, outs[0][1], LSE_ABS, None, "LSE across splits")


def test_more_splits_than_pages():
    inp = inputs.make_decode([20, 40], 8, 2, 128, 16, seed=6101)
    assert_decode_matches(inp, 9)


def test_page_permutation_is_invisible():
    """The same context in a differently permuted pool gives the same output."""
    inp = inputs.make_decode([500, 47], 8, 2, 128, 16, seed=6102)
    o1, l1 = run_gpu(inp, 4)
    perm = torch.randperm(inp.num_pages, generator=torch.Generator().manual_seed(1))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(inp.num_pages)
    inp2 = inputs.DecodeInputs("perm", inp.q, inp.k_pages[perm], inp.v_pages[perm],
                               torch.where(inp.block_table >= 0, inv[inp.block_table.clamp(min=0).long()].int(), inp.block_table),
                               inp.seq_lens, inp.page_size, inp.scale)
    o2, l2 = run_gpu(inp2, 4)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


@pytest.mark.parametrize("ps", [1, 2, 3, 8, 24])
def test_bad_block_table_entry_with_the_per_token_gather(ps):
    """Page sizes that are not multiples of 16 gather token by token: a used
    entry outside the pool is read as zeros, never dereferenced, and
    FA_ERR_DEVICE_BOUNDS is recorded; the other request is exact."""
    inp = inputs.make_decode([64, 64], 8, 2, 128, ps, seed=6103 + ps)
    q, kp, vp, bt, sl = to_dev(inp)
    bt[0, 1] = inp.num_pages + 7
    o, lse = api.decode_paged(q, kp, vp, bt, sl, num_splits=2)
    assert api.device_error() == api.FA_ERR_DEVICE_BOUNDS
    assert torch.isfinite(o.float()).all()
    o_ref, lse_ref = reference(inp)
    check_bf16(to_np(o)[1:], o_ref[1:], "O, request with valid entries")
    check_close(to_np(lse)[1:], lse_ref[1:], LSE_ABS, None, "LSE, request with valid entries")


def test_empty_pool_and_empty_batch():
    """num_pages = 0 with every context empty is valid: O = 0 and LSE = -inf,
    and no page is read (the pool pointer is non-null, its page count 0)."""
    import ctypes
    B, Hq, Hkv, d, ps = 3, 8, 2, 128, 16
    q = torch.randn(B, Hq, d, device="cuda").to(torch.bfloat16)
    pool = torch.zeros(16, dtype=torch.bfloat16, device="cuda")  # never read
    bt = torch.full((B, 4), -1, dtype=torch.int32, device="cuda")
    sl = torch.zeros(B, dtype=torch.int32, device="cuda")
    lib = api.load_library()
    for splits in (1, 3, 0):
        S = splits or api.decode_auto_splits(B, Hq, Hkv, 4, ps)
        ws = torch.empty(max(api.decode_workspace_size(B, Hq, d, S), 1), dtype=torch.uint8,
                         device="cuda")
        o = torch.full((B, Hq, d), 7.0, dtype=torch.bfloat16, device="cuda")
        lse = torch.zeros(B, Hq, dtype=torch.float32, device="cuda")
        ptr = lambda t: ctypes.c_void_p(t.data_ptr())
        st = lib.fa_decode_paged(ptr(q), ptr(pool), ptr(pool), ptr(bt), ptr(sl), ps, splits, ptr(o),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), B, Hq,
                                 Hkv, d, 4, 0, 0.0, ptr(lse), ptr(ws), ws.numel())
        assert st == api.FA_OK
        assert api.device_error() == api.FA_OK
        assert torch.count_nonzero(o) == 0
        assert torch.isneginf(lse).all()


def test_bad_block_table_entry_reports_bounds_error():
    """A used block-table entry outside the pool is never dereferenced: the
    gather reads zeros for it and FA_ERR_DEVICE_BOUNDS is recorded."""
    inp = inputs.make_decode([64, 64], 4, 1, 128, 16, seed=6104)
    q, kp, vp, bt, sl = to_dev(inp)
    bt[0, 2] = inp.num_pages + 5
    bt[1, 0] = -3
    o, _ = api.decode_paged(q, kp, vp, bt, sl, num_splits=2)
    assert api.device_error() == api.FA_ERR_DEVICE_BOUNDS
    assert torch.isfinite(o.float()).all()


def test_caller_workspace_and_lse_optional():
    inp = inputs.make_decode([900, 17], 32, 8, 128, 16, seed=6105)
    q, kp, vp, bt, sl = to_dev(inp)
    S = 5
    ws = torch.empty(api.decode_workspace_size(2, 32, 128, S), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(q)
    api.fa_decode_paged(q, kp, vp, bt, sl, S, o, None, inp.scale, ws)
    o_ref, _ = reference(inp)
    check_bf16(to_np(o), o_ref, "O with caller workspace")
    # library-allocated (stream-ordered) workspace
    o2 = torch.empty_like(q)
    api.fa_decode_paged(q, kp, vp, bt, sl, S, o2, None, inp.scale, None)
    assert torch.equal(o, o2)


@pytest.mark.parametrize("ps", [1, 3, 16])
def test_fp32_debug_path(ps):
    seq_lens = [1, 40, 0, 129]
    Hq, Hkv, d = 8, 2, 64
    gen = torch.Generator().manual_seed(6200 + ps)
    bt, num_pages = inputs.paged_layout(seq_lens, ps, gen)
    q = inputs.randn_f32((4, Hq, d), gen)
    kp = inputs.randn_f32((num_pages, ps, Hkv, d), gen)
    vp = inputs.randn_f32((num_pages, ps, Hkv, d), gen)
    sl = torch.tensor(seq_lens, dtype=torch.int32)
    o, lse = api.decode_paged_f32(q.cuda(), kp.cuda(), vp.cuda(), bt.cuda(), sl.cuda(), scale=0.125)
    o_ref, lse_ref = oracle.decode_paged(q, kp, vp, bt, sl, 0.125)
    check_close(to_np(o), o_ref, F32_ABS, None, "O fp32")
    check_close(to_np(lse), lse_ref, F32_ABS, None, "LSE fp32")


# ---- full-size workloads, checked in full with the plain bounds ------------
def test_paged_decode_full_size():
    inp = inputs.paged_decode()
    assert_decode_matches(inp, 0, plain=True)


def test_long_decode_full_size():
    inp = inputs.long_decode()
    o, lse = assert_decode_matches(inp, 0, plain=True)
    o1, lse1 = run_gpu(inp, 1)  # one split walks the whole 131072-token context
    o_ref, lse_ref = reference(inp)
    check_bf16_plain(o1, o_ref, "O one split")
    check_close(lse1, lse_ref, LSE_ABS, None, "LSE one split")
