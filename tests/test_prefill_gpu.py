"""Parity of the tcgen05 prefill kernel (and the fp32 debug path) with the
fp64 oracle, through the C ABI, on seeded inputs.

Small shapes span several 128-row tiles with ragged tails and zero-length
sequences; the full workloads (causal MHA B=4 H=16 L=2048 d=128, and the
varlen GQA batch) are checked on sampled rows, which the oracle computes
exactly one by one.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_86_b200 import api, inputs
from parity import (BF16_MAX_ABS, BF16_MEAN_ABS, F32_ABS, LSE_ABS, check_bf16, check_bf16_peaked,
                    check_bf16_plain, check_close, to_np)

pytestmark = pytest.mark.gpu


def run_gpu(inp, causal=None):
    causal = inp.causal if causal is None else causal
    dev = "cuda"
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    cu = inp.cu_seqlens.to(dev)
    o, lse = api.prefill(q, k, v, cu, causal=causal, scale=inp.scale,
                         max_seqlen=max(inp.lengths) if inp.lengths else 0)
    torch.cuda.synchronize()
    assert api.device_error() == api.FA_OK
    return to_np(o), to_np(lse)


def assert_prefill_matches(inp, causal=None):
    causal = inp.causal if causal is None else causal
    o, lse = run_gpu(inp, causal)
    o_ref, lse_ref = oracle.prefill(inp.q, inp.k, inp.v, inp.cu_seqlens, causal, inp.scale)
    check_bf16(o, o_ref, "O")
    check_close(lse, lse_ref, LSE_ABS, None, "LSE")


# ---- the tiny exact-attention check: B=1 H=1 L=256 d=64 -------------------
@pytest.mark.parametrize("causal", [False, True])
def test_tiny_bf16(causal):
    """The tiny workload with the plain bounds (no rounding floor)."""
    inp = inputs.tiny(causal)
    o, lse = run_gpu(inp)
    o_ref, lse_ref = oracle.prefill(inp.q, inp.k, inp.v, inp.cu_seqlens, causal, inp.scale)
    check_bf16_plain(o, o_ref, "O")
    check_close(lse, lse_ref, LSE_ABS, None, "LSE")


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_fp32_debug_path(causal):
    inp = inputs.tiny(causal)
    q, k, v = (t.cuda() for t in (inp.q32, inp.k32, inp.v32))
    o, lse = api.prefill_f32(q, k, v, inp.cu_seqlens.cuda(), causal=causal, scale=inp.scale)
    o_ref, lse_ref = oracle.prefill(inp.q32, inp.k32, inp.v32, inp.cu_seqlens, causal, inp.scale)
    check_close(to_np(o), o_ref, F32_ABS, None, "O fp32")
    check_close(to_np(lse), lse_ref, F32_ABS, None, "LSE fp32")


# ---- single sequences across tile boundaries -------------------------------
HEADS = [(1, 1), (2, 1), (4, 4), (8, 2), (32, 8)]
LENGTHS = [1, 2, 3, 15, 16, 17, 127, 128, 129, 255, 256, 257, 383, 512, 700]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("L", LENGTHS)
def test_single_sequence(L, causal, d):
    Hq, Hkv = HEADS[(L + d) % len(HEADS)]
    inp = inputs.make_prefill([L], Hq, Hkv, d, causal, seed=2000 + L + d)
    assert_prefill_matches(inp)


# ---- packed varlen batches --------------------------------------------------
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("lengths,Hq,Hkv", [
    ([0, 1, 300, 0, 129, 513, 64, 1000], 4, 2),
    ([256, 256, 256], 8, 8),
    ([17, 0, 0, 255, 1, 2], 8, 1),
    ([1500, 37], 32, 8),
])
def test_varlen(lengths, Hq, Hkv, causal, d):
    inp = inputs.make_prefill(lengths, Hq, Hkv, d, causal, seed=3000 + sum(lengths) + d)
    assert_prefill_matches(inp)


def test_more_items_than_one_cta_holds():
    """2048 one- and two-token sequences plus two long ones, 16 query heads:
    about 33k work items, more than 148 CTAs can list, so the launch widens
    the grid past one CTA per SM.  Every row is checked.  The rows of the
    one- and two-token sequences are (nearly) single rows of V, up to |O| ~ 5,
    where the bf16 spacing alone (2^-5 on [4, 8)) exceeds the plain bound: they
    take the peaked-row bound; the long sequences' rows the plain one."""
    lengths = [1, 2] * 1024 + [1000, 513]
    inp = inputs.make_prefill(lengths, 16, 4, 128, True, seed=4005)
    o, lse = run_gpu(inp)
    o_ref, lse_ref = oracle.prefill(inp.q, inp.k, inp.v, inp.cu_seqlens, True, inp.scale)
    tiny = 3 * 1024
    check_bf16_peaked(o[:tiny], o_ref[:tiny], "O, one- and two-token sequences")
    check_bf16(o[tiny:], o_ref[tiny:], "O, long sequences")
    check_close(lse, lse_ref, LSE_ABS, None, "LSE")


def test_varlen_equals_separate_calls():
    lengths = [300, 129, 700]
    inp = inputs.make_prefill(lengths, 8, 2, 128, True, seed=4001)
    o_all, lse_all = run_gpu(inp)
    start = 0
    for L in lengths:
        sub = inputs.PrefillInputs("sub", inp.q[start:start + L], inp.k[start:start + L],
                                   inp.v[start:start + L], inputs.cu_seqlens_of([L]), [L], True,
                                   inp.scale)
        o, lse = run_gpu(sub)
        check_close(o, o_all[start:start + L], 0.0, None, "O isolation")
        check_close(lse, lse_all[:, start:start + L], 0.0, None, "LSE isolation")
        start += L


def test_default_scale_is_inverse_sqrt_d():
    inp = inputs.make_prefill([200], 2, 2, 128, True, seed=4002)
    dev = "cuda"
    q, k, v, cu = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.cu_seqlens))
    o0, _ = api.prefill(q, k, v, cu, causal=True, scale=0.0)
    o1, _ = api.prefill(q, k, v, cu, causal=True, scale=inputs.fp32_scale(128))
    assert torch.equal(o0, o1)


def test_bad_cu_seqlens_reports_bounds_error():
    """cu_seqlens[B] beyond total_tokens: the kernel treats the sequence as
    empty and records FA_ERR_DEVICE_BOUNDS instead of reading past the
    buffers."""
    inp = inputs.make_prefill([64, 64], 2, 2, 64, True, seed=4003)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    cu = torch.tensor([0, 64, 500], dtype=torch.int32, device="cuda")
    o = torch.zeros_like(q)
    api.fa_prefill(q, k, v, o, None, cu, True, inp.scale, max_seqlen=436)
    assert api.device_error() == api.FA_ERR_DEVICE_BOUNDS
    assert api.device_error() == api.FA_OK  # cleared by the read
    o_ref, _ = oracle.prefill(inp.q[:64], inp.k[:64], inp.v[:64], inputs.cu_seqlens_of([64]),
                              True, inp.scale)
    check_bf16(to_np(o[:64]), o_ref, "valid sequence")


# ---- full-size workloads, sampled rows ------------------------------------
def sample_rows(lengths, Hq, per_seq_head, seed):
    rng = np.random.default_rng(seed)
    rt, rh = [], []
    start = 0
    for L in lengths:
        for h in range(Hq):
            idx = set(range(min(per_seq_head, L))) | set(range(max(0, L - per_seq_head), L))
            idx |= set(rng.integers(0, L, size=per_seq_head).tolist()) if L else set()
            for i in sorted(idx):
                rt.append(start + i)
                rh.append(h)
        start += L
    return np.array(rt), np.array(rh)


def check_sampled(inp, per_seq_head, seed):
    o, lse = run_gpu(inp)
    rt, rh = sample_rows(inp.lengths, inp.Hq, per_seq_head, seed)
    o_ref, lse_ref = oracle.prefill_rows(inp.q, inp.k, inp.v, inp.cu_seqlens, inp.causal,
                                         inp.scale, rt, rh)
    check_bf16_plain(o[rt, rh], o_ref, "O sampled")
    check_close(lse[rh, rt], lse_ref, LSE_ABS, None, "LSE sampled")
    # properties that hold at any size: finite, and |O| bounded by max|V|
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    assert np.abs(o).max() <= float(inp.v.float().abs().max()) + 1e-2


def test_mha_prefill_full_size_every_row():
    """The causal MHA workload (B=4, H=16, L=2048, d=128) checked in full:
    every row of every (sequence, head) against the fp64 oracle, with the
    plain bounds (max-abs 1e-2, mean-abs 1e-3, no rounding floor)."""
    inp = inputs.mha_prefill()
    o, lse = run_gpu(inp)
    o_ref, lse_ref = oracle.prefill(inp.q, inp.k, inp.v, inp.cu_seqlens, True, inp.scale)
    check_bf16_plain(o, o_ref, "O")
    check_close(lse, lse_ref, LSE_ABS, None, "LSE")


def test_varlen_gqa_prefill_full_size():
    check_sampled(inputs.varlen_gqa_prefill(), per_seq_head=6, seed=5002)


def test_max_seqlen_hint_is_optional():
    """max_seqlen <= 0 means not given: the library bounds the sequences by
    T itself, and the result is bit-identical to a call with the hint."""
    inp = inputs.make_prefill([300, 1000, 0, 129], 8, 2, 128, True, seed=4006)
    q, k, v, cu = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.cu_seqlens))
    o1, l1 = api.prefill(q, k, v, cu, causal=True, scale=inp.scale, max_seqlen=1000)
    o2, l2 = api.prefill(q, k, v, cu, causal=True, scale=inp.scale, max_seqlen=0)
    assert api.device_error() == api.FA_OK
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_repeatable():
    inp = inputs.make_prefill([1000, 333], 8, 2, 128, True, seed=4004)
    a = run_gpu(inp)
    b = run_gpu(inp)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
