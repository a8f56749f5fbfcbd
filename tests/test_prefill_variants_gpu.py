"""Parity of the prefill mask variants -- sliding window, softcap, ALiBi
("flash-attention" skill page, section 3.3) -- with the fp64 oracle, through
the C ABI (fa_prefill_ex), on seeded inputs.

Windows are chosen around the 128-key tile edges (1, 127, 128, 129, 255, ...)
so that bands start and end inside tiles, on tile boundaries, and span
several tiles; lengths have ragged tails.  The long sliding-window workload
is checked on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_86_b200 import api, inputs
from parity import LSE_ABS, check_bf16, check_bf16_peaked, check_close, to_np

pytestmark = pytest.mark.gpu


def run_gpu(inp, causal, **variant):
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    cu = inp.cu_seqlens.cuda()
    if variant.get("alibi_slopes") is not None:
        variant = dict(variant, alibi_slopes=variant["alibi_slopes"].cuda())
    o, lse = api.prefill(q, k, v, cu, causal=causal, scale=inp.scale,
                         max_seqlen=max(inp.lengths), **variant)
    torch.cuda.synchronize()
    assert api.device_error() == api.FA_OK
    return to_np(o), to_np(lse)


def assert_matches(inp, causal, peaked=False, **variant):
    """peaked: the inputs make most rows average one or two keys (see
    parity.check_bf16_peaked); otherwise the plain bf16 bounds apply."""
    o, lse = run_gpu(inp, causal, **variant)
    o_ref, lse_ref = oracle.prefill(inp.q, inp.k, inp.v, inp.cu_seqlens, causal, inp.scale,
                                    **variant)
    (check_bf16_peaked if peaked else check_bf16)(o, o_ref, "O")
    check_close(lse, lse_ref, LSE_ABS, None, "LSE")


LENGTHS = [1, 127, 128, 129, 700, 1500]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("left", [0, 1, 100, 127, 128, 129, 255, 256, 1000])
def test_causal_sliding_window(left, d):
    inp = inputs.make_prefill(LENGTHS, 4, 2, d, True, seed=5000 + left + d)
    # left = 1: every row but the first averages exactly two keys
    assert_matches(inp, True, peaked=left in (1, 2), window=(left, 0))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("window", [(0, 0), (37, 200), (300, 5), (-1, 64), (128, 128),
                                    (129, 127), (5, -1)])
def test_two_sided_window(window, d):
    inp = inputs.make_prefill([3, 129, 640, 1111], 8, 2, d, False, seed=5100 + sum(window) + d)
    assert_matches(inp, False, peaked=window == (0, 0), window=window)


def test_window_normalisation_reaches_the_plain_kernel():
    """(-1, 0) without causal is the causal mask, and windows at least as long
    as every sequence are no window: both give the plain kernels' bits."""
    inp = inputs.make_prefill([300, 1000], 4, 4, 128, False, seed=5200)
    o_c, l_c = run_gpu(inp, True)
    o_w, l_w = run_gpu(inp, False, window=(-1, 0))
    assert np.array_equal(o_c, o_w) and np.array_equal(l_c, l_w)
    o_f, l_f = run_gpu(inp, False)
    o_w, l_w = run_gpu(inp, False, window=(1000, 5000))
    assert np.array_equal(o_f, o_w) and np.array_equal(l_f, l_w)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("softcap,scale", [(50.0, None), (50.0, 1.0), (5.0, 1.0), (1.0, None),
                                           (0.5, 1.0)])
def test_softcap(softcap, scale, causal):
    inp = inputs.make_prefill([1, 200, 513, 1024], 8, 4, 128, causal, seed=5300, scale=scale)
    # scale 1 with d = 128 gives logits of standard deviation ~11: the capped
    # softmax is still dominated by a few keys per row
    assert_matches(inp, causal, peaked=scale == 1.0 and softcap > 8, softcap=softcap)


@pytest.mark.parametrize("causal,window,d", [(True, (150, 0), 128), (False, (40, 260), 64),
                                             (True, (-1, 0), 64), (False, (0, 0), 128)])
def test_softcap_with_window(causal, window, d):
    """Softcap without ALiBi (the kernel caps each score inside its
    exponential loop and the row max once) under band masks, so masked
    scores must stay at zero weight."""
    inp = inputs.make_prefill([2, 300, 129, 900], 8, 2, d, causal, seed=5350 + d + window[0])
    assert_matches(inp, causal, peaked=window == (0, 0), window=window, softcap=5.0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_alibi_per_head(causal, d):
    inp = inputs.make_prefill([1, 130, 777, 1300], 8, 2, d, causal, seed=5400 + d)
    assert_matches(inp, causal, alibi_slopes=inputs.alibi_slopes_geometric(8))


@pytest.mark.parametrize("causal", [False, True])
def test_alibi_per_sequence_and_head(causal):
    lengths = [64, 1, 900, 256, 333]
    inp = inputs.make_prefill(lengths, 4, 4, 128, causal, seed=5500)
    slopes = inputs.uniform_slopes((len(lengths), 4), 0.0, 1.0, torch.Generator().manual_seed(5501))
    assert_matches(inp, causal, alibi_slopes=slopes)


@pytest.mark.parametrize("window,d", [((100, 0), 128), ((300, 0), 64), ((0, 0), 128),
                                      ((-1, 0), 64)])
def test_alibi_causal_with_left_window(window, d):
    """Causal ALiBi without softcap (every visible key precedes its query, so
    the kernel folds the penalty into the row max and the exponent) together
    with a left window bound, including a window of one key."""
    lengths = [3, 600, 129, 1000]
    inp = inputs.make_prefill(lengths, 8, 4, d, True, seed=5450 + d + window[0])
    slopes = inputs.uniform_slopes((len(lengths), 8), 0.0, 0.3, torch.Generator().manual_seed(5451))
    assert_matches(inp, True, peaked=window[0] == 0, window=window, alibi_slopes=slopes)


@pytest.mark.parametrize("causal,window", [(True, (200, 0)), (False, (64, 300)), (True, (-1, 0))])
def test_all_variants_together(causal, window):
    lengths = [0, 5, 1200, 129, 640]
    inp = inputs.make_prefill(lengths, 8, 2, 128, causal, seed=5600 + window[0], scale=0.5)
    slopes = inputs.uniform_slopes((len(lengths), 8), 0.0, 0.5, torch.Generator().manual_seed(5601))
    # slopes up to 0.5 per token concentrate each row on its nearest keys
    assert_matches(inp, causal, peaked=True, window=window, softcap=8.0, alibi_slopes=slopes)


def _sample_rows(lengths, Hq, n_random, seed):
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    rows_t, rows_h = [], []
    for b, L in enumerate(lengths):
        ts = list(range(min(L, 130))) + list(range(max(0, L - 130), L))
        ts += list(rng.integers(0, L, n_random))
        for t in ts:
            rows_t.append(int(cu[b] + t))
            rows_h.append(int(rng.integers(0, Hq)))
    return np.array(rows_t), np.array(rows_h)


def test_window_workload_sampled_rows():
    """The long sliding-window workload ((4096, 0) over 2 x 16384 tokens,
    Hq=32, Hkv=8) at full size, checked on sampled rows."""
    inp = inputs.window_prefill()
    variant = inp.meta["variant"]
    o, lse = run_gpu(inp, True, **variant)
    rt, rh = _sample_rows(inp.lengths, 32, 600, seed=5700)
    o_ref, lse_ref = oracle.prefill_rows(inp.q, inp.k, inp.v, inp.cu_seqlens, True, inp.scale,
                                         rt, rh, **variant)
    check_bf16(o[rt, rh], o_ref, "O")
    check_close(lse[rh, rt], lse_ref, LSE_ABS, None, "LSE")


@pytest.mark.parametrize("name", ["softcap_prefill", "alibi_prefill"])
def test_variant_workloads_sampled_rows(name):
    inp = getattr(inputs, name)()
    variant = inp.meta["variant"]
    o, lse = run_gpu(inp, True, **variant)
    rt, rh = _sample_rows(inp.lengths, 16, 200, seed=5800)
    o_ref, lse_ref = oracle.prefill_rows(inp.q, inp.k, inp.v, inp.cu_seqlens, True, inp.scale,
                                         rt, rh, **variant)
    check_bf16(o[rt, rh], o_ref, "O")
    check_close(lse[rh, rt], lse_ref, LSE_ABS, None, "LSE")


def test_rejects_bad_variant_arguments():
    inp = inputs.make_prefill([16], 2, 2, 64, True, seed=5900)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    cu = inp.cu_seqlens.cuda()
    for bad in (dict(softcap=-1.0), dict(softcap=float("inf")), dict(softcap=float("nan"))):
        with pytest.raises(api.FAError) as e:
            api.prefill(q, k, v, cu, causal=True, **bad)
        assert e.value.code == api.FA_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        api.prefill(q, k, v, cu, causal=True, alibi_slopes=torch.ones(3, device="cuda"))
