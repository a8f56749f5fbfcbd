"""Pins of the oracle's mask variants: sliding window, softcapping and ALiBi
("flash-attention" skill page, section 3.3, advanced features).

As for the plain pins, none of these compares the oracle with itself or with
the CUDA path.  Each is a closed form (window counts with identical keys, a
softcap case whose tanh is known exactly, geometric ALiBi weights), a
reduction to the already pinned plain attention (window (-1, 0) is causal;
causal ALiBi is plain attention with one extra coordinate), or a brute
force with torch's fp64 band masks and softmax.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_86_b200 import inputs

TOL = 1e-12


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64)


def _packed(lengths, Hq, Hkv, d, seed):
    T = sum(lengths)
    return (_rand((T, Hq, d), seed), _rand((T, Hkv, d), seed + 1), _rand((T, Hkv, d), seed + 2),
            inputs.cu_seqlens_of(lengths))


# --------------------------------------------------------------------------
# sliding window
# --------------------------------------------------------------------------
def test_window_special_cases_reduce_to_plain_masks():
    """(-1, 0) is the causal mask; (-1, -1) and windows at least as long as
    the sequence are the full mask; causal with (left, -1) keeps j <= i."""
    q, k, v, cu = _packed([21, 5, 33], 4, 2, 8, seed=101)
    o_c, l_c = oracle.prefill(q, k, v, cu, True, 0.3)
    o_f, l_f = oracle.prefill(q, k, v, cu, False, 0.3)
    for causal, window, ref in ((False, (-1, 0), (o_c, l_c)), (False, (-1, -1), (o_f, l_f)),
                                (False, (33, 33), (o_f, l_f)), (True, (40, -1), (o_c, l_c)),
                                (True, (-1, 7), (o_c, l_c))):
        o, lse = oracle.prefill(q, k, v, cu, causal, 0.3, window=window)
        np.testing.assert_allclose(o, ref[0], atol=TOL, rtol=0)
        np.testing.assert_allclose(lse, ref[1], atol=TOL, rtol=0)


def test_window_zero_sees_only_itself():
    q, k, v, cu = _packed([17], 2, 2, 8, seed=103)
    scale = 0.6
    for causal in (False, True):
        o, lse = oracle.prefill(q, k, v, cu, causal, scale, window=(0, 0))
        np.testing.assert_allclose(o, v.numpy(), atol=TOL, rtol=0)
        for h in range(2):
            s_ii = scale * (q[:, h] * k[:, h]).sum(-1).numpy()
            np.testing.assert_allclose(lse[h], s_ii, atol=TOL, rtol=0)


@pytest.mark.parametrize("causal,window", [(True, (3, -1)), (True, (0, -1)), (False, (2, 5)),
                                           (False, (-1, 1)), (False, (6, 0)), (True, (1, 4))])
def test_window_counts_with_identical_keys(causal, window):
    """With one key repeated, each row averages the values of exactly the
    keys i - left .. i + right (clipped to the sequence, and to j <= i when
    causal), and LSE = s + ln(count)."""
    L, d = 29, 4
    q, _, v, cu = _packed([L], 1, 1, d, seed=105)
    krow = _rand((d,), 106)
    k = krow.expand(L, 1, d).clone()
    scale = 0.7
    o, lse = oracle.prefill(q, k, v, cu, causal, scale, window=window)
    left, right = window
    for i in range(L):
        lo = 0 if left < 0 else max(0, i - left)
        hi = L - 1 if right < 0 else min(L - 1, i + right)
        if causal:
            hi = min(hi, i)
        n = hi - lo + 1
        np.testing.assert_allclose(o[i, 0], v[lo:hi + 1, 0].numpy().mean(axis=0), atol=TOL, rtol=0)
        s = scale * float(q[i, 0] @ krow)
        assert abs(lse[0, i] - (s + math.log(n))) <= TOL


def _torch_band_reference(q, k, v, cu, causal, scale, left, right):
    """softmax(QK^T*scale + band mask)V with torch's fp64 routines; the band
    is the intersection of triu(diagonal=-left) and tril(diagonal=right)."""
    T, Hq, d = q.shape
    g = Hq // k.shape[1]
    o = torch.zeros(T, Hq, d, dtype=torch.float64)
    lse = torch.zeros(Hq, T, dtype=torch.float64)
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        L = s1 - s0
        if L == 0:
            continue
        keep = torch.ones(L, L, dtype=torch.bool)
        if left >= 0:
            keep &= torch.triu(torch.ones(L, L, dtype=torch.bool), diagonal=-left)
        if right >= 0:
            keep &= torch.tril(torch.ones(L, L, dtype=torch.bool), diagonal=right)
        if causal:
            keep &= torch.tril(torch.ones(L, L, dtype=torch.bool), diagonal=0)
        for h in range(Hq):
            S = (q[s0:s1, h] @ k[s0:s1, h // g].T) * scale
            S = S.masked_fill(~keep, float("-inf"))
            o[s0:s1, h] = torch.softmax(S, dim=-1) @ v[s0:s1, h // g]
            lse[h, s0:s1] = torch.logsumexp(S, dim=-1)
    return o.numpy(), lse.numpy()


@pytest.mark.parametrize("causal,window", [(True, (5, -1)), (False, (3, 2)), (False, (0, 9)),
                                           (True, (16, 0)), (False, (-1, 3))])
def test_window_brute_force_band_mask(causal, window):
    q, k, v, cu = _packed([19, 1, 40, 8], 4, 2, 16, seed=107)
    o, lse = oracle.prefill(q, k, v, cu, causal, 0.25, window=window)
    o_ref, lse_ref = _torch_band_reference(q, k, v, cu, causal, 0.25, *window)
    np.testing.assert_allclose(o, o_ref, atol=TOL, rtol=0)
    np.testing.assert_allclose(lse, lse_ref, atol=TOL, rtol=0)


def test_window_probabilities_rows_sum_to_one_inside_the_band():
    q, k, _, cu = _packed([23], 2, 1, 8, seed=109)
    P = oracle.prefill_probs(q, k, cu, False, 0.4, 0, 1, Hkv=1, window=(4, 2))
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=TOL, rtol=0)
    i, j = np.indices(P.shape)
    assert np.count_nonzero(P[(j < i - 4) | (j > i + 2)]) == 0
    assert (P[(j >= i - 4) & (j <= i + 2)] > 0).all()


# --------------------------------------------------------------------------
# softcapping
# --------------------------------------------------------------------------
def test_softcap_closed_form():
    """d = 1, scale 1/2, cap 2.  Key 0 is 0 (logit 0); key 1 is 2 ln 3, so
    its logit is ln 3 = 2 atanh(1/2) and the capped logit is
    2 tanh(atanh(1/2)) = 1 exactly.  Query 1 then weighs the two values
    1/(1+e) and e/(1+e), with LSE ln(1 + e)."""
    q = torch.ones(2, 1, 1, dtype=torch.float64)
    k = torch.tensor([0.0, 2.0 * math.log(3.0)], dtype=torch.float64).reshape(2, 1, 1)
    v = torch.tensor([3.0, -5.0], dtype=torch.float64).reshape(2, 1, 1)
    cu = inputs.cu_seqlens_of([2])
    o, lse = oracle.prefill(q, k, v, cu, True, 0.5, softcap=2.0)
    e = math.e
    assert abs(o[1, 0, 0] - (3.0 / (1 + e) - 5.0 * e / (1 + e))) <= TOL
    assert abs(lse[0, 1] - math.log(1 + e)) <= TOL
    assert abs(o[0, 0, 0] - 3.0) <= TOL and abs(lse[0, 0]) <= TOL


def test_softcap_limits():
    """A cap far above every logit changes nothing (c tanh(x/c) = x - x^3/(3c^2)
    + ...); a cap far below squeezes every logit to within c of 0, so the
    weights are uniform and LSE = ln(count) up to c."""
    q, k, v, cu = _packed([31, 12], 2, 1, 8, seed=111)
    for causal in (False, True):
        o, lse = oracle.prefill(q, k, v, cu, causal, 0.35)
        o2, lse2 = oracle.prefill(q, k, v, cu, causal, 0.35, softcap=1e7)
        np.testing.assert_allclose(o2, o, atol=1e-10, rtol=0)
        np.testing.assert_allclose(lse2, lse, atol=1e-10, rtol=0)
        c = 1e-9
        o3, lse3 = oracle.prefill(q, k, v, cu, causal, 0.35, softcap=c)
        for b, (s0, s1) in enumerate(((0, 31), (31, 43))):
            for i in range(s1 - s0):
                n = i + 1 if causal else s1 - s0
                mean = v[s0:s0 + n, 0].numpy().mean(axis=0)
                np.testing.assert_allclose(o3[s0 + i, 1], mean, atol=1e-7, rtol=0)
                assert abs(lse3[0, s0 + i] - math.log(n)) <= 3 * c


def test_softcap_bounds_the_logits():
    """Capped logits lie in [-c, c] (tanh saturates to exactly +-1 in fp64
    for the large logits used here), so LSE - ln(count) lies in [-c, c]."""
    q, k, v, cu = _packed([25], 2, 2, 16, seed=113)
    c = 1.5
    o, lse = oracle.prefill(30.0 * q, k, v, cu, True, 1.0, softcap=c)
    n = np.arange(1, 26)
    excess = lse - np.log(n)
    assert (excess <= c + TOL).all() and (excess >= -c - TOL).all()
    # without the cap the same logits are far outside that range
    _, lse_plain = oracle.prefill(30.0 * q, k, v, cu, True, 1.0)
    assert (np.abs(lse_plain - np.log(n)) > 4 * c).any()


# --------------------------------------------------------------------------
# ALiBi
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_alibi_geometric_weights_with_identical_keys(causal):
    """Equal scores leave only the penalty -slope |i - j|: the weights are
    r^|i-j| with r = exp(-slope), so LSE = s + ln(sum of a geometric series
    on each side of i) in closed form."""
    L, d, Hq = 26, 4, 2
    slopes = np.array([0.5, 0.125], np.float32)
    q, _, v, cu = _packed([L], Hq, 1, d, seed=115)
    krow = _rand((d,), 116)
    k = krow.expand(L, 1, d).clone()
    scale = 0.3
    o, lse = oracle.prefill(q, k, v, cu, causal, scale, alibi_slopes=slopes)
    for h in range(Hq):
        r = math.exp(-float(slopes[h]))
        for i in range(L):
            left = (1 - r ** (i + 1)) / (1 - r)                           # r^0 .. r^i
            right = 0.0 if causal else r * (1 - r ** (L - 1 - i)) / (1 - r)  # r^1 .. r^(L-1-i)
            s = scale * float(q[i, h] @ krow)
            assert abs(lse[h, i] - (s + math.log(left + right))) <= 1e-12
            js = np.arange(L) if not causal else np.arange(i + 1)
            w = r ** np.abs(i - js)
            np.testing.assert_allclose(o[i, h], (w @ v[js, 0].numpy()) / w.sum(), atol=TOL, rtol=0)


def test_alibi_causal_equals_plain_attention_with_a_position_coordinate():
    """For j <= i, -slope (i - j) = slope j - slope i.  Appending 1 to each
    query and slope j / scale to key j adds slope j to every logit, so plain
    causal attention on the augmented vectors gives the same O, and its LSE
    exceeds the ALiBi LSE by slope i."""
    L, d, Hq = 37, 8, 4
    slopes = np.array([0.7, 0.25, 0.03125, 0.0], np.float32)
    q, k, v, cu = _packed([L], Hq, 1, d, seed=117)
    scale = 0.2
    o, lse = oracle.prefill(q, k, v, cu, True, scale, alibi_slopes=slopes)
    pos = torch.arange(L, dtype=torch.float64)
    for h in range(Hq):
        sl = float(slopes[h])
        qa = torch.cat([q[:, h:h + 1], torch.ones(L, 1, 1, dtype=torch.float64)], dim=2)
        ka = torch.cat([k, (sl * pos / scale).reshape(L, 1, 1)], dim=2)
        va = torch.cat([v, torch.zeros(L, 1, 1, dtype=torch.float64)], dim=2)  # same d as q, k
        oa, la = oracle.prefill(qa, ka, va, cu, True, scale)
        np.testing.assert_allclose(o[:, h], oa[:, 0, :d], atol=1e-11, rtol=0)
        np.testing.assert_allclose(lse[h], la[0] - sl * pos.numpy(), atol=1e-11, rtol=0)


def test_alibi_slope_layouts():
    """(Hq,) slopes: query head h uses slope h (not its kv head's).
    (B, Hq) slopes: sequence b uses row b.  Both equal separate
    single-sequence, single-head calls."""
    lengths, Hq, Hkv, d = [11, 19], 4, 2, 8
    q, k, v, cu = _packed(lengths, Hq, Hkv, d, seed=119)
    per_head = np.array([0.9, 0.3, 0.05, 0.6], np.float32)
    per_seq = np.array([[0.2, 0.4, 0.8, 1.6], [1.0, 0.5, 0.25, 0.125]], np.float32)
    for slopes in (per_head, per_seq):
        for causal in (False, True):
            o, lse = oracle.prefill(q, k, v, cu, causal, 0.3, alibi_slopes=slopes)
            for b, L in enumerate(lengths):
                s0 = int(cu[b])
                sl = slice(s0, s0 + L)
                for h in range(Hq):
                    row = slopes if slopes.ndim == 1 else slopes[b]
                    one = np.array([row[h]], np.float32)
                    ob, lb = oracle.prefill(q[sl, h:h + 1], k[sl, h // 2:h // 2 + 1],
                                            v[sl, h // 2:h // 2 + 1], inputs.cu_seqlens_of([L]),
                                            causal, 0.3, alibi_slopes=one)
                    np.testing.assert_array_equal(o[sl, h], ob[:, 0])
                    np.testing.assert_array_equal(lse[h, sl], lb[0])


def test_cap_then_alibi_order():
    """The cap applies to the scaled score and the ALiBi penalty is added to
    the capped value: with identical keys every capped logit is
    c tanh(s / c), and the weights stay exactly geometric."""
    L, d = 15, 4
    q, _, v, cu = _packed([L], 1, 1, d, seed=121)
    krow = _rand((d,), 122)
    k = krow.expand(L, 1, d).clone()
    c, slope, scale = 1.0, 0.75, 0.9
    o, lse = oracle.prefill(q, k, v, cu, True, scale, softcap=c,
                            alibi_slopes=np.array([slope], np.float32))
    r = math.exp(-slope)
    for i in range(L):
        s = scale * float(q[i, 0] @ krow)
        capped = c * math.tanh(s / c)
        assert abs(lse[0, i] - (capped + math.log((1 - r ** (i + 1)) / (1 - r)))) <= 1e-12


def test_all_variants_brute_force():
    """Window, cap and ALiBi together against torch fp64: band mask, tanh cap,
    then the distance penalty, then softmax."""
    lengths, Hq, Hkv, d = [27, 3, 18], 4, 1, 8
    q, k, v, cu = _packed(lengths, Hq, Hkv, d, seed=123)
    slopes = np.array([[0.3, 0.1, 0.7, 0.05], [0.2, 0.2, 0.2, 0.2], [1.0, 0.0, 0.5, 0.25]],
                      np.float32)
    scale, c, (left, right) = 0.45, 2.5, (6, 3)
    o, lse = oracle.prefill(q, k, v, cu, False, scale, window=(left, right), softcap=c,
                            alibi_slopes=slopes)
    for b in range(3):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        L = s1 - s0
        i = torch.arange(L).unsqueeze(1)
        j = torch.arange(L).unsqueeze(0)
        keep = torch.triu(torch.ones(L, L, dtype=torch.bool), diagonal=-left) & \
            torch.tril(torch.ones(L, L, dtype=torch.bool), diagonal=right)
        for h in range(Hq):
            S = c * torch.tanh((q[s0:s1, h] @ k[s0:s1, 0].T) * scale / c)
            S = S - float(slopes[b, h]) * (i - j).abs().double()
            S = S.masked_fill(~keep, float("-inf"))
            np.testing.assert_allclose(o[s0:s1, h], (torch.softmax(S, -1) @ v[s0:s1, 0]).numpy(),
                                       atol=TOL, rtol=0)
            np.testing.assert_allclose(lse[h, s0:s1], torch.logsumexp(S, -1).numpy(), atol=TOL,
                                       rtol=0)
