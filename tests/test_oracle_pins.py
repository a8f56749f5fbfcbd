"""Pins of the fp64 oracle to facts fixed by the pages and by mathematics.

None of these compares the oracle with itself or with the CUDA path.  Each
pin is one of: a closed form, an invariant, a special case that reduces to a
library routine (torch's fp64 softmax/matmul), the online-softmax streaming
recurrence the pages describe (written independently here), or a printed
example from the pages.  ``test_oracle_mutants.py`` shows that plausible
mistakes planted in the oracle's source fail at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_86_b200 import inputs

TOL = 1e-12
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64).to(dtype)


def _packed(lengths, Hq, Hkv, d, seed):
    T = sum(lengths)
    q = _rand((T, Hq, d), seed)
    k = _rand((T, Hkv, d), seed + 1)
    v = _rand((T, Hkv, d), seed + 2)
    return q, k, v, inputs.cu_seqlens_of(lengths)


# --------------------------------------------------------------------------
# I6: brute force against torch's fp64 softmax and matmul on tiny shapes
# --------------------------------------------------------------------------
def _torch_reference(q, k, v, cu, causal, scale):
    """softmax(QK^T*scale + mask)V per sequence and head, with library routines."""
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    o = torch.zeros(T, Hq, d, dtype=torch.float64)
    lse = torch.zeros(Hq, T, dtype=torch.float64)
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        if s1 == s0:
            continue
        for h in range(Hq):
            Q = q[s0:s1, h].double()
            K = k[s0:s1, h // g].double()
            V = v[s0:s1, h // g].double()
            S = (Q @ K.T) * scale
            if causal:
                L = s1 - s0
                mask = torch.triu(torch.ones(L, L, dtype=torch.bool), diagonal=1)
                S = S.masked_fill(mask, float("-inf"))
            o[s0:s1, h] = torch.softmax(S, dim=-1) @ V
            lse[h, s0:s1] = torch.logsumexp(S, dim=-1)
    return o, lse


@pytest.mark.parametrize("d", [1, 2, 4, 64])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("lengths,Hq,Hkv", [([1], 1, 1), ([17], 2, 1), ([3, 0, 16, 5], 4, 2),
                                            ([15, 2], 8, 8)])
def test_brute_force_matches_library_softmax(d, causal, lengths, Hq, Hkv):
    q, k, v, cu = _packed(lengths, Hq, Hkv, d, seed=7 + d)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.prefill(q, k, v, cu, causal, scale)
    o_ref, lse_ref = _torch_reference(q, k, v, cu, causal, scale)
    np.testing.assert_allclose(o, o_ref.numpy(), atol=TOL, rtol=0)
    np.testing.assert_allclose(lse, lse_ref.numpy(), atol=TOL, rtol=0)


def test_bf16_and_f32_inputs_upcast_exactly():
    """bf16 and fp32 inputs must give the fp64 result of their exact values."""
    q, k, v, cu = _packed([9, 4], 2, 1, 8, seed=3)
    for dt in (torch.bfloat16, torch.float32):
        qa, ka, va = q.to(dt), k.to(dt), v.to(dt)
        o, lse = oracle.prefill(qa, ka, va, cu, True, 0.25)
        o_ref, lse_ref = oracle.prefill(qa.double(), ka.double(), va.double(), cu, True, 0.25)
        assert np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref)


# --------------------------------------------------------------------------
# I1: every row of P sums to one; P is zero above the diagonal when causal
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    q, k, v, cu = _packed([13, 31], 4, 2, 16, seed=11)
    for b in range(2):
        for h in range(4):
            P = oracle.prefill_probs(q, k, cu, causal, 0.3, b, h, Hkv=2)
            np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=TOL, rtol=0)
            assert (P >= 0).all()
            if causal:
                assert np.count_nonzero(np.triu(P, 1)) == 0
            # the same P reproduces the oracle's output rows
            s0, s1 = int(cu[b]), int(cu[b + 1])
            o, _ = oracle.prefill(q, k, v, cu, causal, 0.3)
            np.testing.assert_allclose(P @ v[s0:s1, h // 2].numpy(), o[s0:s1, h], atol=TOL,
                                       rtol=0)


# --------------------------------------------------------------------------
# I2: the online-softmax recurrence (running max m and sum l with
# rescaling), run over any partition of the keys in any order, equals the
# oracle's two-pass softmax.  The pages state that the block-wise streaming
# form is exactly equal to the global softmax (gsyq.cn FA vs FIA, section 1).
# --------------------------------------------------------------------------
def _online(qrow, K, V, scale, blocks):
    m, l = -np.inf, 0.0
    acc = np.zeros(V.shape[1])
    for idx in blocks:
        s = (K[idx] @ qrow) * scale
        m_new = max(m, s.max())
        alpha = math.exp(m - m_new) if m != -np.inf else 0.0
        p = np.exp(s - m_new)
        l = alpha * l + p.sum()
        acc = alpha * acc + p @ V[idx]
        m = m_new
    return acc / l, m + math.log(l)


@pytest.mark.parametrize("causal", [False, True])
def test_online_recurrence_on_any_tiling(causal):
    L, d = 97, 32
    q, k, v, cu = _packed([L], 1, 1, d, seed=21)
    scale = 0.17
    o, lse = oracle.prefill(q, k, v, cu, causal, scale)
    rng = np.random.default_rng(5)
    Q, K, V = q[:, 0].numpy(), k[:, 0].numpy(), v[:, 0].numpy()
    for i in (0, 1, 50, L - 1):
        n = i + 1 if causal else L
        keys = np.arange(n)
        tilings = [
            [keys[j:j + bc] for j in range(0, n, bc)] for bc in (1, 3, 64, 128)
        ]
        cuts = np.sort(rng.choice(np.arange(1, n), size=min(5, n - 1), replace=False)) if n > 1 else []
        tilings.append(np.split(keys, cuts))
        perm = rng.permutation(n)            # any visiting order
        tilings.append(np.array_split(perm, max(1, n // 7)))
        for blocks in tilings:
            blocks = [b for b in blocks if len(b)]
            o_on, lse_on = _online(Q[i], K, V, scale, blocks)
            np.testing.assert_allclose(o_on, o[i, 0], atol=TOL, rtol=0)
            assert abs(lse_on - lse[0, i]) <= TOL


# --------------------------------------------------------------------------
# I3: identical keys -> every visible key has the same score, so O is the
# mean of the visible values and LSE = s + ln(n_visible)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_mean_of_values(causal):
    L, d = 40, 8
    q, _, v, cu = _packed([L], 2, 1, d, seed=31)
    krow = _rand((d,), 99)
    k = krow.expand(L, 1, d).clone()
    scale = 0.5
    o, lse = oracle.prefill(q, k, v, cu, causal, scale)
    for h in range(2):
        for i in range(L):
            n = i + 1 if causal else L
            np.testing.assert_allclose(o[i, h], v[:n, 0].numpy().mean(axis=0), atol=TOL, rtol=0)
            s = scale * float(q[i, h] @ krow)
            assert abs(lse[h, i] - (s + math.log(n))) <= TOL


# --------------------------------------------------------------------------
# I4: one dominant logit selects its value row
# --------------------------------------------------------------------------
def test_dominant_logit_selects_its_value():
    """Key j* has projection 10 on a unit direction e, every other key at
    most 1; the query is 10 e, so the logit gap is at least 90 and the
    softmax weight off j* is below L * exp(-90)."""
    L, d, jstar = 33, 16, 5
    g = torch.Generator().manual_seed(41)
    e = torch.randn(d, generator=g, dtype=torch.float64)
    e = e / e.norm()
    keys = torch.randn(L, d, generator=g, dtype=torch.float64)
    proj = keys @ e
    keys = keys - (proj - proj.clamp(max=1.0)).unsqueeze(1) * e
    keys[jstar] = 10.0 * e
    q = (10.0 * e).expand(L, 1, d).clone()
    v = _rand((L, 1, d), 42)
    cu = inputs.cu_seqlens_of([L])
    o, _ = oracle.prefill(q, keys.reshape(L, 1, d), v, cu, False, 1.0)
    for i in range(L):
        np.testing.assert_allclose(o[i, 0], v[jstar, 0].numpy(), atol=1e-12, rtol=0)
    oc, _ = oracle.prefill(q, keys.reshape(L, 1, d), v, cu, True, 1.0)
    for i in range(jstar, L):
        np.testing.assert_allclose(oc[i, 0], v[jstar, 0].numpy(), atol=1e-12, rtol=0)


# --------------------------------------------------------------------------
# I5: under the causal mask the first query sees only key 0; a length-1
# sequence likewise
# --------------------------------------------------------------------------
def test_causal_first_row_and_length_one():
    q, k, v, cu = _packed([12, 1, 7], 2, 2, 8, seed=51)
    scale = 0.4
    o, lse = oracle.prefill(q, k, v, cu, True, scale)
    for start in (0, 12, 13):
        for h in range(2):
            np.testing.assert_allclose(o[start, h], v[start, h].numpy(), atol=TOL, rtol=0)
            s00 = scale * float(q[start, h] @ k[start, h])
            assert abs(lse[h, start] - s00) <= TOL
    o2, lse2 = oracle.prefill(q, k, v, cu, False, scale)
    np.testing.assert_allclose(o2[12], v[12].numpy(), atol=TOL, rtol=0)


# --------------------------------------------------------------------------
# I7: affine values: rows of P sum to one, so O(aV + c) = a O(V) + c
# --------------------------------------------------------------------------
def test_affine_values():
    q, k, v, cu = _packed([25, 6], 4, 2, 8, seed=61)
    c = _rand((8,), 62)
    a = -1.7
    for causal in (False, True):
        o, lse = oracle.prefill(q, k, v, cu, causal, 0.3)
        o2, lse2 = oracle.prefill(q, k, a * v + c, cu, causal, 0.3)
        np.testing.assert_allclose(o2, a * o + c.numpy(), atol=TOL, rtol=0)
        np.testing.assert_allclose(lse2, lse, atol=TOL, rtol=0)


# --------------------------------------------------------------------------
# I9: grouped heads equal full multi-head attention on repeated K/V
# (skill page, GQA/MQA appendix: q heads 32 over kv heads 8, no repeat_kv)
# --------------------------------------------------------------------------
def test_gqa_equals_mha_on_repeated_kv():
    Hq, Hkv = 8, 2
    q, k, v, cu = _packed([19, 11], Hq, Hkv, 16, seed=71)
    o, lse = oracle.prefill(q, k, v, cu, True, 0.25)
    kr = k.repeat_interleave(Hq // Hkv, dim=1)
    vr = v.repeat_interleave(Hq // Hkv, dim=1)
    o2, lse2 = oracle.prefill(q, kr, vr, cu, True, 0.25)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


# --------------------------------------------------------------------------
# I10: packed sequences do not see each other (skill page, section 3.4)
# --------------------------------------------------------------------------
def test_varlen_equals_separate_sequences():
    lengths = [7, 0, 23, 1, 16]
    q, k, v, cu = _packed(lengths, 2, 1, 8, seed=81)
    for causal in (False, True):
        o, lse = oracle.prefill(q, k, v, cu, causal, 0.5)
        for b, L in enumerate(lengths):
            s0 = int(cu[b])
            sl = slice(s0, s0 + L)
            ob, lb = oracle.prefill(q[sl], k[sl], v[sl], inputs.cu_seqlens_of([L]), causal, 0.5)
            assert np.array_equal(o[sl], ob)
            assert np.array_equal(lse[:, sl], lb)


def test_rows_api_matches_full():
    q, k, v, cu = _packed([30, 9], 4, 2, 8, seed=91)
    o, lse = oracle.prefill(q, k, v, cu, True, 0.3)
    rt = [0, 5, 29, 30, 38, 17]
    rh = [0, 3, 1, 2, 3, 0]
    orow, lrow = oracle.prefill_rows(q, k, v, cu, True, 0.3, rt, rh)
    for r, (t, h) in enumerate(zip(rt, rh)):
        assert np.array_equal(orow[r], o[t, h])
        assert lrow[r] == lse[h, t]


# --------------------------------------------------------------------------
# Decode: paged layout (skill page, PagedAttention appendix)
# --------------------------------------------------------------------------
def _decode_case(seq_lens, Hq, Hkv, d, ps, seed):
    gen = torch.Generator().manual_seed(seed)
    bt, num_pages = inputs.paged_layout(seq_lens, ps, gen)
    q = _rand((len(seq_lens), Hq, d), seed + 1)
    kp = _rand((num_pages, ps, Hkv, d), seed + 2)
    vp = _rand((num_pages, ps, Hkv, d), seed + 3)
    return q, kp, vp, bt, torch.tensor(seq_lens, dtype=torch.int32)


def _contiguous_from_pages(kp, bt, seq_lens, ps):
    """Gather each request's tokens into a contiguous [len, Hkv, d] tensor."""
    out = []
    for b, n in enumerate(seq_lens):
        rows = [kp[int(bt[b, t // ps]), t % ps] for t in range(n)]
        out.append(torch.stack(rows) if rows else kp[:0, 0])
    return out


@pytest.mark.parametrize("ps", [1, 3, 16])
def test_decode_equals_causal_prefill_last_row(ps):
    """One query at the last position sees every cached token: the decode
    result equals the last row of causal prefill on the contiguous sequence
    whose last query is the decode query."""
    seq_lens = [1, 5, 33, 16]
    Hq, Hkv, d = 4, 2, 8
    q, kp, vp, bt, sl = _decode_case(seq_lens, Hq, Hkv, d, ps, seed=101)
    o, lse = oracle.decode_paged(q, kp, vp, bt, sl, 0.35)
    ks = _contiguous_from_pages(kp, bt, seq_lens, ps)
    vs = _contiguous_from_pages(vp, bt, seq_lens, ps)
    for b, n in enumerate(seq_lens):
        qseq = torch.zeros(n, Hq, d, dtype=torch.float64)
        qseq[-1] = q[b]
        op, lp = oracle.prefill(qseq, ks[b], vs[b], inputs.cu_seqlens_of([n]), True, 0.35)
        np.testing.assert_allclose(o[b], op[-1], atol=TOL, rtol=0)
        np.testing.assert_allclose(lse[b], lp[:, -1], atol=TOL, rtol=0)


def test_decode_page_permutation_is_invisible():
    """I11: a random placement of pages, the identity placement and a
    contiguous cache give the same result."""
    seq_lens = [9, 30, 1, 17]
    ps = 4
    q, kp, vp, bt, sl = _decode_case(seq_lens, 8, 2, 16, ps, seed=111)
    o, lse = oracle.decode_paged(q, kp, vp, bt, sl, 0.25)
    # identity table over a re-laid-out pool
    order = [int(bt[b, i]) for b, n in enumerate(seq_lens) for i in range((n + ps - 1) // ps)]
    kp2, vp2 = kp[order], vp[order]
    bt2 = torch.full_like(bt, -1)
    off = 0
    for b, n in enumerate(seq_lens):
        m = (n + ps - 1) // ps
        bt2[b, :m] = torch.arange(off, off + m)
        off += m
    o2, lse2 = oracle.decode_paged(q, kp2, vp2, bt2, sl, 0.25)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)
    # one page holding the whole context (page_size = max length) = contiguous cache
    maxlen = max(seq_lens)
    kc = torch.zeros(len(seq_lens), maxlen, 2, 16, dtype=torch.float64)
    vc = torch.zeros_like(kc)
    for b, (kb, vb) in enumerate(zip(_contiguous_from_pages(kp, bt, seq_lens, ps),
                                     _contiguous_from_pages(vp, bt, seq_lens, ps))):
        kc[b, :seq_lens[b]] = kb
        vc[b, :seq_lens[b]] = vb
    bt3 = torch.arange(len(seq_lens), dtype=torch.int32).reshape(-1, 1)
    o3, lse3 = oracle.decode_paged(q, kc, vc, bt3, sl, 0.25)
    assert np.array_equal(o, o3) and np.array_equal(lse, lse3)


def test_decode_lse_merge_of_any_key_partition():
    """I8: splitting a request's pages into contiguous ranges, attending to
    each range alone and merging the partial results by log-sum-exp gives
    the unsplit result; an empty range (LSE = -inf) contributes nothing.
    This is the reduce step of split-KV decoding (skill page, FlashDecoding
    appendix)."""
    seq_lens = [45, 7, 64]
    ps = 4
    q, kp, vp, bt, sl = _decode_case(seq_lens, 4, 1, 8, ps, seed=121)
    o, lse = oracle.decode_paged(q, kp, vp, bt, sl, 0.3)
    rng = np.random.default_rng(3)
    for b, n in enumerate(seq_lens):
        pages = (n + ps - 1) // ps
        for nsplit in (1, 2, 3, pages, pages + 2):
            cuts = np.sort(rng.choice(np.arange(0, pages + 1), size=nsplit - 1, replace=True))
            bounds = [0, *cuts.tolist(), pages]
            parts_o, parts_l = [], []
            for p0, p1 in zip(bounds[:-1], bounds[1:]):
                tok = max(0, min(n, p1 * ps) - p0 * ps)
                btp = torch.full((1, max(1, p1 - p0)), -1, dtype=torch.int32)
                btp[0, : p1 - p0] = bt[b, p0:p1]
                op, lp = oracle.decode_paged(q[b:b + 1], kp, vp, btp,
                                             torch.tensor([tok], dtype=torch.int32), 0.3)
                parts_o.append(op[0])
                parts_l.append(lp[0])
            L = np.stack(parts_l)              # [nsplit, Hq]
            Lmax = L.max(axis=0)
            LSE = Lmax + np.log(np.exp(L - Lmax).sum(axis=0))
            w = np.exp(L - LSE)                # [nsplit, Hq]
            merged = (w[:, :, None] * np.stack(parts_o)).sum(axis=0)
            np.testing.assert_allclose(merged, o[b], atol=TOL, rtol=0)
            np.testing.assert_allclose(LSE, lse[b], atol=TOL, rtol=0)


def test_decode_empty_context():
    q, kp, vp, bt, sl = _decode_case([0, 3], 2, 1, 4, 2, seed=131)
    o, lse = oracle.decode_paged(q, kp, vp, bt, sl, 1.0)
    assert (o[0] == 0).all() and np.isneginf(lse[0]).all()
    np.testing.assert_allclose(o[1].sum(), o[1].sum())  # finite


def test_decode_rejects_out_of_pool_pages():
    q, kp, vp, bt, sl = _decode_case([5], 1, 1, 4, 2, seed=141)
    bt[0, 1] = kp.shape[0]
    with pytest.raises(IndexError):
        oracle.decode_paged(q, kp, vp, bt, sl, 1.0)


# --------------------------------------------------------------------------
# Golden values printed by the pages (host-side layout facts)
# --------------------------------------------------------------------------
def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                a, b = line.split("|")
                rows.append((a.split(), b.split()))
    return rows


def test_golden_cu_seqlens_examples():
    for lengths, cu in _golden_rows("cu_seqlens.txt"):
        got = inputs.cu_seqlens_of([int(x) for x in lengths]).tolist()
        assert got == [int(x) for x in cu]


def test_golden_score_matrix_memory():
    """The printed memory of a materialised N x N score matrix is 4 N^2
    bytes; this is the quantity the method never writes to HBM."""
    units = {"MB": 2 ** 20, "GB": 2 ** 30}
    for (n,), (val, unit) in _golden_rows("score_matrix_memory.txt"):
        assert 4 * int(n) ** 2 == int(val) * units[unit]
