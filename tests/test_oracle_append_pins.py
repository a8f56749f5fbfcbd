"""Pins of the oracle's decode-with-append step and its RoPE ("flash-attention"
skill page, section 3.5: k_new / v_new appended at cache_seqlens, rotary_cos /
rotary_sin / rotary_interleaved).

The rotation is pinned by closed forms (identity and quarter-turn tables,
the norm identity |R x|^2 = (cos^2 + sin^2) |x|^2), by the rotation property
that makes RoPE relative (q.k after rotation depends only on the position
difference), and by the exact relation between the interleaved and the
half-split pairings.  The append is pinned against the already pinned plain
paged decode on a cache the test writes itself.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_86_b200 import inputs

TOL = 1e-12


def _rand(shape, seed, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64).to(dtype)


def _tables(max_pos, half, base=10000.0):
    """fp32 cos/sin tables of angle pos * base^(-i/half)."""
    pos = torch.arange(max_pos, dtype=torch.float64).unsqueeze(1)
    inv = base ** (-torch.arange(half, dtype=torch.float64) / half)
    ang = pos * inv
    return torch.cos(ang).float(), torch.sin(ang).float()


# --------------------------------------------------------------------------
# RoPE
# --------------------------------------------------------------------------
def test_rope_identity_and_quarter_turn():
    d, rd = 16, 12
    x = _rand((5, d), 201)
    one, zero = torch.ones(3, rd // 2), torch.zeros(3, rd // 2)
    np.testing.assert_array_equal(oracle.rope(x, [0] * 5, one, zero, rd), x.numpy())
    # cos 0, sin 1: each pair (a, b) turns into (-b, a); dims >= rd untouched
    for inter in (False, True):
        out = oracle.rope(x, [1] * 5, torch.stack([one[0], zero[0]]), torch.stack([zero[0], one[0]]),
                          rd, inter)
        X = x.numpy()
        for i in range(rd // 2):
            a, b = (2 * i, 2 * i + 1) if inter else (i, i + rd // 2)
            np.testing.assert_array_equal(out[:, a], -X[:, b])
            np.testing.assert_array_equal(out[:, b], X[:, a])
        np.testing.assert_array_equal(out[:, rd:], X[:, rd:])


def test_rope_pair_norms():
    """|R x|^2 = (cos^2 + sin^2) |x|^2 for every rotated pair."""
    d = rd = 32
    cos, sin = _tables(50, rd // 2)
    x = _rand((7, d), 203)
    pos = [0, 3, 11, 17, 29, 42, 49]
    out = oracle.rope(x, pos, cos, sin, rd)
    X = x.numpy()
    for r, p in enumerate(pos):
        c, s = cos[p].double().numpy(), sin[p].double().numpy()
        n_in = X[r, :rd // 2] ** 2 + X[r, rd // 2:] ** 2
        n_out = out[r, :rd // 2] ** 2 + out[r, rd // 2:] ** 2
        np.testing.assert_allclose(n_out, (c * c + s * s) * n_in, rtol=1e-12, atol=0)


@pytest.mark.parametrize("interleaved", [False, True])
def test_rope_is_relative(interleaved):
    """<R(p+t) q, R(p'+t) k> = <R(p) q, R(p') k>: rotations by position
    angles make the score depend on p - p' only (up to the fp32 tables'
    rounding, ~1e-7 relative)."""
    d, rd = 64, 48
    cos, sin = _tables(400, rd // 2)
    q, k = _rand((1, d), 205), _rand((1, d), 206)
    for p, pp, t in ((5, 2, 100), (300, 17, 57), (0, 0, 399)):
        a = oracle.rope(q, [p + t], cos, sin, rd, interleaved) @ oracle.rope(k, [pp + t], cos, sin, rd, interleaved).T
        b = oracle.rope(q, [p], cos, sin, rd, interleaved) @ oracle.rope(k, [pp], cos, sin, rd, interleaved).T
        assert abs(a.item() - b.item()) < 5e-5 * (1 + abs(b.item()))
        # and it does depend on the difference
        c = oracle.rope(q, [p + 1], cos, sin, rd, interleaved) @ oracle.rope(k, [pp], cos, sin, rd, interleaved).T
        assert abs(c.item() - b.item()) > 1e-3


def test_rope_interleaved_is_half_split_on_permuted_dims():
    """Interleaved pairs (2i, 2i+1) are the half-split pairs (i, i + rd/2)
    after moving even dims to the front half and odd dims to the back."""
    d, rd = 24, 16
    cos, sin = _tables(20, rd // 2)
    x = _rand((6, d), 207)
    pos = [1, 4, 7, 9, 13, 19]
    perm = list(range(0, rd, 2)) + list(range(1, rd, 2)) + list(range(rd, d))
    inv = np.argsort(perm)
    a = oracle.rope(x, pos, cos, sin, rd, interleaved=True)
    b = oracle.rope(x[:, perm], pos, cos, sin, rd, interleaved=False)[:, inv]
    np.testing.assert_array_equal(a, b)


# --------------------------------------------------------------------------
# append + attend
# --------------------------------------------------------------------------
def _layout(ctx, page_size, Hq, Hkv, d, seed, extra_pages=2):
    """A paged cache with room for one more token per request."""
    gen = torch.Generator().manual_seed(seed)
    need = [(c + 1 + page_size - 1) // page_size for c in ctx]
    npages = sum(need) + extra_pages
    perm = torch.randperm(npages, generator=gen)
    maxb = max(need)
    bt = torch.full((len(ctx), maxb), -1, dtype=torch.int32)
    at = 0
    for b, n in enumerate(need):
        bt[b, :n] = perm[at:at + n].to(torch.int32)
        at += n
    B = len(ctx)
    q = inputs.randn_bf16((B, Hq, d), gen)
    kn = inputs.randn_bf16((B, Hkv, d), gen)
    vn = inputs.randn_bf16((B, Hkv, d), gen)
    kp = inputs.randn_bf16((npages, page_size, Hkv, d), gen)
    vp = inputs.randn_bf16((npages, page_size, Hkv, d), gen)
    return q, kn, vn, kp, vp, bt, torch.tensor(ctx, dtype=torch.int32)


def _write(kp, vp, bt, ctx, kn, vn, page_size):
    kp, vp = kp.clone(), vp.clone()
    for b, c in enumerate(ctx):
        page = int(bt[b, c // page_size])
        kp[page, c % page_size] = kn[b]
        vp[page, c % page_size] = vn[b]
    return kp, vp


@pytest.mark.parametrize("page_size", [1, 16, 5])
def test_append_without_rope_equals_decode_on_the_written_cache(page_size):
    ctx = [0, 1, 15, 16, 40, 3]
    q, kn, vn, kp, vp, bt, cs = _layout(ctx, page_size, 8, 2, 16, seed=211)
    o, lse, kp2, vp2, qr = oracle.decode_paged_append(q, kn, vn, kp, vp, bt, cs, 0.25)
    kref, vref = _write(kp, vp, bt, ctx, kn, vn, page_size)
    assert np.array_equal(kp2, kref.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(vp2, vref.view(torch.int16).numpy().view(np.uint16))
    o_ref, lse_ref = oracle.decode_paged(q, kref, vref, bt, cs + 1, 0.25)
    np.testing.assert_allclose(o, o_ref, atol=TOL, rtol=0)
    np.testing.assert_allclose(lse, lse_ref, atol=TOL, rtol=0)
    np.testing.assert_array_equal(qr, q.double().numpy())


@pytest.mark.parametrize("interleaved", [False, True])
@pytest.mark.parametrize("rd", [16, 10])
def test_append_with_rope_rotates_query_and_new_key_only(interleaved, rd):
    """With tables: the appended key is bf16(R(pos) k_new), v_new is stored as
    is, the query is bf16(R(pos) q), and the result is the plain decode of
    that query over the written cache of cache_seqlens + 1 tokens."""
    ctx, page_size, Hq, Hkv, d = [0, 7, 33, 64], 16, 4, 2, 16
    q, kn, vn, kp, vp, bt, cs = _layout(ctx, page_size, Hq, Hkv, d, seed=213)
    cos, sin = _tables(80, rd // 2)
    o, lse, kp2, vp2, qr = oracle.decode_paged_append(q, kn, vn, kp, vp, bt, cs, 0.3, cos, sin,
                                                      rd, interleaved)
    B = len(ctx)
    pos_q = np.repeat(np.array(ctx), Hq)
    pos_k = np.repeat(np.array(ctx), Hkv)
    q_rot = oracle.rope(q.reshape(B * Hq, d), pos_q, cos, sin, rd, interleaved)
    k_rot = oracle.rope(kn.reshape(B * Hkv, d), pos_k, cos, sin, rd, interleaved)
    q_b = torch.from_numpy(q_rot).to(torch.bfloat16).reshape(B, Hq, d)
    k_b = torch.from_numpy(k_rot).to(torch.bfloat16).reshape(B, Hkv, d)
    np.testing.assert_array_equal(qr, q_b.double().numpy())
    kref, vref = _write(kp, vp, bt, ctx, k_b, vn, page_size)
    assert np.array_equal(kp2, kref.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(vp2, vref.view(torch.int16).numpy().view(np.uint16))
    o_ref, lse_ref = oracle.decode_paged(q_b, kref, vref, bt, cs + 1, 0.3)
    np.testing.assert_allclose(o, o_ref, atol=TOL, rtol=0)
    np.testing.assert_allclose(lse, lse_ref, atol=TOL, rtol=0)


def test_append_first_token_attends_to_itself():
    """cache_seqlens = 0: the query sees only the token it appends, so O is
    v_new and LSE is scale * <q, k_new> (no rotation at position 0 when the
    table row 0 is the identity)."""
    q, kn, vn, kp, vp, bt, cs = _layout([0, 0], 4, 2, 1, 8, seed=215)
    cos, sin = _tables(4, 4)
    o, lse, *_ = oracle.decode_paged_append(q, kn, vn, kp, vp, bt, cs, 0.5, cos, sin, 8)
    for b in range(2):
        for h in range(2):
            np.testing.assert_array_equal(o[b, h], vn[b, 0].double().numpy())
            s = 0.5 * float((q[b, h].double() * kn[b, 0].double()).sum())
            assert abs(lse[b, h] - s) <= TOL


def test_rotated_query_is_rounded_to_nearest_bf16_ties_to_even():
    """The rotated vectors are rounded once to bf16, to nearest with ties to
    even.  With cos = 0.75 and sin = 0.5 (both exact) and bf16 inputs, every
    rotated value needs at most 12 significant bits, so it is exact in fp32
    and torch's fp32 -> bf16 conversion is the single correct rounding; the
    first pair lands exactly halfway between two bf16 values."""
    a = torch.tensor([1.0 + 2 ** -7, 3.0, -1.0, 1.25, 0.375, 0.5, -2.0], dtype=torch.float64)
    b = torch.tensor([0.5, 1.0, 0.25, 0.75, -0.5, 0.125, 1.5], dtype=torch.float64)
    half = a.numel()
    d = 2 * half
    q = torch.cat([a, b]).to(torch.bfloat16).reshape(1, 1, d)
    zeros = torch.zeros(1, 1, d, dtype=torch.bfloat16)
    kp = torch.zeros(1, 1, 1, d, dtype=torch.bfloat16)
    bt = torch.zeros(1, 1, dtype=torch.int32)
    cos, sin = torch.full((1, half), 0.75), torch.full((1, half), 0.5)
    *_, qr = oracle.decode_paged_append(q, zeros, zeros, kp, kp.clone(), bt,
                                        torch.tensor([0], dtype=torch.int32), 1.0, cos, sin, d)
    exact = torch.cat([0.75 * a - 0.5 * b, 0.5 * a + 0.75 * b])
    want = exact.float().to(torch.bfloat16).double()
    np.testing.assert_array_equal(qr[0, 0], want.numpy())
    # 0.5 + 3 * 2^-9 is a tie between 0.5 + 2^-8 and 0.5 + 2^-7: even wins
    assert exact[0].item() == 0.5 + 3 * 2 ** -9 and qr[0, 0, 0] == 0.5 + 2 ** -7
