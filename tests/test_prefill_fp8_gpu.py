"""Parity of the FP8 (e4m3) prefill with the fp64 oracle, through the C ABI
(fa_prefill_fp8).

The oracle computes the exact attention of the descaled e4m3 values.  The
kernel's only rounding beyond fp32 accumulation is that of the softmax
weights to e4m3 before the P V product (and of O to bf16).  For weights w_j
rounded to w_j (1 + e_j) with |e_j| <= 2^-4 (normal e4m3) -- or absolutely by
at most 2^-10 of the row's largest weight (values flushed below e4m3's
smallest subnormal) -- and O divided by the rounded sum, the error of each
output element is at most

    2^-3 / (1 - 2^-4) * sum_j w_j |v_j - O|  +  2^-9 * w_max * sum_j |v_j - O|

plus the bf16 rounding of O (2^-9 |O|).  That bound, computed per element
from the oracle's exact weights, is the tolerance here; the LSE, which uses
the unrounded sum, keeps the 1e-3 bound.  On the full-size workload the
bound is evaluated through |v_j - O| <= |v_j| + |O| (the triangle
inequality), which turns both sums into products with |V| and so needs no
L x L x d array: a slightly looser bound, still a derived one.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_86_b200 import api, inputs
from parity import LSE_ABS, check_close, to_np

pytestmark = pytest.mark.gpu


def run(inp):
    qs, ks, vs = inp.meta["descale"]
    q, k, v, cu = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.cu_seqlens))
    o, lse = api.prefill_fp8(q, k, v, cu, causal=inp.causal, scale=inp.scale, q_descale=qs,
                             k_descale=ks, v_descale=vs, max_seqlen=max(inp.lengths))
    torch.cuda.synchronize()
    assert api.device_error() == api.FA_OK
    return to_np(o), to_np(lse)


def check_rows(inp, o, lse, pairs=None, loose=False):
    qs, ks, vs = inp.meta["descale"]
    q64, k64, v64 = inp.q.double() * qs, inp.k.double() * ks, inp.v.double() * vs
    o_ref, lse_ref = oracle.prefill_fp8(inp.q, inp.k, inp.v, inp.cu_seqlens, inp.causal, inp.scale,
                                        qs, ks, vs)
    check_close(lse, lse_ref, LSE_ABS, None, "LSE")
    Hq, Hkv = inp.q.shape[1], inp.k.shape[1]
    cu = inp.cu_seqlens.tolist()
    if pairs is None:
        pairs = [(b, h) for b in range(len(cu) - 1) for h in range(Hq)]
    worst = 0.0
    for b, h in pairs:
        s0, s1 = cu[b], cu[b + 1]
        if s1 == s0:
            continue
        P = oracle.prefill_probs(q64, k64, inp.cu_seqlens, inp.causal, inp.scale, b, h, Hkv)
        V = v64[s0:s1, h // (Hq // Hkv)].numpy()                   # [L, d]
        O = o_ref[s0:s1, h]                                         # [L, d]
        if loose:
            # sum_j w_j |v_j - O| <= (P |V|) + |O|;  sum_j |v_j - O| <= sum_j |v_j| + n |O|
            # over the visible keys j (where P > 0)
            vis = (P > 0).astype(np.float64)
            rel = P @ np.abs(V) + np.abs(O)
            tot = vis @ np.abs(V) + vis.sum(axis=1, keepdims=True) * np.abs(O)
        else:
            dev = np.abs(V[None, :, :] - O[:, None, :])             # [L, L, d]
            rel = np.einsum("ij,ijc->ic", P, dev)
            tot = dev.sum(axis=1)
        bound = (2.0 ** -3 / (1 - 2.0 ** -4)) * rel \
            + 2.0 ** -9 * P.max(axis=1, keepdims=True) * tot \
            + 2.0 ** -9 * np.abs(O) + 1e-6
        err = np.abs(o[s0:s1, h] - O)
        ratio = (err / bound).max()
        worst = max(worst, ratio)
        assert ratio <= 1.0, f"(b={b}, h={h}): error {err.max():.3e} exceeds the derived bound"
    return worst


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("L", [1, 17, 128, 129, 300, 700])
def test_single_sequence(L, causal):
    inp = inputs.make_prefill_fp8([L], 4, 2, 128, causal, seed=7000 + L)
    o, lse = run(inp)
    check_rows(inp, o, lse)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_gqa(causal):
    inp = inputs.make_prefill_fp8([0, 5, 257, 129, 640], 8, 2, 128, causal, seed=7100)
    o, lse = run(inp)
    check_rows(inp, o, lse)


def test_descale_factors():
    """Wider e4m3 values with descales that bring them back to unit scale."""
    inp = inputs.make_prefill_fp8([333, 200], 4, 4, 128, True, seed=7200, spread=(8.0, 0.25, 30.0))
    o, lse = run(inp)
    check_rows(inp, o, lse)


def test_fp8_workload_every_pair():
    """Causal B=4 H=16 L=2048 d=128 in e4m3: the LSE everywhere and O on all
    64 (sequence, head) pairs, every row, against the derived bound."""
    inp = inputs.fp8_prefill()
    o, lse = run(inp)
    check_rows(inp, o, lse, loose=True)


def _random_case(i):
    """Configuration i of a seeded random sweep (a pure function of i): 1-4
    packed sequences of 1-400 tokens, GQA groups 1-8, causal or full, and
    per-tensor spreads that the descales bring back to unit scale."""
    rng = np.random.default_rng(7400 + i)
    lengths = [int(rng.integers(1, 400)) for _ in range(int(rng.integers(1, 5)))]
    Hkv = int(rng.choice([1, 2, 4]))
    group = int(rng.choice([1, 2, 4, 8]))
    causal = bool(rng.random() < 0.6)
    spread = tuple(float(x) for x in rng.choice([0.5, 1.0, 4.0, 16.0], size=3))
    return lengths, Hkv * group, Hkv, causal, spread


@pytest.mark.parametrize("i", range(16))
def test_random_configuration(i):
    lengths, Hq, Hkv, causal, spread = _random_case(i)
    inp = inputs.make_prefill_fp8(lengths, Hq, Hkv, 128, causal, seed=7500 + i, spread=spread)
    o, lse = run(inp)
    # the exact form of the bound holds an L x L x d array per pair: the
    # triangle-inequality form above 256 tokens
    check_rows(inp, o, lse, loose=max(lengths) > 256)


def test_rejects_bad_descale_and_head_dim():
    inp = inputs.make_prefill_fp8([16], 2, 2, 128, True, seed=7300)
    q, k, v, cu = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.cu_seqlens))
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(api.FAError) as e:
            api.prefill_fp8(q, k, v, cu, causal=True, q_descale=bad)
        assert e.value.code == api.FA_ERR_INVALID_ARG
    q64 = torch.zeros(16, 2, 64, dtype=torch.float8_e4m3fn, device="cuda")
    with pytest.raises(api.FAError) as e:
        api.prefill_fp8(q64, q64, q64, cu, causal=True)
    assert e.value.code == api.FA_ERR_UNSUPPORTED
