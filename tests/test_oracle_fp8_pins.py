"""Pins of the oracle's FP8 prefill (Q, K, V as e4m3 with per-tensor
descale factors; the pages list FP8 among the supported data types).

The e4m3 decoder is checked against torch's float8_e4m3fn conversion for all
256 byte values (a library routine), and the FP8 prefill against the pinned
fp64 prefill on the decoded, descaled values.
"""
import math

import numpy as np
import torch

import oracle
from exact_io_aware_86_b200 import inputs


def test_e4m3_decoder_matches_torch_for_every_byte():
    b = torch.arange(256, dtype=torch.uint8)
    ref = b.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_value(int(x)) for x in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # a few values by hand: 0x38 = 1.0, 0x7E = 448 (largest), 0x01 = 2^-9 (smallest)
    assert got[0x38] == 1.0 and got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9
    assert got[0xB8] == -1.0 and got[0x08] == 2.0 ** -6


def test_fp8_prefill_is_the_definition_on_descaled_values():
    lengths, Hq, Hkv, d = [37, 1, 130], 4, 2, 32
    T = sum(lengths)
    g = torch.Generator().manual_seed(301)
    q = (torch.randn(T, Hq, d, generator=g) * 2).to(torch.float8_e4m3fn)
    k = torch.randn(T, Hkv, d, generator=g).to(torch.float8_e4m3fn)
    v = (torch.randn(T, Hkv, d, generator=g) * 3).to(torch.float8_e4m3fn)
    cu = inputs.cu_seqlens_of(lengths)
    qs, ks, vs = 0.5, 1.25, 0.0625
    for causal in (False, True):
        o, lse = oracle.prefill_fp8(q, k, v, cu, causal, 0.2, qs, ks, vs)
        o_ref, lse_ref = oracle.prefill(q.double() * qs, k.double() * ks, v.double() * vs, cu,
                                        causal, 0.2)
        np.testing.assert_array_equal(o, o_ref)
        np.testing.assert_array_equal(lse, lse_ref)


def test_fp8_descales_scale_the_logits_and_the_output():
    """q_descale * k_descale multiplies every logit (so it acts like the
    softmax scale) and v_descale multiplies O; LSE ignores v_descale."""
    lengths, H, d = [50], 2, 16
    g = torch.Generator().manual_seed(303)
    q = torch.randn(50, H, d, generator=g).to(torch.float8_e4m3fn)
    k = torch.randn(50, H, d, generator=g).to(torch.float8_e4m3fn)
    v = torch.randn(50, H, d, generator=g).to(torch.float8_e4m3fn)
    cu = inputs.cu_seqlens_of(lengths)
    o1, l1 = oracle.prefill_fp8(q, k, v, cu, True, 0.3, 2.0, 0.5, 4.0)
    o2, l2 = oracle.prefill_fp8(q, k, v, cu, True, 0.3, 1.0, 1.0, 1.0)
    np.testing.assert_allclose(o1, 4.0 * o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)
    o3, l3 = oracle.prefill_fp8(q, k, v, cu, True, 0.6, 1.0, 1.0, 1.0)
    o4, l4 = oracle.prefill_fp8(q, k, v, cu, True, 0.3, 2.0, 1.0, 1.0)
    np.testing.assert_allclose(o3, o4, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l3, l4, rtol=0, atol=1e-12)
