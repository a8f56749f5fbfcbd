"""Parity of the decode step with cache append and RoPE ("flash-attention"
skill page, section 3.5) with the fp64 oracle, through the C ABI
(fa_decode_paged_append).

O and LSE are held to the bf16 bounds; the page pools after the call must
equal the oracle's updated copies bit for bit (the rotated key is the exact
rotation rounded once to bf16 on both sides), which also checks that no other
slot was touched.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_86_b200 import api, inputs
from parity import LSE_ABS, check_bf16, check_close, to_np

pytestmark = pytest.mark.gpu


def run(inp, num_splits=0):
    dev = "cuda"
    q, kn, vn = (t.to(dev) for t in (inp.q, inp.k_new, inp.v_new))
    kp, vp = inp.k_pages.to(dev), inp.v_pages.to(dev)
    bt, cs = inp.block_table.to(dev), inp.cache_seqlens.to(dev)
    cos = inp.cos.to(dev) if inp.cos is not None else None
    sin = inp.sin.to(dev) if inp.sin is not None else None
    o, lse = api.decode_paged_append(q, kn, vn, kp, vp, bt, cs, num_splits=num_splits,
                                     scale=inp.scale, rotary_cos=cos, rotary_sin=sin,
                                     rotary_dim=inp.rotary_dim or None,
                                     rotary_interleaved=inp.interleaved)
    torch.cuda.synchronize()
    err = api.device_error()
    return to_np(o), to_np(lse), kp.cpu(), vp.cpu(), err


def reference(inp):
    return oracle.decode_paged_append(inp.q, inp.k_new, inp.v_new, inp.k_pages, inp.v_pages,
                                      inp.block_table, inp.cache_seqlens, inp.scale, inp.cos,
                                      inp.sin, inp.rotary_dim or None, inp.interleaved)


def bits(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def assert_matches(inp, num_splits=0):
    o, lse, kp, vp, err = run(inp, num_splits)
    assert err == api.FA_OK
    o_ref, lse_ref, kp_ref, vp_ref, _ = reference(inp)
    assert np.array_equal(bits(kp), kp_ref), "k page pool differs from the oracle's"
    assert np.array_equal(bits(vp), vp_ref), "v page pool differs from the oracle's"
    check_bf16(o, o_ref, "O")
    check_close(lse, lse_ref, LSE_ABS, None, "LSE")


CTX = [0, 1, 15, 16, 17, 31, 63, 64, 200, 1000]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("page_size", [16, 64])
@pytest.mark.parametrize("heads", [(8, 8), (32, 8), (16, 2)])
def test_append_without_rope(heads, page_size, d):
    Hq, Hkv = heads
    inp = inputs.make_append_decode(CTX, Hq, Hkv, d, page_size, seed=6000 + Hq + page_size + d)
    assert_matches(inp)


@pytest.mark.parametrize("rotary", [(128, False), (128, True), (64, False), (2, True)])
@pytest.mark.parametrize("num_splits", [1, 3, 0])
def test_append_with_rope(rotary, num_splits):
    rd, inter = rotary
    inp = inputs.make_append_decode(CTX, 32, 8, 128, 16, seed=6100 + rd + inter, rotary_dim=rd,
                                    interleaved=inter, max_pos=1200)
    assert_matches(inp, num_splits)


def test_append_rope_d64_partial():
    inp = inputs.make_append_decode([5, 77, 300], 8, 4, 64, 16, seed=6200, rotary_dim=32,
                                    interleaved=False, max_pos=400)
    assert_matches(inp)


def test_append_workload_full_size():
    """64 requests, ctx U[1024, 32767], Hq=32 Hkv=8 d=128, page 16, RoPE over
    all 128 dims: O and LSE of every request, and the whole page pool."""
    inp = inputs.append_decode()
    assert_matches(inp)


def test_position_outside_the_table_is_rejected_per_request():
    """A request whose cache is already full (cache_seqlens = max_blocks *
    page_size) cannot append: the kernel records a bounds error, writes
    nothing for it and returns O = 0, LSE = -inf; the others are unaffected."""
    inp = inputs.make_append_decode([10, 40, 5], 8, 8, 128, 16, seed=6300)
    full = inp.block_table.shape[1] * inp.page_size
    bad = inputs.AppendInputs(**{**inp.__dict__, "cache_seqlens": torch.tensor([10, full, 5], dtype=torch.int32)})
    o, lse, kp, vp, err = run(bad)
    assert err == api.FA_ERR_DEVICE_BOUNDS
    assert np.all(o[1] == 0) and np.all(np.isneginf(lse[1]))
    good = inputs.AppendInputs(**{**inp.__dict__})
    o_ref, lse_ref, kp_ref, vp_ref, _ = reference(good)
    for b in (0, 2):
        check_bf16(o[b], o_ref[b], "O")
        check_close(lse[b], lse_ref[b], LSE_ABS, None, "LSE")
    # request 1 wrote nothing: the pools equal the oracle's, whose request-1
    # append landed in the slot of position 40 (its own page); undo that one
    page = int(inp.block_table[1, 40 // 16])
    kp_ref[page, 40 % 16] = bits(inp.k_pages)[page, 40 % 16]
    vp_ref[page, 40 % 16] = bits(inp.v_pages)[page, 40 % 16]
    assert np.array_equal(bits(kp), kp_ref) and np.array_equal(bits(vp), vp_ref)
