"""A seeded random sweep of the decode step with cache append and RoPE
("flash-attention" skill page, section 3.5) against the fp64 oracle, through
the C ABI: contexts of 0 to ~2000 tokens, any page size (1-80, both
gathers), GQA groups 1-16, head sizes 64 and 128, no rotation or a full,
partial or interleaved one, and automatic or fixed split counts.

O and LSE are held to the bf16 bounds (mean above the rounding floor, as for
the other stress shapes); both page pools must equal the oracle's updated
copies bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_86_b200 import api, inputs
from parity import LSE_ABS, check_bf16, check_close, to_np

pytestmark = pytest.mark.gpu

N_CASES = 20


def _case(i):
    """Configuration i of the sweep (a pure function of i)."""
    rng = np.random.default_rng(9000 + i)
    B = int(rng.integers(1, 9))
    ctx = [0 if rng.random() < 0.15 else int(rng.integers(1, 2000)) for _ in range(B)]
    page_size = int(rng.choice([1, 3, 8, 16, 24, 64, 80]))
    Hkv = int(rng.choice([1, 2, 4, 8]))
    group = int(rng.choice([1, 2, 4, 8, 12, 16]))
    d = int(rng.choice([64, 128]))
    kind = int(rng.integers(0, 4))
    if kind == 0:
        rotary_dim, interleaved = 0, False
    else:
        rotary_dim = d if kind == 1 else int(rng.choice([2, 16, 32, d // 2]))
        interleaved = bool(rng.random() < 0.5)
    num_splits = 0 if rng.random() < 0.5 else int(rng.integers(1, 8))
    return ctx, Hkv * group, Hkv, d, page_size, rotary_dim, interleaved, num_splits


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("i", range(N_CASES))
def test_random_append_configuration(i):
    ctx, Hq, Hkv, d, page_size, rd, inter, num_splits = _case(i)
    inp = inputs.make_append_decode(ctx, Hq, Hkv, d, page_size, seed=9200 + i, rotary_dim=rd,
                                    interleaved=inter, max_pos=max(ctx) + 8 if rd else None)
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
    assert api.device_error() == api.FA_OK
    o_ref, lse_ref, kp_ref, vp_ref, _ = oracle.decode_paged_append(
        inp.q, inp.k_new, inp.v_new, inp.k_pages, inp.v_pages, inp.block_table,
        inp.cache_seqlens, inp.scale, inp.cos, inp.sin, inp.rotary_dim or None, inp.interleaved)
    what = f"case {i}: ctx {ctx} Hq {Hq} Hkv {Hkv} d {d} page {page_size} rotary {rd} " \
           f"interleaved {inter} splits {num_splits}"
    assert np.array_equal(_bits(kp.cpu()), kp_ref), "k page pool differs, " + what
    assert np.array_equal(_bits(vp.cpu()), vp_ref), "v page pool differs, " + what
    check_bf16(to_np(o), o_ref, "O, " + what)
    check_close(to_np(lse), lse_ref, LSE_ABS, None, "LSE, " + what)
