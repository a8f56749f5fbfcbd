"""A seeded random sweep of paged split-KV decode configurations against the
fp64 oracle, through the C ABI: batches of 1-12 requests with contexts of 0
to ~3000 tokens, page sizes 1-80 (multiples of 16 take the TMA gather, the
rest the token-by-token gather), GQA groups 1-16 over 1-8 kv heads, head
sizes 64 and 128, and automatic or fixed split counts ("flash-attention"
skill page, appendices "PagedAttention" and "FlashDecoding / Split-KV").

Rows of one key (a context of one token) and the peaked rows of short
contexts are held, like the stress shapes elsewhere, to max-abs 1e-2 and
mean-abs 1e-3 above the rounding floor (parity.check_bf16); the LSE to 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_86_b200 import api, inputs
from parity import LSE_ABS, check_bf16, check_close, to_np

pytestmark = pytest.mark.gpu

N_CASES = 30


def _case(i):
    """Configuration i of the sweep (a pure function of i)."""
    rng = np.random.default_rng(8000 + i)
    B = int(rng.integers(1, 13))
    seq_lens = [0 if rng.random() < 0.1 else int(rng.integers(1, 3000)) for _ in range(B)]
    if max(seq_lens) == 0:
        seq_lens[0] = int(rng.integers(1, 3000))
    page_size = int(rng.choice([1, 3, 8, 16, 24, 32, 48, 64, 80]))
    Hkv = int(rng.choice([1, 2, 4, 8]))
    group = int(rng.choice([1, 2, 4, 8, 12, 16]))
    d = int(rng.choice([64, 128]))
    num_splits = 0 if rng.random() < 0.5 else int(rng.integers(1, 10))
    return seq_lens, Hkv * group, Hkv, d, page_size, num_splits


@pytest.mark.parametrize("i", range(N_CASES))
def test_random_decode_configuration(i):
    seq_lens, Hq, Hkv, d, page_size, num_splits = _case(i)
    inp = inputs.make_decode(seq_lens, Hq, Hkv, d, page_size, seed=8200 + i)
    q, kp, vp, bt, sl = (t.cuda() for t in (inp.q, inp.k_pages, inp.v_pages, inp.block_table,
                                            inp.seq_lens))
    o, lse = api.decode_paged(q, kp, vp, bt, sl, num_splits=num_splits, scale=inp.scale)
    torch.cuda.synchronize()
    assert api.device_error() == api.FA_OK
    o_ref, lse_ref = oracle.decode_paged(inp.q, inp.k_pages, inp.v_pages, inp.block_table,
                                         inp.seq_lens, inp.scale)
    what = f"case {i}: seq_lens {seq_lens} Hq {Hq} Hkv {Hkv} d {d} page {page_size} " \
           f"splits {num_splits}"
    check_bf16(to_np(o), o_ref, "O, " + what)
    check_close(to_np(lse), lse_ref, LSE_ABS, None, "LSE, " + what)
