"""A seeded random sweep of prefill configurations against the fp64 oracle,
through the C ABI: packed lengths with ragged tails (1 token up to ~1000,
around the 128-row tile edges), GQA groups 1-8, head sizes 64 and 128,
causal or full masks, and every mask variant of the "flash-attention" skill
page, section 3.3 (sliding windows, softcap, ALiBi per head or per
(sequence, head), and their combinations), so that each of the prefill
kernels (plain, band alone, causal ALiBi, softcap, and the general in-place
kernel) meets shapes the targeted tests do not name.

Random variants make peaked rows (one- or two-key windows, steep slopes,
short sequences), so every case is held to the peaked-row bound of
parity.check_bf16_peaked (max-abs 1e-2 + 2^-8 |O|, mean-abs 1e-3 above the
rounding floor) and the LSE to 1e-3; the targeted tests hold the named
workloads to the plain bounds.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_86_b200 import api, inputs
from parity import LSE_ABS, check_bf16_peaked, check_close, to_np

pytestmark = pytest.mark.gpu

N_CASES = 40


def _case(i):
    """Configuration i of the sweep (a pure function of i)."""
    rng = np.random.default_rng(7000 + i)
    n_seq = int(rng.integers(1, 5))
    pool = [1, 2, 127, 128, 129, 255, 256, 257]
    lengths = [int(rng.choice(pool)) if rng.random() < 0.4 else int(rng.integers(1, 1000))
               for _ in range(n_seq)]
    Hkv = int(rng.choice([1, 2, 4]))
    group = int(rng.choice([1, 2, 4, 8]))
    d = int(rng.choice([64, 128]))
    causal = bool(rng.random() < 0.6)
    variant = {}
    kind = int(rng.integers(0, 6))
    if kind in (1, 4, 5):
        left = int(rng.choice([-1, 0, 1, int(rng.integers(2, 600))]))
        right = 0 if causal else int(rng.choice([-1, 0, 1, int(rng.integers(2, 600))]))
        variant["window"] = (left, right)
    if kind in (2, 4, 5):
        variant["softcap"] = float(rng.uniform(2.0, 50.0))
    if kind in (3, 5) or (kind == 4 and rng.random() < 0.5):
        gen = torch.Generator().manual_seed(7100 + i)
        shape = (Hkv * group,) if rng.random() < 0.5 else (n_seq, Hkv * group)
        variant["alibi_slopes"] = inputs.uniform_slopes(shape, 0.0, 0.3, gen)
    scale = None if rng.random() < 0.5 else float(rng.uniform(0.05, 0.2))
    return lengths, Hkv * group, Hkv, d, causal, variant, scale


@pytest.mark.parametrize("i", range(N_CASES))
def test_random_prefill_configuration(i):
    lengths, Hq, Hkv, d, causal, variant, scale = _case(i)
    inp = inputs.make_prefill(lengths, Hq, Hkv, d, causal, seed=7200 + i, scale=scale)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    cu = inp.cu_seqlens.cuda()
    dev_variant = dict(variant)
    if dev_variant.get("alibi_slopes") is not None:
        dev_variant["alibi_slopes"] = dev_variant["alibi_slopes"].cuda()
    o, lse = api.prefill(q, k, v, cu, causal=causal, scale=inp.scale, **dev_variant)
    torch.cuda.synchronize()
    assert api.device_error() == api.FA_OK
    o_ref, lse_ref = oracle.prefill(inp.q, inp.k, inp.v, inp.cu_seqlens, causal, inp.scale,
                                    **variant)
    what = f"case {i}: lengths {lengths} Hq {Hq} Hkv {Hkv} d {d} causal {causal} " \
           f"variant {sorted(variant)} scale {inp.scale:.4f}"
    check_bf16_peaked(to_np(o), o_ref, "O, " + what)
    check_close(to_np(lse), lse_ref, LSE_ABS, None, "LSE, " + what)
