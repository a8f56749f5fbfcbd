"""Seeded synthetic inputs for the exact-attention workloads.

This module only draws random numbers and lays them out: sequence lengths,
packed Q/K/V tensors, the page pool and its block table.  It holds none of
the attention arithmetic, so the CUDA path and the CPU oracle can both be fed
from it without sharing any of the method.

Recipe (every workload): a ``torch.Generator`` on the CPU seeded with the
workload's seed draws, in this order, (1) sequence/context lengths, (2) the
page permutation (paged workloads), (3) q, (4) k, (5) v.  Values are fp32
N(0, 1) rounded to bf16 (round-to-nearest-even); the fp32 originals are kept
where a workload also needs them.  Large tensors are drawn in fixed-size
chunks in a fixed order, so the bits depend only on the seed.

Workload shapes follow the pages' cases: head_dim 128 at sequence length
2048 (skill page appendix "performance reference"), 32 query heads over 8
kv heads (skill page, GQA/MQA appendix), packed varlen batches described by
cu_seqlens (skill page section 3.4), and paged KV caches addressed by a
block table (skill page, PagedAttention appendix).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

_CHUNK = 1 << 24


def randn_f32(shape, gen: torch.Generator) -> torch.Tensor:
    """fp32 N(0,1) of ``shape``, drawn in fixed chunks so the result depends only on the seed."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.float32)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        out[s:e] = torch.randn(e - s, generator=gen, dtype=torch.float32)
    return out.view(*shape)


def randn_bf16(shape, gen: torch.Generator) -> torch.Tensor:
    """bf16 N(0,1): fp32 draws rounded to nearest-even, chunk by chunk."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.bfloat16)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        out[s:e] = torch.randn(e - s, generator=gen, dtype=torch.float32).to(torch.bfloat16)
    return out.view(*shape)


def uniform_lengths(n: int, lo: int, hi: int, gen: torch.Generator) -> list[int]:
    """``n`` integers uniform on [lo, hi] inclusive."""
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=gen)]


def cu_seqlens_of(lengths) -> torch.Tensor:
    """int32 [B+1] running totals of the lengths, starting at 0 (the varlen layout)."""
    out = [0]
    for L in lengths:
        out.append(out[-1] + int(L))
    return torch.tensor(out, dtype=torch.int32)


def paged_layout(seq_lens, page_size: int, gen: torch.Generator):
    """Scatter each request's pages over a pool by a seeded permutation.

    The pool holds exactly sum(ceil(len/page_size)) pages.  Request b takes
    the next ceil(len_b/page_size) entries of ``randperm(pool)``; unused
    block-table entries are -1.  Returns (block_table int32 [B, max_blocks],
    num_pages).
    """
    need = [(int(L) + page_size - 1) // page_size for L in seq_lens]
    num_pages = sum(need)
    max_blocks = max(need) if need else 0
    perm = torch.randperm(num_pages, generator=gen).to(torch.int32)
    bt = torch.full((len(need), max(max_blocks, 1)), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(need):
        bt[b, :n] = perm[off:off + n]
        off += n
    return bt, num_pages


@dataclass
class PrefillInputs:
    name: str
    q: torch.Tensor            # [T, Hq, d] bf16
    k: torch.Tensor            # [T, Hkv, d] bf16
    v: torch.Tensor            # [T, Hkv, d] bf16
    cu_seqlens: torch.Tensor   # [B+1] int32
    lengths: list
    causal: bool
    scale: float               # the fp32 value both sides receive
    q32: torch.Tensor | None = None   # fp32 originals (tiny workload only)
    k32: torch.Tensor | None = None
    v32: torch.Tensor | None = None
    meta: dict = field(default_factory=dict)

    @property
    def B(self):
        return len(self.lengths)

    @property
    def Hq(self):
        return self.q.shape[1]

    @property
    def Hkv(self):
        return self.k.shape[1]

    @property
    def d(self):
        return self.q.shape[2]

    @property
    def T(self):
        return self.q.shape[0]


@dataclass
class DecodeInputs:
    name: str
    q: torch.Tensor            # [B, Hq, d] bf16
    k_pages: torch.Tensor      # [num_pages, page_size, Hkv, d] bf16
    v_pages: torch.Tensor
    block_table: torch.Tensor  # [B, max_blocks] int32, -1 unused
    seq_lens: torch.Tensor     # [B] int32
    page_size: int
    scale: float
    meta: dict = field(default_factory=dict)

    @property
    def B(self):
        return self.q.shape[0]

    @property
    def Hq(self):
        return self.q.shape[1]

    @property
    def Hkv(self):
        return self.k_pages.shape[2]

    @property
    def d(self):
        return self.q.shape[2]

    @property
    def num_pages(self):
        return self.k_pages.shape[0]


def fp32_scale(d: int) -> float:
    """The default softmax scale 1/sqrt(head_dim), rounded once to fp32."""
    return float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32).item())


def make_prefill(lengths, Hq: int, Hkv: int, d: int, causal: bool, seed: int,
                 name: str = "prefill", keep_f32: bool = False,
                 scale: float | None = None) -> PrefillInputs:
    """Packed prefill inputs for the given sequence lengths."""
    gen = torch.Generator().manual_seed(seed)
    T = sum(int(L) for L in lengths)
    if keep_f32:
        q32 = randn_f32((T, Hq, d), gen)
        k32 = randn_f32((T, Hkv, d), gen)
        v32 = randn_f32((T, Hkv, d), gen)
        q, k, v = (x.to(torch.bfloat16) for x in (q32, k32, v32))
    else:
        q32 = k32 = v32 = None
        q = randn_bf16((T, Hq, d), gen)
        k = randn_bf16((T, Hkv, d), gen)
        v = randn_bf16((T, Hkv, d), gen)
    return PrefillInputs(name=name, q=q, k=k, v=v, cu_seqlens=cu_seqlens_of(lengths),
                         lengths=[int(L) for L in lengths], causal=causal,
                         scale=fp32_scale(d) if scale is None else scale,
                         q32=q32, k32=k32, v32=v32, meta={"seed": seed})


def make_decode(seq_lens, Hq: int, Hkv: int, d: int, page_size: int, seed: int,
                name: str = "decode", scale: float | None = None) -> DecodeInputs:
    """Paged decode inputs for the given context lengths."""
    gen = torch.Generator().manual_seed(seed)
    bt, num_pages = paged_layout(seq_lens, page_size, gen)
    B = len(seq_lens)
    q = randn_bf16((B, Hq, d), gen)
    k = randn_bf16((num_pages, page_size, Hkv, d), gen)
    v = randn_bf16((num_pages, page_size, Hkv, d), gen)
    return DecodeInputs(name=name, q=q, k_pages=k, v_pages=v, block_table=bt,
                        seq_lens=torch.tensor([int(x) for x in seq_lens], dtype=torch.int32),
                        page_size=page_size, scale=fp32_scale(d) if scale is None else scale,
                        meta={"seed": seed})


# ---------------------------------------------------------------------------
# The five named workloads.  Seed 1000 + k for workload k.
# ---------------------------------------------------------------------------

WORKLOADS = {
    "tiny": "B=1 H=1 L=256 d=64 fp32 N(0,1) with a bf16 copy, causal and non-causal",
    "mha_prefill": "causal MHA prefill B=4 Hq=Hkv=16 L=2048 d=128 bf16",
    "varlen_gqa_prefill": "varlen GQA causal prefill, 8 seqs L~U[512,8192], Hq=32 Hkv=8 d=128",
    "paged_decode": "paged decode, 64 requests, Hq=32 Hkv=8 d=128, ctx~U[1024,32768], page 16",
    "long_decode": "split-KV decode, 2 requests x 131072 ctx, Hq=32 Hkv=8 d=128, page 64",
    # mask variants of the skill page's advanced-features table (section 3.3)
    "window_prefill": "sliding-window causal prefill, window (4096, 0), 2 seqs x 16384, "
                      "Hq=32 Hkv=8 d=128",
    "softcap_prefill": "causal MHA prefill B=4 Hq=Hkv=16 L=2048 d=128 with softcap 50",
    "alibi_prefill": "causal MHA prefill B=4 Hq=Hkv=16 L=2048 d=128 with ALiBi slopes",
    "fp8_prefill": "causal MHA prefill B=4 Hq=Hkv=16 L=2048 d=128, Q/K/V in e4m3",
    # inference KV cache step (skill page section 3.5)
    "append_decode": "paged decode with cache append + RoPE (rotary_dim 128), 64 requests, "
                     "Hq=32 Hkv=8 d=128, ctx~U[1024,32767], page 16",
}


def alibi_slopes_geometric(H: int) -> torch.Tensor:
    """fp32 [H]: the geometric slope sequence 2^(-8 (h+1) / H) that ALiBi
    models use for H heads (H a power of two).  The pages give the ALiBi
    argument's shape but no values; this is input data, not the method."""
    return torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float32)


def uniform_slopes(shape, lo: float, hi: float, gen: torch.Generator) -> torch.Tensor:
    """fp32 slopes drawn uniformly from [lo, hi)."""
    return (torch.rand(*shape, generator=gen, dtype=torch.float32) * (hi - lo) + lo).contiguous()


def tiny(causal: bool) -> PrefillInputs:
    return make_prefill([256], 1, 1, 64, causal, seed=1001, name="tiny", keep_f32=True)


def mha_prefill() -> PrefillInputs:
    return make_prefill([2048] * 4, 16, 16, 128, True, seed=1002, name="mha_prefill")


def varlen_gqa_prefill() -> PrefillInputs:
    gen = torch.Generator().manual_seed(1003)
    lengths = uniform_lengths(8, 512, 8192, gen)
    T = sum(lengths)
    q = randn_bf16((T, 32, 128), gen)
    k = randn_bf16((T, 8, 128), gen)
    v = randn_bf16((T, 8, 128), gen)
    return PrefillInputs(name="varlen_gqa_prefill", q=q, k=k, v=v,
                         cu_seqlens=cu_seqlens_of(lengths), lengths=lengths, causal=True,
                         scale=fp32_scale(128), meta={"seed": 1003})


def make_prefill_fp8(lengths, Hq: int, Hkv: int, d: int, causal: bool, seed: int,
                     name: str = "prefill_fp8", spread=(1.0, 1.0, 1.0)) -> PrefillInputs:
    """e4m3 inputs: fp32 N(0, spread^2) draws rounded to float8_e4m3fn (round to
    nearest even).  ``meta['descale']`` holds the per-tensor factors (1/spread
    each) that bring the values back to unit scale."""
    gen = torch.Generator().manual_seed(seed)
    T = sum(int(L) for L in lengths)
    q = (randn_f32((T, Hq, d), gen) * spread[0]).to(torch.float8_e4m3fn)
    k = (randn_f32((T, Hkv, d), gen) * spread[1]).to(torch.float8_e4m3fn)
    v = (randn_f32((T, Hkv, d), gen) * spread[2]).to(torch.float8_e4m3fn)
    return PrefillInputs(name=name, q=q, k=k, v=v, cu_seqlens=cu_seqlens_of(lengths),
                         lengths=[int(L) for L in lengths], causal=causal, scale=fp32_scale(d),
                         meta={"seed": seed, "descale": tuple(1.0 / x for x in spread)})


def fp8_prefill() -> PrefillInputs:
    """The causal MHA workload's shape in e4m3 (descale factors 1)."""
    return make_prefill_fp8([2048] * 4, 16, 16, 128, True, seed=1008, name="fp8_prefill")


def window_prefill() -> PrefillInputs:
    """Mistral-style sliding window (4096, 0) (skill page, section 3.3) over
    two long sequences."""
    inp = make_prefill([16384, 16384], 32, 8, 128, True, seed=1006, name="window_prefill")
    inp.meta["variant"] = {"window": (4096, 0)}
    return inp


def softcap_prefill() -> PrefillInputs:
    """The causal MHA workload with the page's example cap, softcap=50."""
    inp = mha_prefill()
    inp.name = "softcap_prefill"
    inp.meta["variant"] = {"softcap": 50.0}
    return inp


def alibi_prefill() -> PrefillInputs:
    """The causal MHA workload with one ALiBi slope per head."""
    inp = mha_prefill()
    inp.name = "alibi_prefill"
    inp.meta["variant"] = {"alibi_slopes": alibi_slopes_geometric(16)}
    return inp


@dataclass
class AppendInputs:
    """One decode step that appends a token per request (skill page 3.5)."""
    name: str
    q: torch.Tensor              # [B, Hq, d] bf16
    k_new: torch.Tensor          # [B, Hkv, d] bf16
    v_new: torch.Tensor
    k_pages: torch.Tensor        # [num_pages, page_size, Hkv, d] bf16 (room for ctx + 1)
    v_pages: torch.Tensor
    block_table: torch.Tensor    # [B, max_blocks] int32
    cache_seqlens: torch.Tensor  # [B] int32: tokens already cached
    page_size: int
    scale: float
    cos: torch.Tensor | None     # [max_pos, rotary_dim / 2] fp32
    sin: torch.Tensor | None
    rotary_dim: int
    interleaved: bool
    meta: dict = field(default_factory=dict)

    @property
    def B(self):
        return self.q.shape[0]

    @property
    def Hq(self):
        return self.q.shape[1]

    @property
    def Hkv(self):
        return self.k_pages.shape[2]

    @property
    def d(self):
        return self.q.shape[2]


def rope_tables(max_pos: int, rotary_dim: int, base: float = 10000.0):
    """fp32 cos/sin tables [max_pos, rotary_dim/2] of the angles
    pos * base^(-2i/rotary_dim), the usual RoPE frequencies (computed in
    fp64, rounded once).  Input data: the pages give the argument, not its
    values."""
    half = rotary_dim // 2
    pos = torch.arange(max_pos, dtype=torch.float64).unsqueeze(1)
    inv = base ** (-2.0 * torch.arange(half, dtype=torch.float64) / rotary_dim)
    ang = pos * inv
    return torch.cos(ang).float().contiguous(), torch.sin(ang).float().contiguous()


def make_append_decode(ctx, Hq: int, Hkv: int, d: int, page_size: int, seed: int,
                       rotary_dim: int = 0, interleaved: bool = False, max_pos: int | None = None,
                       name: str = "append_decode") -> AppendInputs:
    """Paged cache holding ctx[b] tokens of request b, with room for one more
    (pages placed by a seeded permutation), plus the new token's q/k/v."""
    gen = torch.Generator().manual_seed(seed)
    bt, num_pages = paged_layout([int(c) + 1 for c in ctx], page_size, gen)
    B = len(ctx)
    q = randn_bf16((B, Hq, d), gen)
    k_new = randn_bf16((B, Hkv, d), gen)
    v_new = randn_bf16((B, Hkv, d), gen)
    k = randn_bf16((num_pages, page_size, Hkv, d), gen)
    v = randn_bf16((num_pages, page_size, Hkv, d), gen)
    cos = sin = None
    if rotary_dim:
        cos, sin = rope_tables(max_pos if max_pos is not None else max(ctx) + 1, rotary_dim)
    return AppendInputs(name=name, q=q, k_new=k_new, v_new=v_new, k_pages=k, v_pages=v,
                        block_table=bt, cache_seqlens=torch.tensor([int(c) for c in ctx], dtype=torch.int32),
                        page_size=page_size, scale=fp32_scale(d), cos=cos, sin=sin,
                        rotary_dim=rotary_dim, interleaved=interleaved, meta={"seed": seed})


def append_decode() -> AppendInputs:
    """The paged-decode workload's shape, one token appended per request, with
    RoPE over the full head dimension."""
    gen = torch.Generator().manual_seed(1007)
    ctx = uniform_lengths(64, 1024, 32767, gen)
    return make_append_decode(ctx, 32, 8, 128, 16, seed=1007, rotary_dim=128, max_pos=32768)


def _decode_from_lengths(name, seq_lens, page_size, seed, gen):
    bt, num_pages = paged_layout(seq_lens, page_size, gen)
    B = len(seq_lens)
    q = randn_bf16((B, 32, 128), gen)
    k = randn_bf16((num_pages, page_size, 8, 128), gen)
    v = randn_bf16((num_pages, page_size, 8, 128), gen)
    return DecodeInputs(name=name, q=q, k_pages=k, v_pages=v, block_table=bt,
                        seq_lens=torch.tensor(seq_lens, dtype=torch.int32),
                        page_size=page_size, scale=fp32_scale(128), meta={"seed": seed})


def paged_decode() -> DecodeInputs:
    gen = torch.Generator().manual_seed(1004)
    lens = uniform_lengths(64, 1024, 32768, gen)
    return _decode_from_lengths("paged_decode", lens, 16, 1004, gen)


def long_decode() -> DecodeInputs:
    gen = torch.Generator().manual_seed(1005)
    return _decode_from_lengths("long_decode", [131072, 131072], 64, 1005, gen)
