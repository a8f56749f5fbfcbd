// append_rope.cuh -- the step before a decode that appends the new token:
// rotate q and k_new by RoPE at the token's position, write k and v into the
// paged cache, and publish the new context lengths ("flash-attention" skill
// page, section 3.5: flash_attn_with_kvcache with k_new, v_new,
// cache_seqlens, block_table, rotary_cos, rotary_sin, rotary_interleaved).
//
// Request b's new token sits at position pos = cache_seqlens[b].  Pair i of
// a rotated vector is (x_i, x_{i + rd/2}), or (x_{2i}, x_{2i+1}) when
// interleaved; it turns by the angle whose cosine and sine are
// cos[pos][i] and sin[pos][i] (fp32 tables of rd/2 columns).  Dimensions
// past rd are copied.  The rotation is evaluated in fp64 and rounded once to
// bf16 (nearest, ties to even): the cache and the tensor-core decode hold
// bf16, and one rounding of a nearly exact value is the plainest reading of
// "the rotated key stored in the cache".
//
// One CTA per request; the work is (Hq + 2 Hkv) * d elements per request,
// negligible next to the decode's reads of the cache.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace fa {
namespace append {

constexpr int THREADS = 256;

struct Params {
  const __nv_bfloat16* q;      // [B, Hq, d]
  const __nv_bfloat16* k_new;  // [B, Hkv, d]
  const __nv_bfloat16* v_new;  // [B, Hkv, d]
  __nv_bfloat16* k_pages;      // [num_pages, page_size, Hkv, d]
  __nv_bfloat16* v_pages;
  const int32_t* block_table;  // [B, max_blocks]
  const int32_t* cache_seqlens;
  const float* cos;            // [max_pos, rd/2] or null (no rotation)
  const float* sin;
  __nv_bfloat16* q_rot;        // [B, Hq, d] out
  int32_t* seq_lens_new;       // [B] out: cache_seqlens + 1 (0 for a rejected request)
  int B, Hq, Hkv, d, page_size, max_blocks, num_pages, max_pos, rd, interleaved;
};

// Element e of the rotated vector x (d values): the pair partner and which
// side of the pair e is determine the formula.
__device__ __forceinline__ double rotated(const __nv_bfloat16* x, int e, const Params& p,
                                          const float* cos_row, const float* sin_row) {
  const double xe = (double)__bfloat162float(x[e]);
  if (!cos_row || e >= p.rd) return xe;
  const int half = p.rd / 2;
  int i, partner;
  bool first;
  if (p.interleaved) {
    i = e >> 1;
    first = (e & 1) == 0;
    partner = e ^ 1;
  } else {
    first = e < half;
    i = first ? e : e - half;
    partner = first ? e + half : e - half;
  }
  const double xp = (double)__bfloat162float(x[partner]);
  const double c = (double)__ldg(cos_row + i), s = (double)__ldg(sin_row + i);
  // first:  x_a c - x_b s      second: x_a s + x_b c   (a = first, b = second)
  return first ? xe * c - xp * s : xp * s + xe * c;
}

__global__ void __launch_bounds__(THREADS) append_rope_kernel(const Params p) {
  const int b = blockIdx.x;
  const int pos = __ldg(p.cache_seqlens + b);
  // the token must fit the block table (and the rotary table, if any)
  bool ok = pos >= 0 && (long long)pos < (long long)p.max_blocks * p.page_size &&
            (!p.cos || pos < p.max_pos);
  int page = -1;
  if (ok) {
    page = __ldg(p.block_table + (size_t)b * p.max_blocks + pos / p.page_size);
    ok = page >= 0 && page < p.num_pages;
  }
  if (!ok) {
    // a rejected request is treated as empty: O = 0, LSE = -inf
    if (threadIdx.x == 0) {
      report_error(kDevErrBounds);
      p.seq_lens_new[b] = 0;
    }
    return;
  }
  const float* cos_row = p.cos ? p.cos + (size_t)pos * (p.rd / 2) : nullptr;
  const float* sin_row = p.cos ? p.sin + (size_t)pos * (p.rd / 2) : nullptr;
  const int slot = pos % p.page_size;
  const int d = p.d;
  // rotated queries
  for (int idx = threadIdx.x; idx < p.Hq * d; idx += THREADS) {
    const int h = idx / d, e = idx - h * d;
    const size_t row = ((size_t)b * p.Hq + h) * d;
    p.q_rot[row + e] = __double2bfloat16(rotated(p.q + row, e, p, cos_row, sin_row));
  }
  // rotated key and plain value into the page slot
  for (int idx = threadIdx.x; idx < p.Hkv * d; idx += THREADS) {
    const int kh = idx / d, e = idx - kh * d;
    const size_t src = ((size_t)b * p.Hkv + kh) * d;
    const size_t dst = (((size_t)page * p.page_size + slot) * p.Hkv + kh) * d;
    p.k_pages[dst + e] = __double2bfloat16(rotated(p.k_new + src, e, p, cos_row, sin_row));
    p.v_pages[dst + e] = p.v_new[src + e];
  }
  if (threadIdx.x == 0) p.seq_lens_new[b] = pos + 1;
}

}  // namespace append
}  // namespace fa
