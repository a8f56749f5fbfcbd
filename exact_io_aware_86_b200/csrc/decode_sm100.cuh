// decode_sm100.cuh -- split-KV decode over a paged KV cache, and the
// log-sum-exp combine of the splits.
//
// Method (pages: "flash-attention" skill page, PagedAttention appendix: the
// cache is [num_blocks, block_size, kv_heads, head_dim] addressed through
// block_table[batch, max_blocks] and cache_seqlens; FlashDecoding / Split-KV
// appendix: besides batch and heads, the KV length is split so several
// thread blocks take different KV ranges of one head, followed by a final
// reduce; "gsyq.cn FA vs FIA" section 2: the decode kernel walks the whole
// KV cache block by block and lets the online softmax do the reduction, on
// non-contiguous pages without copying them into a contiguous tensor):
//
//   D1 (split kernel): one CTA per (split, group of up to 8 kv heads,
//   request).  A producer warp gathers the split's pages 16 tokens at a time
//   into a shared-memory ring with TMA (3-D tensor maps over the pool with
//   128-byte swizzle, one 16-token box per kv head and 64-wide half of
//   head_dim; page_size is a multiple of 16).  Each consumer warp owns one kv head and the Hq/Hkv <= 8 query
//   heads that read it, so every K/V byte is read from HBM once for the whole
//   group.  Scores and the P V product use warp-level bf16 tensor-core MMAs
//   (S^T = K Q^T with tokens as rows, O^T += V^T P^T); the online softmax
//   keeps a running max and sum per query head.  The split writes its
//   normalised partial O and its LSE (fp32) to the workspace, or, with one
//   split, the final bf16 O and LSE directly.
//
//   D2 (combine): per (request, query head), LSE = log sum_s exp(lse_s) and
//   O = sum_s exp(lse_s - LSE) O_s; splits with no tokens have lse = -inf and
//   weigh zero.
#pragma once

#include "ptx.cuh"

namespace fa {
namespace decode {

constexpr int TOK = 16;      // tokens per pipeline stage (one MMA row block)
constexpr int MAX_HPB = 8;   // kv heads per CTA
constexpr int STAGES = 3;
constexpr int MAX_GROUP = 8; // query heads per kv head (MMA N = 8)

struct Params {
  const __nv_bfloat16* q;     // [B, Hq, D]
  const int32_t* block_table; // [B, max_blocks]
  const int32_t* seq_lens;    // [B]
  float* o_part;              // [B, Hq, S, D]  (num_splits > 1)
  float* lse_part;            // [B, Hq, S]
  __nv_bfloat16* o;           // [B, Hq, D]     (num_splits == 1)
  float* lse;                 // [B, Hq] or null
  int B, Hq, Hkv, group, hpb;
  int page_size, max_blocks, num_pages, num_splits;
  int half_bytes;             // bytes of the K (or V) part of one stage
  float scale_log2;
};

template <int D>
struct Cfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static constexpr int PANELS = D / 64;
  static constexpr int KS = D / 16;  // MMA k-steps over head_dim / m-tiles over head_dim
};

// One TMA box = 16 tokens x 64 head_dim elements of one kv head (2 KB), 128 B
// per row.  Shared-memory layout of the K (or V) half of a stage:
// [panel][kv head][token][128 B]; every box starts on a 1024-byte boundary
// and the TMA 128-byte swizzle XORs the 16-byte chunk index with (token & 7).
constexpr int BOX_BYTES = TOK * 128;

__host__ __device__ inline int stage_bytes(int half_bytes) { return 2 * half_bytes; }

__device__ __forceinline__ uint32_t kv_off(int hpb, int panel, int hh, int tok, int ch) {
  return (uint32_t)((panel * hpb + hh) * BOX_BYTES + tok * 128 + ((ch ^ (tok & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__((MAX_HPB + 1) * 32)
    split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int sbytes = stage_bytes(p.half_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * sbytes);
  uint64_t* empty = full + STAGES;
  int* abort_flag = reinterpret_cast<int*>(empty + STAGES);
  volatile int* abort = abort_flag;

  const int split = blockIdx.x;
  const int kvh0 = blockIdx.y * p.hpb;
  const int b = blockIdx.z;
  const int warp = warp_id(), lane = lane_id();
  const int nconsumers = p.hpb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], nconsumers);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // The split's token range: pages [p0, p1) of this request.
  int seq = __ldg(p.seq_lens + b);
  if (seq < 0 || seq > p.max_blocks * p.page_size) {
    if (threadIdx.x == 0) report_error(kDevErrBounds);
    seq = seq < 0 ? 0 : p.max_blocks * p.page_size;
  }
  const int npages = (seq + p.page_size - 1) / p.page_size;
  const int chunk = (npages + p.num_splits - 1) / p.num_splits;
  const int pg0 = min(npages, split * chunk);
  const int pg1 = min(npages, pg0 + chunk);
  const int tok_begin = pg0 * p.page_size;
  const int tok_end = min(seq, pg1 * p.page_size);
  const int nstages = tok_end > tok_begin ? (tok_end - tok_begin + TOK - 1) / TOK : 0;

  if (warp == nconsumers) {
    // ======================= producer =======================
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int32_t* bt = p.block_table + (size_t)b * p.max_blocks;
      int st = 0;
      for (; st < nstages; ++st) {
        const int slot = st % STAGES;
        if (!mbar_wait(&empty[slot], ((st / STAGES) & 1) ^ 1, abort)) break;
        // page_size is a multiple of TOK, so a stage never crosses a page
        const int t0 = tok_begin + st * TOK;
        const int page = __ldg(bt + t0 / p.page_size);
        int z;
        if (page < 0 || page >= p.num_pages) {
          report_error(kDevErrBounds);
          z = -TOK;  // whole box outside the pool: TMA fills zeros
        } else {
          z = page * p.page_size + (t0 % p.page_size);
        }
        mbar_arrive_expect_tx(&full[slot], 2 * p.half_bytes);
        uint8_t* kdst = smem + slot * sbytes;
        uint8_t* vdst = kdst + p.half_bytes;
        for (int pn = 0; pn < C::PANELS; ++pn)
          for (int hh = 0; hh < p.hpb; ++hh) {
            const int off = (pn * p.hpb + hh) * BOX_BYTES;
            tma_load_3d(kdst + off, &tmK, &full[slot], pn * 64, kvh0 + hh, z);
            tma_load_3d(vdst + off, &tmV, &full[slot], pn * 64, kvh0 + hh, z);
          }
      }
      // every load issued must land before the CTA exits
      for (int s = 0; s < STAGES && s < st; ++s) {
        const int last = st - 1 - ((st - 1 - s) % STAGES);
        mbar_wait_bounded(&full[last % STAGES], (last / STAGES) & 1);
      }
    }
  } else {
    // ======================= consumers: one warp per kv head =======================
    const int hh = warp;
    const int kvh = kvh0 + hh;
    const int g = lane >> 2, tq = lane & 3;
    // Q^T fragments (MMA B operand, k = head_dim, n = query head of the group)
    uint32_t qb0[C::KS], qb1[C::KS];
    {
      const bool real = g < p.group;
      const __nv_bfloat16* qrow = p.q + ((size_t)b * p.Hq + (size_t)kvh * p.group + (real ? g : 0)) * D;
#pragma unroll
      for (int ks = 0; ks < C::KS; ++ks) {
        const uint32_t* w = reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * tq);
        qb0[ks] = real ? __ldg(w) : 0u;
        qb1[ks] = real ? __ldg(w + 4) : 0u;
      }
    }
    float acc[C::KS][4];
#pragma unroll
    for (int mt = 0; mt < C::KS; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    // query heads 2tq, 2tq+1: running max, exact sum of exp (for the LSE) and
    // sum of the bf16-rounded weights the PV MMA uses (normalises O)
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f, r0 = 0.f, r1 = 0.f;
    const float sl = p.scale_log2;
    const uint32_t sbase = smem_u32(smem);

    // ldmatrix row/chunk assignment of this lane
    const int lm = lane >> 3, lr = lane & 7;
    for (int st = 0; st < nstages; ++st) {
      const int slot = st % STAGES;
      if (!mbar_wait(&full[slot], (st / STAGES) & 1, abort)) break;
      const uint32_t kb = sbase + slot * sbytes;
      const uint32_t vb = kb + p.half_bytes;
      const int valid = min(TOK, tok_end - (tok_begin + st * TOK));
      if (valid < TOK) {
        // V rows past the context are not part of the sum; their P is zero,
        // but 0 * (garbage) may be NaN, so clear them for this warp's head.
        uint8_t* vgen = smem + slot * sbytes + p.half_bytes;
        for (int idx = lane; idx < (TOK - valid) * C::PANELS * 8; idx += 32) {
          const int tok = valid + idx / (C::PANELS * 8);
          const int rem = idx % (C::PANELS * 8);
          *reinterpret_cast<uint4*>(vgen + kv_off(p.hpb, rem / 8, hh, tok, rem % 8)) =
              make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
      }
      // ---- S^T[tok][n] = sum_d K[tok][d] Q[n][d] ----
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < C::KS; ++ks) {
        // matrices: 0 = tok 0-7 / d lo, 1 = tok 8-15 / d lo, 2 = tok 0-7 / d hi, 3 = tok 8-15 / d hi
        const int tok = lr + ((lm & 1) << 3);
        const int d0 = ks * 16 + ((lm >> 1) << 3);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(kb + kv_off(p.hpb, d0 >> 6, hh, tok, (d0 & 63) >> 3), a0, a1, a2, a3);
        mma_bf16_16816(c, a0, a1, a2, a3, qb0[ks], qb1[ks]);
      }
      // rows: token g (c0, c1) and g + 8 (c2, c3); columns: query heads 2tq, 2tq+1
      float s00 = c[0] * sl, s01 = c[1] * sl, s10 = c[2] * sl, s11 = c[3] * sl;
      if (g >= valid) s00 = s01 = -INFINITY;
      if (g + 8 >= valid) s10 = s11 = -INFINITY;
      float mx0 = fmaxf(s00, s10), mx1 = fmaxf(s01, s11);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);  // finite: valid >= 1
      const float al0 = ex2(m0 - mn0), al1 = ex2(m1 - mn1);    // ex2(-inf) = 0
      const float p00 = ex2(s00 - mn0), p01 = ex2(s01 - mn1);
      const float p10 = ex2(s10 - mn0), p11 = ex2(s11 - mn1);
      // P^T in bf16 (the MMA operand); the row sums use the same rounded values
      const uint32_t x0 = pack_bf16x2(p00, p01), x1 = pack_bf16x2(p10, p11);
      l0 = l0 * al0 + (p00 + p10);
      l1 = l1 * al1 + (p01 + p11);
      r0 = r0 * al0 + (__uint_as_float(x0 << 16) + __uint_as_float(x1 << 16));
      r1 = r1 * al1 + (__uint_as_float(x0 & 0xFFFF0000u) + __uint_as_float(x1 & 0xFFFF0000u));
      m0 = mn0;
      m1 = mn1;
#pragma unroll
      for (int mt = 0; mt < C::KS; ++mt) {
        acc[mt][0] *= al0;
        acc[mt][1] *= al1;
        acc[mt][2] *= al0;
        acc[mt][3] *= al1;
      }
      // P^T as the MMA B operand (k = token, n = query head)
      const uint32_t pb0 = movmatrix_trans(x0);
      const uint32_t pb1 = movmatrix_trans(x1);
      // ---- O^T[d][n] += sum_tok V[tok][d] P[n][tok] ----
#pragma unroll
      for (int mt = 0; mt < C::KS; ++mt) {
        // matrices: 0 = tok 0-7 / d lo, 1 = tok 0-7 / d hi, 2 = tok 8-15 / d lo, 3 = tok 8-15 / d hi
        const int tok = lr + ((lm >> 1) << 3);
        const int d0 = mt * 16 + ((lm & 1) << 3);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(vb + kv_off(p.hpb, d0 >> 6, hh, tok, (d0 & 63) >> 3), a0, a1, a2, a3);
        mma_bf16_16816(acc[mt], a0, a1, a2, a3, pb0, pb1);
      }
      if (valid < TOK) fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
    // ---- finish: row sums over the 8 token lanes, normalise, write ----
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
      r0 += __shfl_xor_sync(0xffffffffu, r0, off);
      r1 += __shfl_xor_sync(0xffffffffu, r1, off);
    }
    const float inv0 = r0 > 0.f ? 1.f / r0 : 0.f, inv1 = r1 > 0.f ? 1.f / r1 : 0.f;
    const float ln2 = 0.69314718055994531f;
    const float lse0 = l0 > 0.f ? (m0 + __log2f(l0)) * ln2 : -INFINITY;
    const float lse1 = l1 > 0.f ? (m1 + __log2f(l1)) * ln2 : -INFINITY;
    const int n0 = 2 * tq, n1 = 2 * tq + 1;
    const size_t head0 = (size_t)b * p.Hq + (size_t)kvh * p.group;
    if (p.num_splits > 1) {
      const int S = p.num_splits;
#pragma unroll
      for (int mt = 0; mt < C::KS; ++mt) {
        const int d = mt * 16 + g;
        if (n0 < p.group) {
          float* dst = p.o_part + ((head0 + n0) * S + split) * D;
          dst[d] = acc[mt][0] * inv0;
          dst[d + 8] = acc[mt][2] * inv0;
        }
        if (n1 < p.group) {
          float* dst = p.o_part + ((head0 + n1) * S + split) * D;
          dst[d] = acc[mt][1] * inv1;
          dst[d + 8] = acc[mt][3] * inv1;
        }
      }
      if (g == 0) {
        if (n0 < p.group) p.lse_part[(head0 + n0) * S + split] = lse0;
        if (n1 < p.group) p.lse_part[(head0 + n1) * S + split] = lse1;
      }
    } else {
#pragma unroll
      for (int mt = 0; mt < C::KS; ++mt) {
        const int d = mt * 16 + g;
        if (n0 < p.group) {
          __nv_bfloat16* dst = p.o + (head0 + n0) * D;
          dst[d] = __float2bfloat16_rn(acc[mt][0] * inv0);
          dst[d + 8] = __float2bfloat16_rn(acc[mt][2] * inv0);
        }
        if (n1 < p.group) {
          __nv_bfloat16* dst = p.o + (head0 + n1) * D;
          dst[d] = __float2bfloat16_rn(acc[mt][1] * inv1);
          dst[d + 8] = __float2bfloat16_rn(acc[mt][3] * inv1);
        }
      }
      if (g == 0 && p.lse) {
        if (n0 < p.group) p.lse[head0 + n0] = lse0;
        if (n1 < p.group) p.lse[head0 + n1] = lse1;
      }
    }
  }
  __syncthreads();
}

// One warp per (request, query head).
template <int D>
__global__ void __launch_bounds__(128)
    combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                   __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int rows, int S) {
  const int r = blockIdx.x * 4 + warp_id();
  const int lane = lane_id();
  if (r >= rows) return;
  const float* lp = lse_part + (size_t)r * S;
  const float log2e = 1.4426950408889634f;
  float mx = -INFINITY;
  for (int s = lane; s < S; s += 32) mx = fmaxf(mx, lp[s]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  constexpr int PER = D / 32;
  float out[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) out[i] = 0.f;
  float total_lse = -INFINITY;
  if (mx != -INFINITY) {
    float sum = 0.f;
    for (int s = lane; s < S; s += 32) sum += ex2((lp[s] - mx) * log2e);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    total_lse = mx + __logf(sum);
    const float* op = o_part + (size_t)r * S * D + lane * PER;
    for (int s = 0; s < S; ++s) {
      const float w = ex2((lp[s] - total_lse) * log2e);
      if (w == 0.f) continue;  // empty split (lse = -inf) or negligible
      if constexpr (PER == 4) {
        const float4 v = *reinterpret_cast<const float4*>(op + (size_t)s * D);
        out[0] += w * v.x;
        out[1] += w * v.y;
        out[2] += w * v.z;
        out[3] += w * v.w;
      } else {
        const float2 v = *reinterpret_cast<const float2*>(op + (size_t)s * D);
        out[0] += w * v.x;
        out[1] += w * v.y;
      }
    }
  }
  __nv_bfloat16* dst = o + (size_t)r * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; i += 2)
    *reinterpret_cast<uint32_t*>(dst + i) = pack_bf16x2(out[i], out[i + 1]);
  if (lse && lane == 0) lse[r] = total_lse;
}

}  // namespace decode
}  // namespace fa
