// decode_sm100.cuh -- split-KV decode over a paged KV cache, and the
// log-sum-exp combine of the splits.
//
// Method (pages: "flash-attention" skill page, PagedAttention appendix: the
// cache is [num_blocks, block_size, kv_heads, head_dim] addressed through
// block_table[batch, max_blocks] and cache_seqlens; FlashDecoding / Split-KV
// appendix: besides batch and heads, the KV length is split so several
// thread blocks take different KV ranges of one head, followed by a final
// reduce; GQA/MQA appendix: many query heads share one kv head; "gsyq.cn FA
// vs FIA" section 2: the decode kernel walks the whole KV cache block by
// block and lets the online softmax do the reduction, on non-contiguous
// pages without copying them into a contiguous tensor):
//
//   Plan: each request's context is cut into page ranges; the exclusive
//   prefix sums of the per-request range counts (from the device-side
//   seq_lens) turn the ranges of all requests into one flat list of work
//   items (the pages' Plan-Run split of scheduling and execution, "gsyq.cn
//   FA vs FIA" section 2).  Every CTA of the split kernel builds the prefix
//   itself in shared memory (up to PLAN_MAX_B requests); larger batches get
//   it from a one-CTA plan kernel.
//
//   D1 (split kernel): persistent, one CTA per SM; CTA c takes items c,
//   c + #CTAs, ... of the flat list.  An item is (request, page range, group
//   of hpb kv heads, chunk of query heads).  A producer warp gathers the
//   range's pages 16 tokens at a time into a shared-memory ring: with TMA
//   (3-D tensor maps over the pool, 128-byte swizzle, one 16-token box of
//   all the CTA's kv heads per 64-wide half of head_dim) when page_size is a
//   multiple of 16, and otherwise token by token with 16-byte cp.async
//   copies into the same swizzled layout (a stage may then span pages).
//   Each consumer warp owns one kv head and one tile of 8 of the query heads
//   that read it; all the warps of a kv head read the same shared-memory
//   stage, so every K/V byte is read from HBM once for the whole group (a
//   group of more than 64 query heads, 8 tiles, is split into chunks that
//   each read it once).  Scores and the P V product use warp-level bf16
//   tensor-core MMAs (S^T = K Q^T with tokens as rows, O^T += V^T P^T); the
//   online softmax keeps a running max and sum per query head.  A range
//   writes its normalised partial O and its LSE (fp32) to the workspace, or,
//   when it is its request's only range, the final bf16 O and LSE directly.
//   In the automatic mode every range spans the same number of pages, so
//   the flat list is made of near-equal items and the CTAs finish together.
//
//   D2 (combine): per (request, query head), LSE = log sum_s exp(lse_s) and
//   O = sum_s exp(lse_s - LSE) O_s over the request's ranges.  It is
//   launched as a programmatic dependent of D1: its CTAs are scheduled while
//   D1 drains and wait (griddepcontrol.wait) until D1 has completed.
#pragma once

#include "ptx.cuh"

namespace fa {
namespace decode {

constexpr int TOK = 16;           // tokens per pipeline stage (one MMA row block)
constexpr int QTILE = 8;          // query heads per consumer warp (MMA N = 8)
constexpr int MAX_CONSUMERS = 8;  // consumer warps per CTA (kv heads x query tiles)
constexpr int MAX_HPB = 8;        // kv heads per CTA
constexpr int MAX_STAGES = 12;
constexpr int STAGE_BUDGET = 192 * 1024;  // shared memory of the stage ring
constexpr int PLAN_MAX_B = 2048;          // largest batch whose plan a CTA builds itself
constexpr int SMEM_LIMIT = 232448;        // dynamic shared memory per CTA on sm_100

struct Params {
  const __nv_bfloat16* q;        // [B, Hq, D]
  const __nv_bfloat16* k_pages;  // [num_pages, page_size, Hkv, D] (cp.async gather)
  const __nv_bfloat16* v_pages;
  const int32_t* block_table;    // [B, max_blocks]
  const int32_t* seq_lens;       // [B]
  const int32_t* split_prefix;   // [B+1] prefix from the plan kernel, or null
  float* o_part;                 // [B, Hq, s_max, D]   partial outputs (normalised)
  float* lse_part;               // [B, Hq, s_max]      partial LSEs
  __nv_bfloat16* o;              // [B, Hq, D]
  float* lse;                    // [B, Hq] or null
  int B, Hq, Hkv, group;
  int hpb;      // kv heads per CTA
  int qpw;      // query tiles of 8 heads per kv head in a CTA (consumers = hpb * qpw)
  int nq;       // chunks of qpw query tiles per kv head (items per range and kv-head group)
  int ngroups;  // Hkv / hpb
  int page_size, max_blocks, num_pages;
  int s_max;        // partial slots per (request, head); 1 = no split, no plan
  int chunk_pages;  // > 0: every range spans chunk_pages pages; 0: s_max near-equal ranges per request
  int half_bytes;   // bytes of the K (or V) part of one stage
  int stages;       // ring length (<= MAX_STAGES)
  int tma_gather;   // 1: TMA boxes (page_size % 16 == 0); 0: per-token cp.async copies
  int local_plan;   // 1: each CTA builds the range prefix in shared memory
  float scale_log2;
};

// Shared memory of the split kernel after the ring: full and empty
// barriers, the abort flag (16 bytes), the scan scratch of the plan (one int
// per warp, 64 bytes), then the local plan (B + 1 ints).
constexpr int RING_TAIL_BYTES = 2 * MAX_STAGES * 8 + 16 + 64;

// Shared-memory bytes of the split kernel for these parameters, 1024-byte
// alignment slack included.
__host__ __device__ inline int split_smem_bytes(const Params& p) {
  return p.stages * 2 * p.half_bytes + RING_TAIL_BYTES + (p.local_plan ? (p.B + 1) * 4 : 0) + 1024;
}

template <int D>
struct Cfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static constexpr int PANELS = D / 64;
  static constexpr int KS = D / 16;  // MMA k-steps over head_dim / m-tiles over head_dim
};

// The pool is seen by TMA as a 3-D tensor with dimensions ordered (head_dim,
// token, kv head) -- strides 2*Hkv*D and 2*D bytes -- so one box {64 dims,
// 16 tokens, hpb heads} lands in shared memory as [kv head][token][128 B].
// Layout of the K (or V) half of a stage: [panel][kv head][token][128 B];
// each panel's box starts on a 1024-byte boundary and the 128-byte swizzle
// XORs the 16-byte chunk index with (token & 7), so the eight token rows an
// ldmatrix reads for one head fall in different banks.  Two boxes per
// stage for K and two for V (d = 128): few, large TMA operations -- with a
// box per head the gather ran at ~70% of HBM bandwidth, with one box for all
// heads at ~98%.
constexpr int BOX_BYTES = TOK * 128;  // one head's 16 token rows of one panel

__host__ __device__ inline int stage_bytes(int half_bytes) { return 2 * half_bytes; }

__device__ __forceinline__ uint32_t kv_off(int hpb, int panel, int hh, int tok, int ch) {
  return (uint32_t)((panel * hpb + hh) * BOX_BYTES + tok * 128 + ((ch ^ (tok & 7)) << 4));
}

// Context length of request b as the kernels use it (out-of-range values are
// a bounds error and are clamped), and its page count.
__device__ __forceinline__ int request_pages(const Params& p, int b, int& seq, bool report) {
  seq = __ldg(p.seq_lens + b);
  const int cap = p.max_blocks * p.page_size;
  if (seq < 0 || seq > cap) {
    if (report) report_error(kDevErrBounds);
    seq = seq < 0 ? 0 : cap;
  }
  return (seq + p.page_size - 1) / p.page_size;
}

// Pages per range and number of non-empty ranges of a request.
__device__ __forceinline__ int range_pages(const Params& p, int npages) {
  return p.chunk_pages > 0 ? p.chunk_pages : (npages + p.s_max - 1) / p.s_max;
}
__device__ __forceinline__ int num_ranges(const Params& p, int npages) {
  if (npages <= 0) return 0;
  const int c = range_pages(p, npages);
  return (npages + c - 1) / c;
}

// Plan: exclusive prefix sums of the per-request range counts (one CTA of
// 1024 threads, requests in chunks of 1024).
__global__ void __launch_bounds__(1024) plan_kernel(const Params p, int32_t* __restrict__ prefix) {
  __shared__ int warp_sums[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < p.B; base += 1024) {
    const int b = base + tid;
    int n = 0;
    if (b < p.B) {
      int seq;
      n = num_ranges(p, request_pages(p, b, seq, true));
    }
    int x = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_sums[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += y;
      }
      warp_sums[lane] = w;
    }
    __syncthreads();
    const int incl = carry + x + (warp > 0 ? warp_sums[warp - 1] : 0);
    if (b < p.B) prefix[b] = incl - n;
    __syncthreads();
    if (tid == 1023) carry = incl;
    __syncthreads();
  }
  if (tid == 0) prefix[p.B] = carry;
}

// Exclusive prefix sums of the per-request range counts into prefix[0..B]
// (shared memory), by the whole CTA in chunks of blockDim.x requests.
// `scratch` holds one int per warp.  Bad lengths are reported here.
__device__ void build_plan(const Params& p, int* prefix, int* scratch) {
  const int nthr = blockDim.x, tid = threadIdx.x, lane = lane_id(), warp = warp_id();
  const int nwarps = nthr >> 5;
  int carry = 0;
  for (int base = 0; base < p.B; base += nthr) {
    const int b = base + tid;
    int n = 0;
    if (b < p.B) {
      int seq;
      n = num_ranges(p, request_pages(p, b, seq, true));
    }
    int x = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < nwarps; ++w) {
      const int v = scratch[w];
      before += w < warp ? v : 0;
      total += v;
    }
    if (b < p.B) prefix[b] = carry + before + x - n;
    carry += total;
    __syncthreads();
  }
  if (tid == 0) prefix[p.B] = carry;
  __syncthreads();
}

// Work item i -> (request b, range s, kv-head group g, query chunk qc);
// items are the non-empty ranges of every request (all requests, one range
// each, without a plan), kv-head groups and query chunks fastest.
__device__ __forceinline__ void item_of(const Params& p, const int32_t* prefix, int i, int& b,
                                        int& s, int& g, int& qc) {
  const int per = p.ngroups * p.nq;
  const int y = i % per;
  g = y / p.nq;
  qc = y - g * p.nq;
  const int bs = i / per;
  if (!prefix) {
    b = bs;
    s = 0;
    return;
  }
  int lo = 0, hi = p.B - 1;  // last b with prefix[b] <= bs
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= bs) lo = mid; else hi = mid - 1;
  }
  b = lo;
  s = bs - prefix[lo];
}

// Token range [tok_begin, tok_end) of range s of request b.
__device__ __forceinline__ void item_tokens(const Params& p, bool planned, int b, int s,
                                            int& tok_begin, int& tok_end, int& nranges) {
  int seq;
  // with a plan, bad lengths were reported while building it; otherwise here
  const int npages = request_pages(p, b, seq, !planned);
  if (!planned) {
    tok_begin = 0;
    tok_end = seq;
    nranges = 1;
    return;
  }
  const int c = range_pages(p, npages);
  const int pg0 = min(npages, s * c), pg1 = min(npages, pg0 + c);
  tok_begin = pg0 * p.page_size;
  tok_end = min(seq, pg1 * p.page_size);
  nranges = num_ranges(p, npages);
}

// 16-byte global -> shared copy; src_bytes = 0 fills the 16 bytes with zeros
// and reads nothing.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
// Arrives on the mbarrier once every cp.async this thread issued so far has
// completed (the arrival counts against the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Persistent: CTA c takes items c, c + gridDim.x, ...; the ring runs on
// across item boundaries.
template <int D>
__global__ void __launch_bounds__((MAX_CONSUMERS + 1) * 32, 1)
    split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int sbytes = stage_bytes(p.half_bytes);
  const int nstages = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + nstages * sbytes);
  uint64_t* empty = full + MAX_STAGES;
  int* abort_flag = reinterpret_cast<int*>(empty + MAX_STAGES);
  uint64_t* stall_bar = reinterpret_cast<uint64_t*>(abort_flag + 2);  // timeout test hook
  int* scan_scratch = abort_flag + 4;  // one int per warp, only while the plan is built
  int32_t* local_prefix = abort_flag + 4 + 16;
  volatile int* abort = abort_flag;

  const int warp = warp_id(), lane = lane_id();
  const int nconsumers = p.hpb * p.qpw;

  // the combine kernel (a programmatic dependent) may be scheduled now; it
  // waits for this grid to complete before it reads anything
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (threadIdx.x == 0) {
    for (int s = 0; s < nstages; ++s) {
      // TMA: one arrive.expect_tx per stage; cp.async: one arrival per producer lane
      mbar_init(&full[s], p.tma_gather ? 1 : 32);
      mbar_init(&empty[s], nconsumers);
    }
    *abort_flag = 0;
    mbar_init(stall_bar, 1);  // never arrived at
    fence_mbar_init();
  }
  const int32_t* prefix = nullptr;
  if (p.s_max > 1) {
    if (p.local_plan) {
      build_plan(p, local_prefix, scan_scratch);
      prefix = local_prefix;
    } else {
      prefix = p.split_prefix;
    }
  }
  __syncthreads();
  const bool planned = prefix != nullptr;
  const int total = (planned ? prefix[p.B] : p.B) * p.ngroups * p.nq;

  if (warp == nconsumers) {
    // ======================= producer (converged warp) =======================
    // The whole warp runs the loop: the block-table entries of 32 stages are
    // fetched at once, one per lane, and broadcast by shuffle (TMA gather), or
    // each of 16 lanes looks up its token's page (cp.async gather), so no
    // stage waits on a dependent global load; TMA copies are issued by one
    // elected lane, cp.async copies by all lanes.
    if (lane == 0 && p.tma_gather) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    __syncwarp();
    int g = 0;  // stages issued so far (ring position)
    bool ok = true;
    for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
      int b, s, grp, qc, tb, te, nr;
      item_of(p, prefix, i, b, s, grp, qc);
      item_tokens(p, planned, b, s, tb, te, nr);
      const int kvh0 = grp * p.hpb;
      const int32_t* bt = p.block_table + (size_t)b * p.max_blocks;
      const int nst = te > tb ? (te - tb + TOK - 1) / TOK : 0;
      int page_of_lane = 0;
      for (int st = 0; st < nst; ++st, ++g) {
        const int slot = g % nstages;
        const int t0 = tb + st * TOK;
        uint8_t* kdst = smem + slot * sbytes;
        uint8_t* vdst = kdst + p.half_bytes;
        if (p.tma_gather) {
          if ((st & 31) == 0) {
            const int sl = st + lane;  // the stage whose page this lane looks up
            page_of_lane = sl < nst ? __ldg(bt + (tb + sl * TOK) / p.page_size) : 0;
          }
          const int page = __shfl_sync(0xffffffffu, page_of_lane, st & 31);
          if (!mbar_wait(&empty[slot], ((g / nstages) & 1) ^ 1, abort)) { ok = false; break; }
          // page_size is a multiple of TOK, so a stage never crosses a page
          int z;
          if (page < 0 || page >= p.num_pages) {
            if (lane == 0) report_error(kDevErrBounds);
            z = -TOK;  // whole box outside the pool: TMA fills zeros
          } else {
            z = page * p.page_size + (t0 % p.page_size);
          }
          expect_tx_el(&full[slot], 2 * p.half_bytes);
          // one box per 64-wide half of head_dim holds all the CTA's kv heads
          for (int pn = 0; pn < C::PANELS; ++pn) {
            const int off = pn * p.hpb * BOX_BYTES;
            tma_load_3d_el(kdst + off, &tmK, &full[slot], pn * 64, z, kvh0);
            tma_load_3d_el(vdst + off, &tmV, &full[slot], pn * 64, z, kvh0);
          }
        } else {
          // token `lane` (< 16) of this stage: its page, or -1 (past the
          // range, or a bad entry: its rows are filled with zeros)
          const int valid = min(TOK, te - t0);
          int pg = -1;
          if (lane < valid) {
            pg = __ldg(bt + (t0 + lane) / p.page_size);
            if (pg < 0 || pg >= p.num_pages) {
              report_error(kDevErrBounds);
              pg = -1;
            }
          }
          if (!mbar_wait(&empty[slot], ((g / nstages) & 1) ^ 1, abort)) { ok = false; break; }
          // 16-byte chunks of the stage's (token, kv head) rows, consecutive
          // lanes on consecutive chunks of a row: a row of one token's kv
          // heads is contiguous in the pool
          constexpr int CPR = D / 8;  // chunks per row
          const uint32_t kbase = smem_u32(kdst), vbase = smem_u32(vdst);
          for (int q = lane; q < TOK * p.hpb * CPR; q += 32) {
            const int row = q / CPR, c16 = q - row * CPR;
            const int tok = row / p.hpb, hh = row - tok * p.hpb;
            const int page = __shfl_sync(0xffffffffu, pg, tok);
            const uint32_t dst = kv_off(p.hpb, c16 >> 3, hh, tok, c16 & 7);
            size_t src = 0;
            uint32_t bytes = 0;
            if (page >= 0) {
              const int pos = page * p.page_size + (t0 + tok) % p.page_size;
              src = ((size_t)pos * p.Hkv + kvh0 + hh) * D + c16 * 8;
              bytes = 16;
            }
            cp_async_16(kbase + dst, p.k_pages + src, bytes);
            cp_async_16(vbase + dst, p.v_pages + src, bytes);
          }
          cp_async_arrive_noinc(&full[slot]);
        }
      }
    }
    // every load issued must land before the CTA exits
    for (int s = 0; s < nstages && s < g; ++s) {
      const int last = g - 1 - ((g - 1 - s) % nstages);
      mbar_wait_bounded(&full[last % nstages], (last / nstages) & 1);
    }
  } else if (warp < nconsumers) {
    // ============ consumers: one warp per (kv head, tile of 8 query heads) ============
    const int hh = warp / p.qpw;   // kv head of the CTA's group
    const int qtw = warp % p.qpw;  // query tile within the chunk
    const int g8 = lane >> 2, tq = lane & 3;
    const float sl = p.scale_log2;
    const uint32_t sbase = smem_u32(smem);
    const int lm = lane >> 3, lr = lane & 7;  // ldmatrix row/chunk assignment of this lane
    int g = 0;  // stages consumed so far (ring position)
    bool ok = true;
    // timeout test hook: this warp's first stage wait is on a barrier that
    // nothing arrives at
    bool stall = warp == 0 && blockIdx.x == 0 &&
                 *reinterpret_cast<volatile int*>(&g_stall_test) == kStallDecode;
    for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
      int b, s, grp, qc, tb, te, nr;
      item_of(p, prefix, i, b, s, grp, qc);
      item_tokens(p, planned, b, s, tb, te, nr);
      const int kvh = grp * p.hpb + hh;
      const int qt = qc * p.qpw + qtw;  // query tile: heads qt*8 .. qt*8+7 of the kv head's group
      const int nst = te > tb ? (te - tb + TOK - 1) / TOK : 0;
      // Q^T fragments (MMA B operand, k = head_dim, n = query head of the tile)
      uint32_t qb0[C::KS], qb1[C::KS];
      {
        const bool real = qt * QTILE + g8 < p.group;
        const __nv_bfloat16* qrow =
            p.q + ((size_t)b * p.Hq + (size_t)kvh * p.group + qt * QTILE + (real ? g8 : 0)) * D;
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
      // query heads 2tq, 2tq+1 of the tile: running max, exact sum of exp (for
      // the LSE) and sum of the bf16-rounded weights the PV MMA uses
      // (normalises O)
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f, r0 = 0.f, r1 = 0.f;
      for (int st = 0; st < nst; ++st, ++g) {
        const int slot = g % nstages;
        if (!mbar_wait(stall ? stall_bar : &full[slot], (g / nstages) & 1, abort)) {
          ok = false;
          break;
        }
        stall = false;
        const uint32_t kb = sbase + slot * sbytes;
        const uint32_t vb = kb + p.half_bytes;
        const int valid = min(TOK, te - (tb + st * TOK));
        if (valid < TOK && p.tma_gather) {
          // V rows past the context are not part of the sum; their P is zero,
          // but 0 * (garbage) may be NaN, so clear them for this warp's head
          // (every warp of the head writes the same zeros before its reads;
          // the cp.async gather already filled them with zeros).
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
        // rows: token g8 (c0, c1) and g8 + 8 (c2, c3); columns: query heads 2tq, 2tq+1
        float s00 = c[0] * sl, s01 = c[1] * sl, s10 = c[2] * sl, s11 = c[3] * sl;
        if (g8 >= valid) s00 = s01 = -INFINITY;
        if (g8 + 8 >= valid) s10 = s11 = -INFINITY;
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
        if (valid < TOK && p.tma_gather) fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
      }
      if (!ok) break;
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
      // heads of the tile held by this lane, as indices in the kv head's group
      const int n0 = qt * QTILE + 2 * tq, n1 = n0 + 1;
      const size_t head0 = (size_t)b * p.Hq + (size_t)kvh * p.group;
      if (nr > 1) {
        const int S = p.s_max;
#pragma unroll
        for (int mt = 0; mt < C::KS; ++mt) {
          const int d = mt * 16 + g8;
          if (n0 < p.group) {
            float* dst = p.o_part + ((head0 + n0) * S + s) * D;
            dst[d] = acc[mt][0] * inv0;
            dst[d + 8] = acc[mt][2] * inv0;
          }
          if (n1 < p.group) {
            float* dst = p.o_part + ((head0 + n1) * S + s) * D;
            dst[d] = acc[mt][1] * inv1;
            dst[d + 8] = acc[mt][3] * inv1;
          }
        }
        if (g8 == 0) {
          if (n0 < p.group) p.lse_part[(head0 + n0) * S + s] = lse0;
          if (n1 < p.group) p.lse_part[(head0 + n1) * S + s] = lse1;
        }
      } else {
        // the request's only range (or an empty request with no plan): final output
#pragma unroll
        for (int mt = 0; mt < C::KS; ++mt) {
          const int d = mt * 16 + g8;
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
        if (g8 == 0 && p.lse) {
          if (n0 < p.group) p.lse[head0 + n0] = lse0;
          if (n1 < p.group) p.lse[head0 + n1] = lse1;
        }
      }
    }
  }
  __syncthreads();
}

// One CTA of 8 warps per (request, query head): merges the request's ranges.
// All threads find the max and the sum of exp over the range LSEs; warp w
// then accumulates ranges w, w+8, ... (four loads in flight per lane) and the
// eight partial vectors are added in shared memory.  A request with one range
// was written by the split kernel already; one with none (empty context)
// gets O = 0 and LSE = -inf.
constexpr int COMBINE_WARPS = 8;

template <int D>
__global__ void __launch_bounds__(COMBINE_WARPS * 32) combine_kernel(const Params p) {
  constexpr int PER = D / 32;  // output elements per lane
  __shared__ float red[COMBINE_WARPS][D];
  __shared__ float wred[COMBINE_WARPS];
  // launched as a programmatic dependent of the split kernel: wait until it
  // has completed and its partial results are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float* __restrict__ o_part = p.o_part;
  const float* __restrict__ lse_part = p.lse_part;
  __nv_bfloat16* __restrict__ o = p.o;
  float* __restrict__ lse = p.lse;
  const int Hq = p.Hq, S = p.s_max;
  const int r = blockIdx.x;
  const int b = r / Hq;
  const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
  int seq;
  const int n = num_ranges(p, request_pages(p, b, seq, false));
  if (n == 1) return;
  const float* lp = lse_part + (size_t)r * S;
  const float log2e = 1.4426950408889634f;
  // max of the range LSEs
  float mx = -INFINITY;
  for (int s = tid; s < n; s += COMBINE_WARPS * 32) mx = fmaxf(mx, lp[s]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) wred[warp] = mx;
  __syncthreads();
  mx = wred[0];
#pragma unroll
  for (int w = 1; w < COMBINE_WARPS; ++w) mx = fmaxf(mx, wred[w]);
  __syncthreads();
  float total_lse = -INFINITY;
  float out[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) out[i] = 0.f;
  if (mx != -INFINITY) {
    float sum = 0.f;
    for (int s = tid; s < n; s += COMBINE_WARPS * 32) sum += ex2((lp[s] - mx) * log2e);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane == 0) wred[warp] = sum;
    __syncthreads();
    sum = 0.f;
#pragma unroll
    for (int w = 0; w < COMBINE_WARPS; ++w) sum += wred[w];
    total_lse = mx + __logf(sum);
    const float* op = o_part + (size_t)r * S * D + lane * PER;
    int s = warp;
    for (; s + 3 * COMBINE_WARPS < n; s += 4 * COMBINE_WARPS) {
      float v[4][PER], w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int su = s + u * COMBINE_WARPS;
        w[u] = ex2((lp[su] - total_lse) * log2e);
#pragma unroll
        for (int i = 0; i < PER; ++i) v[u][i] = op[(size_t)su * D + i];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int i = 0; i < PER; ++i) out[i] = fmaf(w[u], v[u][i], out[i]);
    }
    for (; s < n; s += COMBINE_WARPS) {
      const float w = ex2((lp[s] - total_lse) * log2e);
#pragma unroll
      for (int i = 0; i < PER; ++i) out[i] = fmaf(w, op[(size_t)s * D + i], out[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) red[warp][lane * PER + i] = out[i];
  __syncthreads();
  if (warp == 0) {
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      acc[i] = 0.f;
#pragma unroll
      for (int w = 0; w < COMBINE_WARPS; ++w) acc[i] += red[w][lane * PER + i];
    }
    __nv_bfloat16* dst = o + (size_t)r * D + lane * PER;
#pragma unroll
    for (int i = 0; i < PER; i += 2)
      *reinterpret_cast<uint32_t*>(dst + i) = pack_bf16x2(acc[i], acc[i + 1]);
    if (lse && lane == 0) lse[r] = total_lse;
  }
}

}  // namespace decode
}  // namespace fa
