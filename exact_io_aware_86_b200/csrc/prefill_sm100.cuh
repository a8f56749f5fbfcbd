// prefill_sm100.cuh -- exact attention prefill on the 5th-generation tensor
// cores (tcgen05), packed variable-length sequences, causal or full mask,
// grouped kv heads.
//
// Method (pages: "gsyq.cn FA vs FIA" section 1, tiling + online softmax;
// "FlashAttention" concept page, Tiling: Q in B_r-row blocks, K/V in
// B_c-row blocks held on chip; cnblogs section 3.2 / 4.2: S and P never
// written to HBM, QK^T + mask + softmax + PV fused in one kernel):
//   for each 128-row query tile, stream 128-key K/V tiles; S = Q K_j^T on
//   the tensor cores into tensor memory; the softmax warps read S, keep the
//   running row max m and sum l, write P = exp(S*scale - m) back into tensor
//   memory as bf16, and the tensor cores accumulate O += P V_j in tensor
//   memory.  At the end O / l is stored as bf16 and LSE = ln2*(m + log2 l).
//   O leaves through a small shared-memory staging region per warp, read
//   back for coalesced 128-byte global stores (rows past a sequence end are
//   skipped).
//
// CTA layout (384 threads = 3 warpgroups, one CTA per SM, persistent):
//   warp 0      TMA producer of K_j, V_j, alternately through a ring of
//               128 x D smem slots
//   warp 1      MMA issuer (converged warp, elected lane) and TMEM owner
//               (512 columns)
//   warp 2      TMA producer of the Q tiles, once per work item, each query
//               tile on its own barrier pair, refilled as soon as it is free
//   warp 3      idle (it completes the first warpgroup)
//   warps 4-7   softmax for query tile 0 (rows q0 .. q0+127)
//   warps 8-11  softmax for query tile 1 (rows q0+128 .. q0+255)
// setmaxnreg moves registers from the first warpgroup to the softmax ones.
// The two query tiles share every K/V tile, and while one softmax group
// works on its S the tensor cores run the other tile's P V and Q K^T.
//
// Tensor memory columns: S0 [0,128), S1 [128,256), O0 [256,256+D),
// O1 [384,384+D).  P_t (bf16, 2 per column) overwrites the first 64 columns
// of S_t once S_t has been read; the MMA that writes the next S_t is issued
// after the P_t V MMAs, and tcgen05 MMAs from one thread execute in order.
// P is released in two 64-key halves, each on its own barrier, so the first
// half's P V MMAs run while the softmax still computes the second half.  At
// an item's last step the MMA warp issues the next item's first S_0 before
// it waits for tile 1's last P (plain causal / full kernels), so the two
// softmax groups stay staggered across work items.
//
// Lazy rescaling: a row's reference max m only moves when the tile max
// exceeds it by more than 8 (log2 units), so P <= 256 and O is rescaled in
// tensor memory only on those (rare) tiles, before any of the tile's P is
// released (every P V of the previous step has completed once S is
// committed).  The final O / l and the LSE use the same reference max, so
// the result is exact up to rounding.
//
// Softmax arithmetic per score: one three-input max per two scores, one
// packed FMA per two scores for s*scale*log2e - m, 2^x on the MUFU unit
// (POLY_EVERY > 0 moves one pair in POLY_EVERY to the FMA pipe,
// exp2_fma_pair; measured, every instantiation is faster all on MUFU), one
// packed add per two scores into the unrounded row sum and two mixed adds
// into the sum of the bf16-rounded weights.  P is rounded to bf16 for the
// MMA; O is divided by the sum of those rounded values (so O is a weighted
// mean with exactly the weights used) and the LSE uses the unrounded sum.
// The row max is taken over the first two 32-column loads of S while the last
// two are still in flight.
//
// Mask variants ("flash-attention" skill page, section 3.3), compiled into
// instantiations of their own (GENERAL = true) so the plain causal / full
// kernel keeps its lean inner loop.  LOGIT selects how the scores reach the
// exponent: 0 (a band alone) scales them like the plain kernel, inside the
// exponent's FMA; 1 rewrites every score in place (softcap, then ALiBi);
// 2 is ALiBi without softcap under a right bound of 0, where every visible
// key precedes its query, so the penalty slope * (key - query) is linear in
// the key's column and joins the row max and the exponent's FMA; 3 is
// softcap without ALiBi: tanh is increasing, so the row max is taken on the
// raw scores and capped once, and each score is capped inside the
// exponential loop:
//   - sliding window (left, right): query i sees keys i-left .. i+right.
//     Each query tile visits only the K/V tiles that intersect its band
//     [lo, hi), so a long sequence costs O(L * window), not O(L^2);
//   - softcap c: the logit x = scale * q.k becomes c * tanh(x / c), with
//     tanh(y) = 1 - 2 / (1 + e^(2y)) from one MUFU exp2 and one MUFU
//     reciprocal (absolute error a few fp32 ulps of 1, times c);
//   - ALiBi: the capped logit gets -slope * |i - j|, one FMA per score.
// In this form a row can see no key at all in its first K/V tile (the band
// starts inside the tile), so its running max may start at -inf; the exp
// argument and the rescale factor are guarded for that.
//
// FP8 (an instantiation of its own, FP8 = true; causal or full mask): Q, K, V
// are e4m3 bytes with per-tensor descale factors.  Both products run as
// tcgen05 kind::f8f6f4 MMAs (K steps of 32 elements = 32 bytes, so a d=128
// row is one 128-byte swizzle panel and a tile is 16 KB).  P is rounded to
// e4m3 (P <= 256 by the lazy rescale, within e4m3's 448) and packed four per
// tensor-memory column; the row sum that normalises O adds the decoded e4m3
// values, the LSE sum the unrounded ones.  q_descale * k_descale joins the
// softmax scale and v_descale the epilogue's 1/l.
#pragma once

#include "ptx.cuh"

namespace fa {
namespace prefill {

constexpr int BM = 128;           // query rows per tile
constexpr int BN = 128;           // keys per K/V tile
constexpr int NQT = 2;            // query tiles per work item
constexpr int ROWS_PER_ITEM = NQT * BM;
constexpr int P_CHUNKS = 2;       // P is handed to the P V MMAs in chunks of BN / P_CHUNKS keys
static_assert(P_CHUNKS == 1 || P_CHUNKS == 2 || P_CHUNKS == 4, "P chunks are whole 32-key quarters");
constexpr int NUM_WARPS = 12;  // 3 warpgroups: control (K/V and Q producers, MMA, 1 idle), softmax x2
constexpr int NUM_THREADS = NUM_WARPS * 32;
// Register split between the warpgroups (setmaxnreg).  The launch allots
// kRegsLaunch per thread; the control group gives most of its share to the
// softmax groups: 128*kRegsControl + 256*kRegsSoftmax <= 384*kRegsLaunch.
constexpr uint32_t kRegsLaunch = 168;
constexpr uint32_t kRegsControl = 104;
constexpr uint32_t kRegsSoftmax = 200;
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= NUM_THREADS * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr uint32_t TMEM_COLS = 512;
constexpr float kRescaleThreshold = 8.0f;
constexpr int MAX_LEVELS = 4096;  // max_seqlen <= 4096 * 256
constexpr int MAX_ITEMS_PER_CTA = 96;
constexpr int SMEM_LIMIT = 232448;  // dynamic shared memory per CTA on sm_100

// Instruction descriptor for e4m3 x e4m3 -> fp32 (kind::f8f6f4): the A and
// B format fields (bits 7-9, 10-12) are 0 for E4M3; the rest as for bf16.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, bool a_mn_major,
                                                      bool b_mn_major) {
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

template <int D, bool FP8 = false>
struct Cfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(!FP8 || D == 128, "the e4m3 path takes head_dim 128");
  static constexpr int ESIZE = FP8 ? 1 : 2;           // bytes per element
  static constexpr int PANEL_ELEMS = 128 / ESIZE;     // elements per 128-byte swizzle row
  static constexpr int PANELS = D / PANEL_ELEMS;      // swizzle panels per tile row
  static constexpr int PANEL_BYTES = BM * 128;        // 128 rows x 128 B
  static constexpr int TILE_BYTES = BM * D * ESIZE;   // one Q, K or V tile
  static constexpr int STAGES = TILE_BYTES <= 16384 ? 8 : 4;  // K/V ring slots
  static constexpr int KSTEP = 32 / ESIZE;            // K elements per MMA (32 bytes)
  static constexpr int S_KSTEPS = D / KSTEP;          // MMAs per S tile
  static constexpr int PV_KSTEPS = BN / KSTEP;        // MMAs per P V tile
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = NQT * TILE_BYTES;
  // O leaves through a 4 KB bf16 staging region per softmax warp (32 rows x
  // 64 columns), 16 KB per query tile
  static constexpr int O_PANEL_BYTES = BM * 128;
  static constexpr int O_PANELS = D / 64;
  static constexpr int O_STAGE_OFF = KV_OFF + STAGES * TILE_BYTES;
  static constexpr int SMEM_TILES = O_STAGE_OFF + NQT * O_PANEL_BYTES;
  static constexpr uint32_t IDESC_S =
      FP8 ? idesc_e4m3_f32(BM, BN, false, false) : idesc_bf16_f32(BM, BN, false, false);
  static constexpr uint32_t IDESC_PV =
      FP8 ? idesc_e4m3_f32(BM, D, false, true) : idesc_bf16_f32(BM, D, false, true);
};

// D[tmem] (+)= A * B with e4m3 operands; A from shared memory or tensor memory
__device__ __forceinline__ void umma_ss_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_ts_e4m3(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// MMAs issued from a converged warp by one elected lane (see the elected
// helpers in ptx.cuh for why the issuing warps stay converged).
#define FA_ELECT "{\n\t.reg .pred P, Q;\n\telect.sync _|P, 0xffffffff;\n\t"
__device__ __forceinline__ void umma_ss_el(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate, bool e4m3) {
  if (e4m3)
    asm volatile(FA_ELECT "setp.ne.b32 Q, %4, 0;\n\t"
                 "@P tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, Q;\n\t}" ::"r"(d_tmem),
                 "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
  else
    asm volatile(FA_ELECT "setp.ne.b32 Q, %4, 0;\n\t"
                 "@P tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, Q;\n\t}" ::"r"(d_tmem),
                 "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
__device__ __forceinline__ void umma_ts_el(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate, bool e4m3) {
  if (e4m3)
    asm volatile(FA_ELECT "setp.ne.b32 Q, %4, 0;\n\t"
                 "@P tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, Q;\n\t}" ::"r"(d_tmem),
                 "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
  else
    asm volatile(FA_ELECT "setp.ne.b32 Q, %4, 0;\n\t"
                 "@P tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, Q;\n\t}" ::"r"(d_tmem),
                 "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
#undef FA_ELECT

// Two floats -> two e4m3 bytes (nearest, saturating to +-448) in the low 16
// bits; lo goes to the lower byte (the lower K index).
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tcvt.u32.u16 %0, t;\n\t}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// a0 += lower e4m3 value, a1 += upper (exactly: e4m3 -> f16 is exact)
__device__ __forceinline__ void add_e4m3x2_f32(uint32_t pq, float& a0, float& a1) {
  asm("{\n\t.reg .b16 q, h0, h1;\n\t.reg .b32 h2;\n\tcvt.u16.u32 q, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 h2, q;\n\tmov.b32 {h0, h1}, h2;\n\t"
      "add.rn.f32.f16 %0, h0, %0;\n\tadd.rn.f32.f16 %1, h1, %1;\n\t}"
      : "+f"(a0), "+f"(a1) : "r"(pq));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
               "r"(r[7])
               : "memory");
}

struct Shared {
  uint64_t q_full[NQT], q_empty[NQT], mma_done;  // Q: one barrier pair per query tile
  uint64_t kv_full[8], kv_empty[8];
  uint64_t s_full[NQT], o_full[NQT];
  uint64_t p_full[NQT][P_CHUNKS];  // one chunk of P written to TMEM
  uint64_t stall;                  // never arrived at (timeout test hook)
  uint64_t q_issued;               // the first item's Q loads have been issued
  uint32_t tmem_base;
  int abort;
  int num_items;                     // items this CTA processes
  int total_items;
  int4 items[MAX_ITEMS_PER_CTA];     // (start, len, level << 16 | h, b)
};

// Work-list construction scratch; only live before the main loop, so it
// shares its shared memory with the K/V ring (which the first TMA load
// overwrites after the prologue).
struct PlanScratch {
  int hist[MAX_LEVELS + 1];          // sequences with exactly n 256-row blocks
  int level_offset[MAX_LEVELS + 1];  // first item index of level (descending order)
};

template <int D, bool FP8 = false>
constexpr int smem_bytes() {
  static_assert(sizeof(PlanScratch) <= Cfg<D, FP8>::STAGES * Cfg<D, FP8>::TILE_BYTES,
                "plan scratch overflows the K/V ring");
  return Cfg<D, FP8>::SMEM_TILES + (int)sizeof(Shared) + 1024;
}
static_assert(smem_bytes<128>() <= SMEM_LIMIT && smem_bytes<64>() <= SMEM_LIMIT &&
                  smem_bytes<128, true>() <= SMEM_LIMIT,
              "shared memory layout exceeds the per-CTA limit");

struct Params {
  __nv_bfloat16* o;
  float* lse;
  const int32_t* cu_seqlens;
  int B, Hq, Hkv, group, T;
  int causal;
  float scale_log2;  // softmax scale * log2(e)
  int num_levels;    // ceil(max_seqlen / 256)
  // key band of query i: [i - wl, i + wr]; -1 = no limit on that side;
  // wr = 0 under the causal mask.  Every kernel instantiation honours the
  // band's tile range; only GENERAL masks inside tiles by wl / wr.
  int wl, wr;
  float o_scale;        // multiplies O / l in the epilogue (v_descale; 1 for bf16)
  float cap_in;         // 2 * log2(e) * scale / softcap (GENERAL, softcap > 0)
  float cap_out;        // softcap * log2(e); 0 = no softcap
  const float* alibi;   // ALiBi slopes (GENERAL), or null
  int alibi_stride;     // slope of (b, h) = alibi[b * alibi_stride + h]
};

// K/V tiles [lo, hi) that a query tile starting at local row rs (< len)
// has to visit: the tiles intersecting the union of its rows' key bands.
__device__ __forceinline__ void tile_kv_range(const Params& p, int rs, int len, int& lo, int& hi) {
  const int nkv = (len + BN - 1) / BN;
  const int re = min(rs + BM, len) - 1;  // last row of the tile
  hi = p.wr >= 0 ? min(nkv, (re + p.wr) / BN + 1) : nkv;
  lo = p.wl >= 0 ? max(0, rs - p.wl) / BN : 0;
}

// K/V tiles a work item (query tiles q0 and q0 + BM) streams: [lo, hi).  The
// second tile's range starts no earlier and ends no earlier than the first's
// and the two overlap or touch, so the union is one interval.
__device__ __forceinline__ void item_kv_range(const Params& p, int q0, int len, int& lo, int& hi) {
  tile_kv_range(p, q0, len, lo, hi);
  if (q0 + BM < len) {
    int lo1, hi1;
    tile_kv_range(p, q0 + BM, len, lo1, hi1);
    hi = max(hi, hi1);
  }
}

// Length of sequence b as the kernel uses it: an inconsistent cu_seqlens
// entry reports a bounds error and makes the sequence empty.
__device__ __forceinline__ void seq_range(const Params& p, int b, int& start, int& len) {
  const int s = __ldg(p.cu_seqlens + b);
  const int e = __ldg(p.cu_seqlens + b + 1);
  if (s < 0 || e < s || e > p.T) {
    start = 0;
    len = 0;
    return;
  }
  start = s;
  len = e - s;
}

__device__ __forceinline__ int blocks_of(int len) { return (len + ROWS_PER_ITEM - 1) / ROWS_PER_ITEM; }

// Work item w -> (b, level, h).  Items are ordered by descending level
// (longest causal work first); within a level by sequence, then head.
__device__ void decode_item(const Params& p, const PlanScratch& sh, int w, int& b, int& level,
                            int& h) {
  // level_offset[k] is the first item of level num_levels-1-k; find the
  // last k whose offset is <= w (empty levels share their successor's offset)
  int a = 0, z = p.num_levels - 1;
  while (a < z) {
    const int mid = (a + z + 1) >> 1;
    if (sh.level_offset[mid] <= w) a = mid; else z = mid - 1;
  }
  const int k = a;
  level = p.num_levels - 1 - k;
  const int r = w - sh.level_offset[k];
  const int rank = r / p.Hq;
  h = r - rank * p.Hq;
  int seen = 0;
  b = 0;
  for (int i = 0; i < p.B; ++i) {
    int st, len;
    seq_range(p, i, st, len);
    if (blocks_of(len) > level) {
      if (seen == rank) {
        b = i;
        return;
      }
      ++seen;
    }
  }
}

template <int D, bool GENERAL, bool FP8 = false, int LOGIT = 0>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV,
                   const Params p) {
  using C = Cfg<D, FP8>;
  static_assert(!(GENERAL && FP8), "mask variants are not built for e4m3");
  static_assert(GENERAL || LOGIT == 0, "softcap and ALiBi come with the mask-variant kernel");
  constexpr bool INPLACE = LOGIT == 1;  // scores rewritten in place
  constexpr bool LINEAR = LOGIT == 2;   // causal ALiBi folded into max and exponent
  constexpr bool SOFTCAP = LOGIT == 3;  // softcap applied in the exponential loop
  // one exp2 pair in POLY_EVERY on the FMA pipe, the rest on MUFU (0: all MUFU)
  constexpr int POLY_EVERY = 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* q_smem = smem + C::Q_OFF;
  uint8_t* kv_smem = smem + C::KV_OFF;
  uint8_t* o_stage = smem + C::O_STAGE_OFF;
  Shared& sh = *reinterpret_cast<Shared*>(smem + C::SMEM_TILES);
  PlanScratch& ps = *reinterpret_cast<PlanScratch*>(kv_smem);

  const int warp = warp_id();
  const int lane = lane_id();
  const int tid = threadIdx.x;

  // ---------------- prologue: barriers, TMEM, work list ----------------
  if (tid == 0) {
    for (int t = 0; t < NQT; ++t) {
      mbar_init(&sh.q_full[t], 1);
      mbar_init(&sh.q_empty[t], 1);
    }
    mbar_init(&sh.mma_done, 1);
    mbar_init(&sh.stall, 1);
    mbar_init(&sh.q_issued, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&sh.kv_full[s], 1);
      mbar_init(&sh.kv_empty[s], 1);
    }
    for (int t = 0; t < NQT; ++t) {
      mbar_init(&sh.s_full[t], 1);
      for (int c = 0; c < P_CHUNKS; ++c) mbar_init(&sh.p_full[t][c], BM);
      mbar_init(&sh.o_full[t], 1);
    }
    sh.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  for (int l = tid; l <= p.num_levels; l += NUM_THREADS) ps.hist[l] = 0;
  __syncthreads();
  for (int b = tid; b < p.B; b += NUM_THREADS) {
    int st, len;
    const int s = __ldg(p.cu_seqlens + b), e = __ldg(p.cu_seqlens + b + 1);
    if (s < 0 || e < s || e > p.T || (b == 0 && s != 0)) report_error(kDevErrBounds);
    seq_range(p, b, st, len);
    int nb = blocks_of(len);
    if (nb > p.num_levels) {
      report_error(kDevErrBounds);
      nb = p.num_levels;
    }
    // level l holds sequence b for every l < nb
    atomicAdd(&ps.hist[nb], 1);
  }
  __syncthreads();
  if (tid == 0) {
    // level l holds the sequences with more than l blocks: sum of hist[n], n > l
    int acc = 0, cnt = 0;
    for (int k = 0; k < p.num_levels; ++k) {
      cnt += ps.hist[p.num_levels - k];
      ps.level_offset[k] = acc;
      acc += cnt * p.Hq;
    }
    ps.level_offset[p.num_levels] = acc;
    sh.total_items = acc;
    // zig-zag assignment: round r takes item r*G + (r even ? c : G-1-c)
    const int G = gridDim.x, c = blockIdx.x;
    int n = 0;
    for (int r = 0;; ++r) {
      const int w = r * G + ((r & 1) ? (G - 1 - c) : c);
      if (w >= acc) break;
      ++n;
    }
    if (n > MAX_ITEMS_PER_CTA) {
      report_error(kDevErrBounds);
      n = MAX_ITEMS_PER_CTA;
    }
    sh.num_items = n;
  }
  __syncthreads();
  for (int i = tid; i < sh.num_items; i += NUM_THREADS) {
    const int G = gridDim.x, c = blockIdx.x;
    const int w = i * G + ((i & 1) ? (G - 1 - c) : c);
    int b, level, h, st, len;
    decode_item(p, ps, w, b, level, h);
    seq_range(p, b, st, len);
    // the sequence range travels with the item: no role reads cu_seqlens
    // (global memory) at an item boundary
    sh.items[i] = make_int4(st, len, (level << 16) | h, b);
  }
  // the plan scratch was written through the generic proxy; the ring's TMA
  // loads (async proxy) overwrite it after the barrier below
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const int num_items = sh.num_items;
  volatile int* abort = &sh.abort;

  if (warp < 4) {
    // ---- warpgroup 0: K/V producer (warp 0), MMA issuer (warp 1), Q producer (warp 2), warp 3 idle ----
    setmaxnreg_dec<kRegsControl>();
   if (warp == 0) {
    // ================ TMA producer (converged warp, elected issue) ================
    {
      uint32_t kv_it = 0;
      for (int it = 0; it < num_items && !*abort; ++it) {
        const int4 item = sh.items[it];
        const int start = item.x, len = item.y, level = item.z >> 16, h = item.z & 0xFFFF;
        const int q0 = level * ROWS_PER_ITEM;
        int jlo, jhi;
        item_kv_range(p, q0, len, jlo, jhi);
        const int kh = h / p.group;
        // K/V tiles of this item, 2*j + which; the ring runs on across items,
        // so the next item's first tiles load while this one drains
        bool stop = false;
        for (int next = 0; next < 2 * (jhi - jlo); ++next) {
          const uint32_t slot = kv_it % C::STAGES;
          if (!mbar_wait(&sh.kv_empty[slot], ((kv_it / C::STAGES) & 1) ^ 1, abort)) {
            stop = true;
            break;
          }
          // At the start every CTA loads at once: the first K tile goes out,
          // then the rest of the ring waits until the first item's Q tiles
          // are issued, so the loads the first Q K^T needs come first.
          if (kv_it == 1 && !mbar_wait(&sh.q_issued, 0, abort)) {
            stop = true;
            break;
          }
          expect_tx_el(&sh.kv_full[slot], C::TILE_BYTES);
          uint8_t* dst = kv_smem + slot * C::TILE_BYTES;
          const CUtensorMap* m = (next & 1) ? &tmV : &tmK;
#pragma unroll
          for (int pn = 0; pn < C::PANELS; ++pn)
            tma_load_2d_el(dst + pn * C::PANEL_BYTES, m, &sh.kv_full[slot],
                           kh * D + pn * C::PANEL_ELEMS, start + (jlo + (next >> 1)) * BN);
          ++kv_it;
        }
        if (stop) break;
      }
      // Before the CTA can exit, every load issued must have landed (bounded
      // wait that ignores the abort flag: the copies finish on their own).
      for (uint32_t s = 0; s < (uint32_t)C::STAGES && s < kv_it; ++s) {
        const uint32_t last = kv_it - 1 - ((kv_it - 1 - s) % C::STAGES);  // last use of slot
        mbar_wait_bounded(&sh.kv_full[last % C::STAGES], (last / C::STAGES) & 1);
      }
    }
   } else if (warp == 2) {
    // ================ Q producer (converged warp, elected issue) ================
    // Each query tile's buffer is refilled as soon as the previous item's
    // last Q K^T of that tile has run (tile 0 usually a step before tile 1),
    // independently of the K/V ring, so the next item's first Q K^T never
    // waits behind a K/V slot.
    {
      uint32_t q_issued[NQT] = {};
      for (int it = 0; it < num_items && !*abort; ++it) {
        const int4 item = sh.items[it];
        const int start = item.x, level = item.z >> 16, h = item.z & 0xFFFF;
        const int q0 = level * ROWS_PER_ITEM;
        bool stop = false;
#pragma unroll
        for (int t = 0; t < NQT; ++t) {
          if (!mbar_wait(&sh.q_empty[t], (it & 1) ^ 1, abort)) { stop = true; break; }
          expect_tx_el(&sh.q_full[t], C::TILE_BYTES);
#pragma unroll
          for (int pn = 0; pn < C::PANELS; ++pn)
            tma_load_2d_el(q_smem + t * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmQ, &sh.q_full[t],
                           h * D + pn * C::PANEL_ELEMS, start + q0 + t * BM);
          ++q_issued[t];
        }
        if (stop) break;
        if (it == 0) {
          // the K/V ring may now fill; the first prefetch below waits until
          // this item's Q has landed, so it never delays the first loads
          if (lane == 0) mbar_arrive(&sh.q_issued);
          __syncwarp();
          if (!mbar_wait(&sh.q_full[NQT - 1], 0, abort)) break;
        }
        if (it + 1 < num_items) {
          // the next item's Q tiles come from DRAM; pull them into L2 now so
          // their load at the next item boundary is short.  (Prefetching the
          // next item's first K/V tiles as well measured slower.)
          const int4 nx = sh.items[it + 1];
          const int nq0 = nx.x + (nx.z >> 16) * ROWS_PER_ITEM, nh = nx.z & 0xFFFF;
#pragma unroll
          for (int t = 0; t < NQT; ++t)
#pragma unroll
            for (int pn = 0; pn < C::PANELS; ++pn)
              tma_prefetch_l2_2d_el(&tmQ, nh * D + pn * C::PANEL_ELEMS, nq0 + t * BM);
        }
      }
      // every Q load issued must have landed before the CTA exits
#pragma unroll
      for (int t = 0; t < NQT; ++t)
        if (q_issued[t] > 0) mbar_wait_bounded(&sh.q_full[t], (q_issued[t] - 1) & 1);
    }
   } else if (warp == 1) {
    // ================ MMA issuer (converged warp, elected issue) ================
    {
      const uint32_t q_addr = smem_u32(q_smem);
      const uint32_t kv_addr = smem_u32(kv_smem);
      uint32_t kv_it = 0;
      uint32_t p_phase0 = 0, p_phase1 = 0;
      bool ok = true;
      // Descriptors of the first Q tile and the first K/V slot; every other
      // operand is the same descriptor with its start address advanced.
      const uint64_t q_desc = sdesc_sw128(q_addr, 16, 1024);           // K-major
      const uint64_t k_desc = sdesc_sw128(kv_addr, 16, 1024);          // K-major
      const uint64_t v_desc = sdesc_sw128(kv_addr, C::PANEL_BYTES, 1024);  // MN-major
      // O_t += P_t V over the keys of P chunk c (A = P from TMEM, B = V,
      // MN-major); the first chunk of a tile's first step overwrites O
      constexpr int PV_PER_CHUNK = C::PV_KSTEPS / P_CHUNKS;
      auto issue_pv = [&](int t, uint32_t v_idx, int c, bool first) {
        const uint64_t vd = sdesc_advance(v_desc, (v_idx % C::STAGES) * C::TILE_BYTES);
        const uint32_t d_tmem = tmem + 256 + t * 128, a_tmem = tmem + t * 128;
        // K step kk: 16 (bf16) or 32 (e4m3) keys = 8 tensor-memory columns of
        // P and KSTEP rows of 128 B of V
#pragma unroll
        for (int q = 0; q < PV_PER_CHUNK; ++q) {
          const int kk = c * PV_PER_CHUNK + q;
          umma_ts_el(d_tmem, a_tmem + kk * 8, sdesc_advance(vd, kk * C::KSTEP * 128), C::IDESC_PV,
                     (first && kk == 0) ? 0u : 1u, FP8);
        }
      };
      // S_t = Q_t K^T   (both K-major)
      auto issue_s = [&](int t, uint32_t k_idx) {
        const uint64_t qd = sdesc_advance(q_desc, t * C::TILE_BYTES);
        const uint64_t kd = sdesc_advance(k_desc, (k_idx % C::STAGES) * C::TILE_BYTES);
        const uint32_t d_tmem = tmem + t * 128;
#pragma unroll
        for (int kk = 0; kk < C::S_KSTEPS; ++kk) {
          const uint32_t off = (kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32;
          umma_ss_el(d_tmem, sdesc_advance(qd, off), sdesc_advance(kd, off), C::IDESC_S,
                     kk > 0 ? 1u : 0u, FP8);
        }
      };
      // Lookahead across items: at an item's last step (only tile 1's last
      // P V left, since tile 1 ends a step after tile 0 under the causal
      // mask), tile 0's first Q K^T of the next item is issued before the
      // wait for tile 1's softmax, so the two softmax groups stay staggered
      // across item boundaries instead of restarting together.  Only the
      // plain causal / full kernels take it: with the masked variants'
      // longer softmax it measured slower.
      bool la_done = false;  // this item's first tile-0 S was issued by the lookahead
      for (int it = 0; it < num_items && ok; ++it) {
        const int4 item = sh.items[it];
        const int len = item.y, level = item.z >> 16;
        const int q0 = level * ROWS_PER_ITEM;
        // K/V tile range of each query tile; an absent second tile gets an
        // empty range
        int lo0, hi0, lo1 = 0, hi1 = 0;
        tile_kv_range(p, q0, len, lo0, hi0);
        if (q0 + BM < len) tile_kv_range(p, q0 + BM, len, lo1, hi1);
        const int jlo = lo0, jhi = max(hi0, hi1);
        // per tile: Q waited for, Q released (each exactly once per item)
        bool qw0 = la_done, qw1 = false;
        bool qr0 = la_done && hi0 - lo0 == 1, qr1 = false;
        const bool skip_s0 = la_done;
        la_done = false;
        const uint32_t base = kv_it;
        // step j issues P V of tile j-1 and Q K^T of tile j, per query tile
        for (int j = jlo; j <= jhi; ++j) {
          const uint32_t k_idx = base + 2 * (j - jlo), v_idx = k_idx - 1;
          // both slots are normally full already: test them together so the
          // two barrier latencies overlap, and block only on a miss
          const bool k_ready = j >= jhi || mbar_try_wait(smem_u32(&sh.kv_full[k_idx % C::STAGES]),
                                                     (k_idx / C::STAGES) & 1);
          const bool v_ready = j <= jlo || mbar_try_wait(smem_u32(&sh.kv_full[v_idx % C::STAGES]),
                                                     (v_idx / C::STAGES) & 1);
          if (!k_ready &&
              !mbar_wait(&sh.kv_full[k_idx % C::STAGES], (k_idx / C::STAGES) & 1, abort)) {
            ok = false;
            break;
          }
          if (!v_ready &&
              !mbar_wait(&sh.kv_full[v_idx % C::STAGES], (v_idx / C::STAGES) & 1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // query tile 0
          if (j > lo0 && j <= hi0) {
            // each chunk's MMAs go out as soon as the softmax has stored it
            bool pv_ok = true;
#pragma unroll
            for (int c = 0; c < P_CHUNKS; ++c) {
              if (!mbar_wait(&sh.p_full[0][c], p_phase0, abort)) { pv_ok = false; break; }
              tc_fence_after();
              issue_pv(0, v_idx, c, j == lo0 + 1);
            }
            if (!pv_ok) { ok = false; break; }
            p_phase0 ^= 1;
            if (j == hi0) commit_el(&sh.o_full[0]);
          }
          // tile 0's Q K^T of this step or, at the item's last step, the
          // next item's first one (lookahead); never both in one step
          int s0_idx = -1;       // K slot of tile 0's Q K^T, if any
          bool s0_last = false;  // it is the last one of its item: release Q0
          if (j >= lo0 && j < hi0 && !(skip_s0 && j == lo0)) {
            if (!qw0) {
              if (!mbar_wait(&sh.q_full[0], it & 1, abort)) { ok = false; break; }
              qw0 = true;
            }
            s0_idx = (int)k_idx;
            s0_last = j == hi0 - 1;
            qr0 = qr0 || s0_last;
          } else if (!GENERAL && j == jhi && hi0 < jhi && qr0 && it + 1 < num_items) {
            const int4 nx = sh.items[it + 1];
            int nlo, nhi;
            tile_kv_range(p, (nx.z >> 16) * ROWS_PER_ITEM, nx.y, nlo, nhi);
            if (nhi > nlo) {
              const uint32_t nk = base + 2 * (jhi - jlo);  // the next item's first K
              if (!mbar_wait(&sh.q_full[0], (it + 1) & 1, abort) ||
                  !mbar_wait(&sh.kv_full[nk % C::STAGES], (nk / C::STAGES) & 1, abort)) {
                ok = false;
                break;
              }
              s0_idx = (int)nk;
              s0_last = nhi - nlo == 1;
              la_done = true;
            }
          }
          if (s0_idx >= 0) {
            tc_fence_after();
            issue_s(0, (uint32_t)s0_idx);
            commit_el(&sh.s_full[0]);
            if (s0_last) commit_el(&sh.q_empty[0]);
          }
          // query tile 1
          if (j > lo1 && j <= hi1) {
            // each chunk's MMAs go out as soon as the softmax has stored it
            bool pv_ok = true;
#pragma unroll
            for (int c = 0; c < P_CHUNKS; ++c) {
              if (!mbar_wait(&sh.p_full[1][c], p_phase1, abort)) { pv_ok = false; break; }
              tc_fence_after();
              issue_pv(1, v_idx, c, j == lo1 + 1);
            }
            if (!pv_ok) { ok = false; break; }
            p_phase1 ^= 1;
            if (j == hi1) commit_el(&sh.o_full[1]);
          }
          if (j >= lo1 && j < hi1) {
            if (!qw1) {
              if (!mbar_wait(&sh.q_full[1], it & 1, abort)) { ok = false; break; }
              qw1 = true;
              tc_fence_after();
            }
            issue_s(1, k_idx);
            commit_el(&sh.s_full[1]);
            if (j == hi1 - 1) { commit_el(&sh.q_empty[1]); qr1 = true; }
          }
          if (j > jlo) commit_el(&sh.kv_empty[v_idx % C::STAGES]);
          if (j < jhi) commit_el(&sh.kv_empty[k_idx % C::STAGES]);
        }
        if (!ok) break;
        // a tile with no Q K^T in this item (past the sequence end) still
        // takes its Q phase and releases its buffer, keeping the phases paired
        if (!qw0 && !mbar_wait(&sh.q_full[0], it & 1, abort)) { ok = false; break; }
        if (!qr0) commit_el(&sh.q_empty[0]);
        if (!qw1 && !mbar_wait(&sh.q_full[1], it & 1, abort)) { ok = false; break; }
        if (!qr1) commit_el(&sh.q_empty[1]);
        kv_it = base + 2 * (jhi - jlo);
      }
      // every MMA issued must finish before TMEM is released
      commit_el(&sh.mma_done);
      mbar_wait_bounded(&sh.mma_done, 0);
    }
   }
  } else {
    // ======================= softmax warpgroups =======================
    setmaxnreg_inc<kRegsSoftmax>();
    const int t = (warp - 4) >> 2;          // query tile of this group
    const int quarter = warp & 3;           // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;    // row of the tile owned by this thread
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t s_col = lane_base + t * 128;
    const uint32_t o_col = lane_base + 256 + t * 128;
    uint32_t s_phase = 0, o_phase = 0;
    // timeout test hook: this group's first S wait is on a barrier that
    // nothing arrives at
    bool stall = t == 0 && blockIdx.x == 0 &&
                 *reinterpret_cast<volatile int*>(&g_stall_test) == kStallPrefill;
    const float sl = p.scale_log2;
    const uint64_t sl2 = f2_pack(sl, sl);
    bool ok = true;
    for (int it = 0; it < num_items && ok; ++it) {
      const int4 item = sh.items[it];
      const int start = item.x, len = item.y, level = item.z >> 16, h = item.z & 0xFFFF, b = item.w;
      const int rs = level * ROWS_PER_ITEM + t * BM;  // first row of this tile
      if (rs >= len) continue;
      int jlo, jhi;
      tile_kv_range(p, rs, len, jlo, jhi);
      const int qpos = rs + row;
      // ALiBi slope of this (sequence, head) in log2 units (LOGIT 1 and 2)
      const float slope2 =
          (LOGIT != 0 && p.alibi) ? __ldg(p.alibi + (size_t)b * p.alibi_stride + h) * 1.4426950408889634f
                               : 0.f;
      float m_ref = -INFINITY;
      // Row sums: le (two interleaved fp32 pairs) = sum of the unrounded
      // weights, gives the LSE; lr = sum of the rounded (bf16, or decoded
      // e4m3) weights the P V MMA consumes, normalises O, so O is a weighted
      // mean with exactly the weights used.
      uint64_t le_a = 0, le_b = 0;
      float lr_a0 = 0.f, lr_a1 = 0.f, lr_b0 = 0.f, lr_b1 = 0.f;
      for (int j = jlo; j < jhi; ++j) {
        if (!mbar_wait(stall ? &sh.stall : &sh.s_full[t], s_phase, abort)) { ok = false; break; }
        stall = false;
        s_phase ^= 1;
        tc_fence_after();
        uint32_t s[4][32];
        const int kv0 = j * BN;
        // masking of chunk c (32 columns): keys outside [0, len) or outside
        // the row's band (GENERAL), keys past the sequence end or after the
        // query (plain)
        bool need_mask;
        int lim_lo = -1, lim_hi = BN;  // visible columns [lim_lo, lim_hi)
        if constexpr (GENERAL) {
          need_mask = kv0 + BN > len || (p.wr >= 0 && kv0 + BN - 1 > rs + p.wr) ||
                      (p.wl >= 0 && kv0 < rs + BM - 1 - p.wl);
          lim_lo = p.wl >= 0 ? qpos - p.wl - kv0 : -1;
          lim_hi = min(len, p.wr >= 0 ? qpos + p.wr + 1 : len) - kv0;
        } else {
          need_mask = kv0 + BN > len || (p.causal && kv0 + BN - 1 > rs);
          lim_hi = min(len, p.causal ? qpos + 1 : len) - kv0;
        }
        // INPLACE (softcap with ALiBi, or ALiBi under a right bound other
        // than 0): logits in log2 units (optional cap, then the ALiBi
        // penalty); then, in every kernel, the mask (band, sequence end,
        // causal)
        auto prepare = [&](uint32_t (&x)[32], int c) {
          if constexpr (INPLACE) {
            if (p.cap_out > 0.f) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                x[e] = __float_as_uint(softcap_log2(__uint_as_float(x[e]), p.cap_in, p.cap_out));
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) x[e] = __float_as_uint(__uint_as_float(x[e]) * sl);
            }
            if (slope2 != 0.f) {
              const float d0 = (float)(kv0 + c * 32 - qpos);  // key - query for column 0 of the chunk
#pragma unroll
              for (int e = 0; e < 32; ++e)
                x[e] = __float_as_uint(
                    fmaf(-slope2, fabsf(d0 + (float)e), __uint_as_float(x[e])));
            }
          }
          if (need_mask) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              x[e] = (c * 32 + e < lim_lo || c * 32 + e >= lim_hi) ? __float_as_uint(-INFINITY)
                                                                  : x[e];
          }
        };
        // row max: four independent chains of three-input maxima per pair of
        // chunks; the max of chunks 0-1 runs while chunks 2-3 load
        float mx[8];
        // LINEAR: the max of s * scale + slope * column (log2 units); the row's
        // constant slope * (kv0 - query) is added once below
        const uint64_t sp2 = f2_pack(slope2, slope2);
        auto chunk_max = [&](const uint32_t (&a)[32], const uint32_t (&b)[32], float* m, int cb) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t* src = (k < 2) ? a : b;
            const int o = (k & 1) * 16;
            if constexpr (LINEAR) {
              const int c0 = cb + (k >> 1) * 32 + o;  // column of src[o]
              float y[16];
#pragma unroll
              for (int e = 0; e < 16; e += 2) {
                const uint64_t t = f2_mul(sp2, f2_pack((float)(c0 + e), (float)(c0 + e + 1)));
                f2_unpack(f2_fma(f2_pack(__uint_as_float(src[o + e]), __uint_as_float(src[o + e + 1])),
                                 sl2, t),
                          y[e], y[e + 1]);
              }
              m[k] = fmaxf(y[0], y[1]);
#pragma unroll
              for (int e = 2; e < 16; e += 2) m[k] = fmax3(m[k], y[e], y[e + 1]);
            } else {
              m[k] = fmaxf(__uint_as_float(src[o]), __uint_as_float(src[o + 1]));
#pragma unroll
              for (int e = 2; e < 16; e += 2)
                m[k] = fmax3(m[k], __uint_as_float(src[o + e]), __uint_as_float(src[o + e + 1]));
            }
          }
        };
        tmem_ld32(s_col, s[0]);
        tmem_ld32(s_col + 32, s[1]);
        tmem_ld_wait(s[0]);
        tmem_ld_tie(s[1]);
        tmem_ld32(s_col + 64, s[2]);
        tmem_ld32(s_col + 96, s[3]);
        prepare(s[0], 0);
        prepare(s[1], 1);
        chunk_max(s[0], s[1], mx, 0);
        tmem_ld_wait(s[2]);
        tmem_ld_tie(s[3]);
        prepare(s[2], 2);
        prepare(s[3], 3);
        chunk_max(s[2], s[3], mx + 4, 64);
        float mx_s = fmaxf(fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5])),
                           fmaxf(mx[6], mx[7]));
        if constexpr (LOGIT == 0) mx_s *= sl;
        if constexpr (LINEAR) mx_s += slope2 * (float)(kv0 - qpos);
        if constexpr (SOFTCAP)
          mx_s = mx_s == -INFINITY ? -INFINITY : softcap_log2(mx_s, p.cap_in, p.cap_out);
        // Lazy rescale, decided per row: the reference max moves only when the
        // tile max exceeds it by more than the threshold.  The exponentials
        // start at once with this row's reference; O is rescaled in tensor
        // memory (a warp-wide pass, if any row of the warp moved) just before
        // the first chunk of P is released.
        float alpha = 1.f;
        bool moved = false;
        if (j == jlo) {
          // GENERAL keeps -inf for a row that sees nothing in this tile
          m_ref = (!GENERAL && mx_s == -INFINITY) ? 0.f : mx_s;
        } else if (mx_s > m_ref + kRescaleThreshold) {
          const float m_new = fmaxf(m_ref, mx_s);
          // (m_ref == m_new also covers -inf == -inf, where the difference is NaN)
          alpha = (GENERAL && m_new == m_ref) ? 1.f : ex2(m_ref - m_new);
          m_ref = m_new;
          moved = true;
          const uint64_t a2 = f2_pack(alpha, alpha);
          le_a = f2_mul(le_a, a2);
          le_b = f2_mul(le_b, a2);
          lr_a0 *= alpha;
          lr_a1 *= alpha;
          lr_b0 *= alpha;
          lr_b1 *= alpha;
        }
        const bool rescale = j != jlo && __any_sync(0xffffffffu, moved);
        auto rescale_o = [&]() {
          // O *= alpha: every P V of step j-1 has completed (they precede
          // S_t(j) in issue order) and none of step j has started.  16
          // columns at a time, since S is still held in registers here.
          const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(o_col + c * 16, o);
            tmem_ld_wait16(o);
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              float o0, o1;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2), o0, o1);
              o[e] = __float_as_uint(o0);
              o[e + 1] = __float_as_uint(o1);
            }
            tmem_st16(o_col + c * 16, o);
          }
        };
        // P = 2^(s*scale*log2e - m); packed bf16 (or e4m3) pairs overwrite
        // s[c][0..] in order
        const float m_use = (GENERAL && m_ref == -INFINITY) ? 0.f : m_ref;
        const uint64_t neg2 = f2_pack(-m_use, -m_use);
        // INPLACE: s already holds scaled logits, so the FMA multiplies by 1
        const uint64_t mul2 = INPLACE ? f2_pack(1.f, 1.f) : sl2;
        const uint64_t cap2 = f2_pack(p.cap_out, p.cap_out);  // SOFTCAP
        // LINEAR: the exponent's addend is slope * (column + kv0 - query) - m
        const uint64_t am2 = LINEAR ? f2_add(f2_pack(slope2 * (float)(kv0 - qpos), slope2 * (float)(kv0 - qpos)), neg2)
                                    : neg2;
        uint32_t e4_lo = 0;  // e4m3: the even pair of a word, waiting for the odd one
        // four 32-key quarters; a chunk is 4 / P_CHUNKS consecutive quarters
        constexpr int QPC = 4 / P_CHUNKS;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            uint64_t x;
            if constexpr (SOFTCAP) {
              // cap * tanh, in log2 units, minus m; a masked score stays -inf
              const float s0 = __uint_as_float(s[c][e]), s1 = __uint_as_float(s[c][e + 1]);
              const uint64_t th = f2_fma(f2_pack(rcp_approx(1.f + ex2(s0 * p.cap_in)),
                                                 rcp_approx(1.f + ex2(s1 * p.cap_in))),
                                         f2_pack(-2.f, -2.f), f2_pack(1.f, 1.f));
              float x0, x1;
              f2_unpack(f2_fma(th, cap2, neg2), x0, x1);
              x = f2_pack(s0 == -INFINITY ? -INFINITY : x0, s1 == -INFINITY ? -INFINITY : x1);
            } else {
              uint64_t add2 = neg2;
              if constexpr (LINEAR)
                add2 = f2_fma(sp2, f2_pack((float)(c * 32 + e), (float)(c * 32 + e + 1)), am2);
              x = f2_fma(f2_pack(__uint_as_float(s[c][e]), __uint_as_float(s[c][e + 1])), mul2, add2);
            }
            uint64_t pr;
            if (POLY_EVERY > 0 && ((e >> 1) % (POLY_EVERY > 0 ? POLY_EVERY : 1)) == POLY_EVERY - 1) {
              pr = exp2_fma_pair(x);
            } else {
              float x0, x1;
              f2_unpack(x, x0, x1);
              pr = f2_pack(ex2(x0), ex2(x1));
            }
            float p0, p1;
            f2_unpack(pr, p0, p1);
            if ((e >> 1) & 1) le_b = f2_add(le_b, pr); else le_a = f2_add(le_a, pr);
            if constexpr (FP8) {
              // four e4m3 per word: pairs 2w and 2w+1 of the chunk form word w
              const uint32_t pq = pack_e4m3x2(p0, p1);
              if ((e >> 1) & 1) {
                add_e4m3x2_f32(pq, lr_b0, lr_b1);
                s[c][e >> 2] = e4_lo | (pq << 16);
              } else {
                add_e4m3x2_f32(pq, lr_a0, lr_a1);
                e4_lo = pq;
              }
            } else {
              s[c][e >> 1] = pack_bf16x2(p0, p1);
            }
          }
          if constexpr (!FP8) {
            // the bf16 weights the P V MMA consumes, summed from the packed
            // words of the quarter (after its exponentials)
#pragma unroll
            for (int w = 0; w < 16; w += 2) {
              lr_a0 = add_bf16lo_f32(s[c][w], lr_a0);
              lr_a1 = add_bf16hi_f32(s[c][w], lr_a1);
              lr_b0 = add_bf16lo_f32(s[c][w + 1], lr_b0);
              lr_b1 = add_bf16hi_f32(s[c][w + 1], lr_b1);
            }
          }
          // the chunk that ended with quarter c-1 has had this quarter's math
          // to land: release it (after the O rescale, before the first
          // release), then store quarter c
          if (c > 0 && c % QPC == 0) {
            if (c == QPC && rescale) rescale_o();
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&sh.p_full[t][c / QPC - 1]);
          }
          if constexpr (FP8)
            tmem_st8(s_col + c * 8, s[c]);  // 32 keys per 8 columns
          else
            tmem_st16(s_col + c * 16, s[c]);
        }
        if (QPC == 4 && rescale) rescale_o();
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&sh.p_full[t][P_CHUNKS - 1]);
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16, LSE ----
      if (!mbar_wait(&sh.o_full[t], o_phase, abort)) { ok = false; break; }
      o_phase ^= 1;
      tc_fence_after();
      float la0, la1, lb0, lb1;
      f2_unpack(le_a, la0, la1);
      f2_unpack(le_b, lb0, lb1);
      const float l_exact = (la0 + la1) + (lb0 + lb1);
      const float l_norm = (lr_a0 + lr_a1) + (lr_b0 + lr_b1);
      const bool valid = qpos < len;
      const float inv_l = p.o_scale / l_norm;
      const size_t grow = (size_t)(start + qpos);
      // Each warp writes its own 32 rows, one 64-column panel at a time:
      // every thread puts its row into the warp's 4 KB staging region
      // (16-byte chunks XOR-swizzled by row, so neither the writes nor the
      // reads conflict on banks), then the warp reads it back four rows per
      // instruction, eight lanes per row, for 128-byte global stores.  Rows
      // past the sequence end are not stored; every lane takes part in the
      // warp-wide TMEM loads.  Only __syncwarp orders the staging.
      uint8_t* wst = o_stage + (t * 4 + quarter) * 4096;
      const int rbase = rs + quarter * 32;  // local row of the warp's lane 0
#pragma unroll
      for (int pn = 0; pn < C::O_PANELS; ++pn) {
        uint32_t o[2][32];
        tmem_ld32(o_col + pn * 64, o[0]);
        tmem_ld32(o_col + pn * 64 + 32, o[1]);
        tmem_ld_wait(o[0]);
        tmem_ld_tie(o[1]);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t* src = o[c >> 2] + (c & 3) * 8;
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(src[0]) * inv_l, __uint_as_float(src[1]) * inv_l);
          v.y = pack_bf16x2(__uint_as_float(src[2]) * inv_l, __uint_as_float(src[3]) * inv_l);
          v.z = pack_bf16x2(__uint_as_float(src[4]) * inv_l, __uint_as_float(src[5]) * inv_l);
          v.w = pack_bf16x2(__uint_as_float(src[6]) * inv_l, __uint_as_float(src[7]) * inv_l);
          *reinterpret_cast<uint4*>(wst + lane * 128 + ((c ^ (lane & 7)) << 4)) = v;
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = i * 4 + (lane >> 3);  // row of the warp
          const int c = lane & 7;             // 16-byte chunk of its 128 bytes
          const uint4 v = *reinterpret_cast<const uint4*>(wst + r * 128 + ((c ^ (r & 7)) << 4));
          if (rbase + r < len)
            *reinterpret_cast<uint4*>(p.o + ((size_t)(start + rbase + r) * p.Hq + h) * D +
                                      pn * 64 + c * 8) = v;
        }
        __syncwarp();
      }
      if (valid && p.lse)
        p.lse[(size_t)h * p.T + grow] = (m_ref + __log2f(l_exact)) * 0.69314718055994531f;
      tc_fence_before();
    }
  }

  // ---------------- teardown ----------------
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace prefill
}  // namespace fa
