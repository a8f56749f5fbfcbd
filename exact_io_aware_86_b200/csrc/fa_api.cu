// fa_api.cu -- the C ABI declared in include/fa.h: host-side argument checks,
// TMA tensor maps, launch configuration, and the device error word.
//
// All kernels live in this one translation unit so they share the error
// word (ptx.cuh) without relocatable device code.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "fa.h"
#include "ptx.cuh"
#include "prefill_sm100.cuh"
#include "decode_sm100.cuh"
#include "debug_f32.cuh"
#include "append_rope.cuh"

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// --------------------------------------------------------------------------
// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library does not link libcuda directly (it loads on machines without a
// GPU driver; the symbol is resolved on first use).
// --------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tensor map with 128-byte swizzle (bf16 elements, or bytes for e4m3);
// dims/strides innermost first, strides in bytes for dims 1.. (dim 0 is
// contiguous).
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box, bool bytes = false) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(m, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        (cuuint32_t)rank,
                        const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms_current() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

float resolve_scale(float scale, int d) { return scale > 0.f ? scale : 1.0f / sqrtf((float)d); }

// max_seqlen <= 0 means "not given": every sequence is at most T long, and
// the work list can hold MAX_LEVELS * 256 rows per sequence.
int resolve_max_seqlen(int max_seqlen, int total_tokens) {
  if (max_seqlen > 0) return max_seqlen;
  return std::min<long long>(total_tokens,
                             (long long)fa::prefill::MAX_LEVELS * fa::prefill::ROWS_PER_ITEM);
}

// How the decode spreads the heads over a CTA's consumer warps: each warp
// takes one kv head and one tile of 8 of its Hq / Hkv query heads.  A CTA
// holds hpb kv heads (a divisor of Hkv) with qpw query tiles each, at most 8
// warps; a kv head with more than 8 tiles (more than 64 query heads) is
// split into nq chunks of 8 tiles, which are separate work items.
struct DecodeLayout {
  int hpb, qpw, nq;
};

DecodeLayout decode_layout(int Hq, int Hkv) {
  using namespace fa::decode;
  const int tiles = (Hq / Hkv + QTILE - 1) / QTILE;
  DecodeLayout L{1, tiles, 1};
  if (tiles > MAX_CONSUMERS) {
    L.qpw = MAX_CONSUMERS;
    L.nq = (tiles + MAX_CONSUMERS - 1) / MAX_CONSUMERS;
    return L;
  }
  for (int h = std::min(MAX_HPB, MAX_CONSUMERS / tiles); h >= 1; --h)
    if (Hkv % h == 0) {
      L.hpb = h;
      break;
    }
  return L;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int kMaxDevices = 64;

// Launches `kernel` with programmatic stream serialization: it may start
// while the stream's previous kernel drains, and must itself execute
// griddepcontrol.wait before it reads or writes global memory that kernel
// could touch.
template <typename... KArgs, typename... Args>
fa_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, int smem,
                     cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess ? FA_OK
                                                                                      : FA_ERR_CUDA;
}

// Launch set-up of one kernel: the dynamic shared-memory limit is an
// attribute of the kernel on a device, so it is set once per device (under a
// lock, as several host threads may launch on several devices), together
// with the register count the compiled kernel launches with.
struct KernelSetup {
  std::mutex mu;
  int state[kMaxDevices] = {};  // 0 not yet, 1 ready, -1 failed
  int regs[kMaxDevices] = {};
};

template <typename K>
bool setup_kernel(KernelSetup& ks, K kernel, int smem_bytes, int* regs = nullptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(ks.mu);
  if (ks.state[dev] == 0) {
    cudaFuncAttributes a;
    const bool ok = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem_bytes) == cudaSuccess &&
                    cudaFuncGetAttributes(&a, kernel) == cudaSuccess;
    ks.regs[dev] = ok ? a.numRegs : 0;
    ks.state[dev] = ok ? 1 : -1;
  }
  if (regs) *regs = ks.regs[dev];
  return ks.state[dev] == 1;
}

// Mask variants after normalisation: window bounds -1 (no limit) or in
// [0, max_seqlen), right bound 0 under the causal mask.
struct Variant {
  int wl = -1, wr = -1;
  float softcap = 0.f;
  const float* alibi = nullptr;
  int alibi_stride = 0;
  // anything beyond the plain causal (wr = 0) or full (wr = -1) mask
  bool general() const { return softcap > 0.f || alibi != nullptr || wl >= 0 || wr > 0; }
};

template <int D, bool GENERAL, bool FP8 = false, int LOGIT = 0>
fa_status launch_prefill(const void* q, const void* k, const void* v, void* o, float* lse,
                         const int32_t* cu, int B, int Hq, int Hkv, int causal, float scale,
                         cudaStream_t stream, int T, int max_seqlen, const Variant& var,
                         float qk_descale = 1.f, float v_descale = 1.f) {
  using namespace fa::prefill;
  using C = Cfg<D, FP8>;
  CUtensorMap tq, tk, tv;
  const cuuint32_t box[2] = {(cuuint32_t)C::PANEL_ELEMS, (cuuint32_t)BM};  // 128 B x 128 rows
  {
    const cuuint64_t dims[2] = {(cuuint64_t)Hq * D, (cuuint64_t)T};
    const cuuint64_t str[1] = {(cuuint64_t)Hq * D * C::ESIZE};
    if (!make_map(&tq, q, 2, dims, str, box, FP8)) return FA_ERR_CUDA;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)Hkv * D, (cuuint64_t)T};
    const cuuint64_t str[1] = {(cuuint64_t)Hkv * D * C::ESIZE};
    if (!make_map(&tk, k, 2, dims, str, box, FP8)) return FA_ERR_CUDA;
    if (!make_map(&tv, v, 2, dims, str, box, FP8)) return FA_ERR_CUDA;
  }
  Params p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.cu_seqlens = cu;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.group = Hq / Hkv;
  p.T = T;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = resolve_scale(scale, D) * qk_descale * kLog2e;
  p.o_scale = v_descale;
  p.num_levels = (max_seqlen + ROWS_PER_ITEM - 1) / ROWS_PER_ITEM;
  p.wl = var.wl;
  p.wr = var.wr;
  p.cap_out = var.softcap > 0.f ? var.softcap * kLog2e : 0.f;
  p.cap_in = var.softcap > 0.f ? 2.f * kLog2e * resolve_scale(scale, D) / var.softcap : 0.f;
  p.alibi = var.alibi;
  p.alibi_stride = var.alibi_stride;

  const int sms = num_sms_current();
  if (sms <= 0) return FA_ERR_CUDA;
  const long long upper = ((long long)T / ROWS_PER_ITEM + B) * Hq;  // >= number of work items
  long long grid = upper < sms ? upper : sms;
  if (grid < 1) grid = 1;
  if ((upper + grid - 1) / grid > MAX_ITEMS_PER_CTA) grid = (upper + MAX_ITEMS_PER_CTA - 1) / MAX_ITEMS_PER_CTA;
  if (grid > 0x7fffffff) return FA_ERR_UNSUPPORTED;

  const int smem = smem_bytes<D, FP8>();
  static KernelSetup setup;
  int launch_regs = 0;
  if (!setup_kernel(setup, prefill_kernel<D, GENERAL, FP8, LOGIT>, smem, &launch_regs)) return FA_ERR_CUDA;
  // The kernel hands registers between its warpgroups with setmaxnreg; the
  // split only fits if the launch allots kRegsLaunch registers per thread
  // (otherwise setmaxnreg.inc could never be satisfied).
  if (launch_regs < (int)kRegsLaunch) return FA_ERR_UNSUPPORTED;
  // (A programmatic dependent launch, to overlap the set-up with the
  // stream's previous kernel, measured no faster.)
  prefill_kernel<D, GENERAL, FP8, LOGIT><<<(unsigned)grid, NUM_THREADS, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Automatic page ranges for the decode: every range spans the same number of
// pages c.  The range count is planned as if every request had max_blocks
// pages; c is picked among the sizes that give r = 1..32 rounds of ranges
// per SM, maximising a simple model: (load balance of the last round) x
// (1 - the partial-output traffic relative to the K/V bytes - a fixed
// per-range cost), with ranges of at least 256 tokens.
int auto_chunk_pages(int B, int Hq, int Hkv, int max_blocks, int page_size, int num_sms) {
  const DecodeLayout L = decode_layout(Hq, Hkv);
  const int hpb = L.hpb;
  const long long ngroups = (long long)(Hkv / hpb) * L.nq;  // items per range
  const int G = num_sms > 0 ? num_sms : 148;
  const long long U = (long long)B * max_blocks * ngroups;
  const int c_min = std::min(max_blocks, std::max(1, ceil_div(256, page_size)));
  const double qpk = (double)Hq / Hkv;
  auto score = [&](int c) {
    const long long ranges = ceil_div(max_blocks, c);
    const long long items = (long long)B * ranges * ngroups;
    const double rounds = (double)items / G;
    const double bal = items >= G ? rounds / std::ceil(rounds) : rounds;
    // fp32 partial O and LSE, written and read once, per byte of K and V
    const double part = ranges > 1 ? 2.0 * qpk / ((double)c * page_size) : 0.0;
    // about 0.5 us of per-range work at ~40 GB/s per SM, per byte a range reads
    const double fixed = 20000.0 / ((double)c * page_size * hpb * 512.0);
    return bal * (1.0 - part - fixed);
  };
  int best_c = max_blocks;
  double best = score(max_blocks);
  for (int r = 1; r <= 32; ++r) {
    long long c = (U + (long long)r * G - 1) / ((long long)r * G);
    for (long long cc = c - 1; cc <= c + 1; ++cc) {
      const int ci = (int)std::max<long long>(c_min, std::min<long long>(cc, max_blocks));
      const double sc = score(ci);
      if (sc > best + 1e-9) {
        best = sc;
        best_c = ci;
      }
    }
  }
  return best_c;
}


template <int D>
fa_status launch_decode(const void* q, const void* kp, const void* vp, const int32_t* bt,
                        const int32_t* sl, int page_size, int num_splits, void* o,
                        cudaStream_t stream, int B, int Hq, int Hkv, int max_blocks, int num_pages,
                        float scale, float* lse, void* ws) {
  using namespace fa::decode;
  const DecodeLayout L = decode_layout(Hq, Hkv);
  const int sms = num_sms_current();
  if (sms <= 0) return FA_ERR_CUDA;
  Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_pages = static_cast<const __nv_bfloat16*>(kp);
  p.v_pages = static_cast<const __nv_bfloat16*>(vp);
  p.block_table = bt;
  p.seq_lens = sl;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.group = Hq / Hkv;
  p.hpb = L.hpb;
  p.qpw = L.qpw;
  p.nq = L.nq;
  p.ngroups = Hkv / L.hpb;
  p.page_size = page_size;
  p.max_blocks = max_blocks;
  p.num_pages = num_pages;
  if (num_splits == 0) {
    p.chunk_pages = auto_chunk_pages(B, Hq, Hkv, max_blocks, page_size, sms);
    p.s_max = ceil_div(max_blocks, p.chunk_pages);
  } else {
    p.chunk_pages = 0;
    p.s_max = num_splits;
  }
  p.half_bytes = Cfg<D>::PANELS * L.hpb * BOX_BYTES;
  p.stages = std::min(MAX_STAGES, STAGE_BUDGET / stage_bytes(p.half_bytes));
  p.tma_gather = page_size % TOK == 0 ? 1 : 0;
  p.scale_log2 = resolve_scale(scale, D) * kLog2e;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  const bool split = p.s_max > 1;
  p.local_plan = split && B <= PLAN_MAX_B ? 1 : 0;
  const size_t opart_bytes = round_up((size_t)B * Hq * p.s_max * D * sizeof(float), 256);
  const size_t lpart_bytes = round_up((size_t)B * Hq * p.s_max * sizeof(float), 256);
  p.o_part = split ? static_cast<float*>(ws) : nullptr;
  p.lse_part = split ? reinterpret_cast<float*>(static_cast<char*>(ws) + opart_bytes) : nullptr;
  int32_t* prefix = split && !p.local_plan
                        ? reinterpret_cast<int32_t*>(static_cast<char*>(ws) + opart_bytes + lpart_bytes)
                        : nullptr;
  p.split_prefix = prefix;
  const long long items = (split ? (long long)B * p.s_max : (long long)B) * p.ngroups * p.nq;
  if (items > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;

  CUtensorMap tk, tv;
  std::memset(&tk, 0, sizeof(tk));
  std::memset(&tv, 0, sizeof(tv));
  if (p.tma_gather) {
    // dimensions (head_dim, token, kv head): a box of the CTA's heads lands in
    // shared memory as [head][token][64 dims] (see decode_sm100.cuh).  An
    // empty pool is mapped as one page, which no copy reads (every page index
    // is then out of range and fetched as zeros).
    const cuuint64_t dims[3] = {(cuuint64_t)D,
                                (cuuint64_t)std::max(num_pages, 1) * (cuuint64_t)page_size,
                                (cuuint64_t)Hkv};
    const cuuint64_t str[2] = {(cuuint64_t)Hkv * D * 2, (cuuint64_t)D * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)TOK, (cuuint32_t)L.hpb};
    if (!make_map(&tk, kp, 3, dims, str, box)) return FA_ERR_CUDA;
    if (!make_map(&tv, vp, 3, dims, str, box)) return FA_ERR_CUDA;
  }

  if (prefix) {
    plan_kernel<<<1, 1024, 0, stream>>>(p, prefix);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  static KernelSetup setup;
  if (!setup_kernel(setup, split_kernel<D>, SMEM_LIMIT)) return FA_ERR_CUDA;
  const int smem = split_smem_bytes(p);
  const int grid = (int)std::min<long long>(items, sms);
  if (grid > 0) {
    split_kernel<D><<<grid, (L.hpb * L.qpw + 1) * 32, smem, stream>>>(tk, tv, p);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  if (split) {
    // a programmatic dependent of the split kernel: its CTAs are scheduled
    // while the split kernel drains and wait for it to complete
    const fa_status st = launch_pdl(combine_kernel<D>, dim3((unsigned)(B * Hq)),
                                    dim3(COMBINE_WARPS * 32), 0, stream, p);
    if (st != FA_OK) return st;
  }
  return FA_OK;
}

}  // namespace

extern "C" {

fa_status fa_prefill_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                        const int32_t* cu_seqlens, int B, int Hq, int Hkv, int d, int causal,
                        float scale, fa_stream_t stream, int total_tokens, int max_seqlen,
                        int window_left, int window_right, float softcap,
                        const float* alibi_slopes, int alibi_batch_stride) {
  if (!q || !k || !v || !o || !cu_seqlens) return FA_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || total_tokens < 0)
    return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(cu_seqlens, 4) || (lse && !aligned(lse, 4)) ||
      (alibi_slopes && !aligned(alibi_slopes, 4)))
    return FA_ERR_INVALID_ARG;
  max_seqlen = resolve_max_seqlen(max_seqlen, total_tokens);
  if (!(softcap >= 0.f) || std::isinf(softcap) || alibi_batch_stride < 0)
    return FA_ERR_INVALID_ARG;
  Variant var;
  // a bound at least max_seqlen can never cut a sequence: no limit
  var.wl = (window_left < 0 || window_left >= max_seqlen) ? -1 : window_left;
  var.wr = causal ? 0 : ((window_right < 0 || window_right >= max_seqlen) ? -1 : window_right);
  if (var.wr == 0) causal = 1;  // a right bound of 0 is the causal mask
  var.softcap = softcap;
  var.alibi = alibi_slopes;
  var.alibi_stride = alibi_slopes ? alibi_batch_stride : 0;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (Hq > 0xFFFF) return FA_ERR_UNSUPPORTED;
  if ((long long)(max_seqlen + fa::prefill::ROWS_PER_ITEM - 1) / fa::prefill::ROWS_PER_ITEM >
      fa::prefill::MAX_LEVELS)
    return FA_ERR_UNSUPPORTED;
  if (B == 0 || total_tokens == 0 || max_seqlen == 0) return FA_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // five kernels per head size: plain causal / full; a band mask alone;
  // causal ALiBi (no softcap), whose penalty is linear in the key; softcap
  // without ALiBi, capped inside the exponential loop; and softcap with
  // ALiBi, or ALiBi under a right bound other than 0, rewriting every score
  const bool gen = var.general();
  const bool cap = var.softcap > 0.f, alibi = var.alibi != nullptr;
  const int logit = cap ? (alibi ? 1 : 3) : (alibi ? (var.wr == 0 ? 2 : 1) : 0);
  if (d == 64) {
    if (!gen)
      return launch_prefill<64, false>(q, k, v, o, lse, cu_seqlens, B, Hq, Hkv, causal, scale, s,
                                       total_tokens, max_seqlen, var);
    if (logit == 1)
      return launch_prefill<64, true, false, 1>(q, k, v, o, lse, cu_seqlens, B, Hq, Hkv, causal,
                                                scale, s, total_tokens, max_seqlen, var);
    if (logit == 3)
      return launch_prefill<64, true, false, 3>(q, k, v, o, lse, cu_seqlens, B, Hq, Hkv, causal,
                                                scale, s, total_tokens, max_seqlen, var);
    if (logit == 2)
      return launch_prefill<64, true, false, 2>(q, k, v, o, lse, cu_seqlens, B, Hq, Hkv, causal,
                                                scale, s, total_tokens, max_seqlen, var);
    return launch_prefill<64, true>(q, k, v, o, lse, cu_seqlens, B, Hq, Hkv, causal, scale, s,
                                    total_tokens, max_seqlen, var);
  }
  if (!gen)
    return launch_prefill<128, false>(q, k, v, o, lse, cu_seqlens, B, Hq, Hkv, causal, scale, s,
                                      total_tokens, max_seqlen, var);
  if (logit == 1)
    return launch_prefill<128, true, false, 1>(q, k, v, o, lse, cu_seqlens, B, Hq, Hkv, causal,
                                               scale, s, total_tokens, max_seqlen, var);
  if (logit == 3)
    return launch_prefill<128, true, false, 3>(q, k, v, o, lse, cu_seqlens, B, Hq, Hkv, causal,
                                              scale, s, total_tokens, max_seqlen, var);
  if (logit == 2)
    return launch_prefill<128, true, false, 2>(q, k, v, o, lse, cu_seqlens, B, Hq, Hkv, causal,
                                               scale, s, total_tokens, max_seqlen, var);
  return launch_prefill<128, true>(q, k, v, o, lse, cu_seqlens, B, Hq, Hkv, causal, scale, s,
                                   total_tokens, max_seqlen, var);
}

fa_status fa_prefill_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                         const int32_t* cu_seqlens, int B, int Hq, int Hkv, int d, int causal,
                         float scale, float q_descale, float k_descale, float v_descale,
                         fa_stream_t stream, int total_tokens, int max_seqlen) {
  if (!q || !k || !v || !o || !cu_seqlens) return FA_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || total_tokens < 0)
    return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(cu_seqlens, 4) || (lse && !aligned(lse, 4)))
    return FA_ERR_INVALID_ARG;
  max_seqlen = resolve_max_seqlen(max_seqlen, total_tokens);
  for (float x : {q_descale, k_descale, v_descale})
    if (!(x > 0.f) || std::isinf(x)) return FA_ERR_INVALID_ARG;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (Hq > 0xFFFF) return FA_ERR_UNSUPPORTED;
  if ((long long)(max_seqlen + fa::prefill::ROWS_PER_ITEM - 1) / fa::prefill::ROWS_PER_ITEM >
      fa::prefill::MAX_LEVELS)
    return FA_ERR_UNSUPPORTED;
  if (B == 0 || total_tokens == 0 || max_seqlen == 0) return FA_OK;
  Variant var;
  var.wr = causal ? 0 : -1;
  return launch_prefill<128, false, true>(q, k, v, o, lse, cu_seqlens, B, Hq, Hkv, causal, scale,
                                          reinterpret_cast<cudaStream_t>(stream), total_tokens,
                                          max_seqlen, var, q_descale * k_descale, v_descale);
}

fa_status fa_prefill(const void* q, const void* k, const void* v, void* o, float* lse,
                     const int32_t* cu_seqlens, int B, int Hq, int Hkv, int d, int causal,
                     float scale, fa_stream_t stream, int total_tokens, int max_seqlen) {
  return fa_prefill_ex(q, k, v, o, lse, cu_seqlens, B, Hq, Hkv, d, causal, scale, stream,
                       total_tokens, max_seqlen, -1, -1, 0.f, nullptr, 0);
}

size_t fa_decode_workspace_size(int B, int Hq, int d, int num_splits) {
  if (B <= 0 || Hq <= 0 || d <= 0 || num_splits <= 1) return 0;
  const size_t o_part = round_up((size_t)B * Hq * num_splits * d * sizeof(float), 256);
  const size_t l_part = round_up((size_t)B * Hq * num_splits * sizeof(float), 256);
  const size_t prefix = round_up((size_t)(B + 1) * sizeof(int32_t), 256);
  return o_part + l_part + prefix;
}

int fa_decode_auto_splits(int B, int Hq, int Hkv, int max_blocks_per_seq, int page_size,
                          int num_sms) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || max_blocks_per_seq <= 0 ||
      page_size <= 0)
    return 1;
  if (num_sms <= 0) num_sms = num_sms_current();
  if (num_sms <= 0) num_sms = 148;
  const int c = auto_chunk_pages(B, Hq, Hkv, max_blocks_per_seq, page_size, num_sms);
  return ceil_div(max_blocks_per_seq, c);
}

fa_status fa_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                          const int32_t* block_table, const int32_t* seq_lens, int page_size,
                          int num_splits, void* o, fa_stream_t stream, int B, int Hq, int Hkv,
                          int d, int max_blocks_per_seq, int num_pages, float scale, float* lse,
                          void* workspace, size_t workspace_bytes) {
  if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !o) return FA_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || page_size < 1 || num_splits < 0 ||
      max_blocks_per_seq < 1 || num_pages < 0)
    return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(o, 16) ||
      !aligned(block_table, 4) || !aligned(seq_lens, 4) || (lse && !aligned(lse, 4)) ||
      (workspace && !aligned(workspace, 256)))
    return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if ((long long)num_pages * page_size > 0x7fffffffLL ||
      (long long)max_blocks_per_seq * page_size > 0x7fffffffLL)
    return FA_ERR_UNSUPPORTED;
  if ((long long)B * Hq > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  if (B == 0) return FA_OK;
  const int S = num_splits == 0
                    ? fa_decode_auto_splits(B, Hq, Hkv, max_blocks_per_seq, page_size, 0)
                    : num_splits;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t need = fa_decode_workspace_size(B, Hq, d, S);
  void* ws = workspace;
  bool owned = false;
  if (need > 0) {
    if (ws) {
      if (workspace_bytes < need) return FA_ERR_INVALID_ARG;
    } else {
      if (cudaMallocAsync(&ws, need, s) != cudaSuccess) return FA_ERR_CUDA;
      owned = true;
    }
  }
  fa_status st;
  if (d == 64)
    st = launch_decode<64>(q, k_pages, v_pages, block_table, seq_lens, page_size, num_splits, o, s,
                           B, Hq, Hkv, max_blocks_per_seq, num_pages, scale, lse, ws);
  else
    st = launch_decode<128>(q, k_pages, v_pages, block_table, seq_lens, page_size, num_splits, o,
                            s, B, Hq, Hkv, max_blocks_per_seq, num_pages, scale, lse, ws);
  if (owned && cudaFreeAsync(ws, s) != cudaSuccess && st == FA_OK) st = FA_ERR_CUDA;
  return st;
}

size_t fa_decode_append_workspace_size(int B, int Hq, int d, int num_splits) {
  if (B <= 0 || Hq <= 0 || d <= 0) return 0;
  return round_up((size_t)B * Hq * d * 2, 256) + round_up((size_t)B * 4, 256) +
         fa_decode_workspace_size(B, Hq, d, num_splits);
}

fa_status fa_decode_paged_append(const void* q, const void* k_new, const void* v_new,
                                 void* k_pages, void* v_pages, const int32_t* block_table,
                                 const int32_t* cache_seqlens, int page_size, int num_splits,
                                 void* o, fa_stream_t stream, int B, int Hq, int Hkv, int d,
                                 int max_blocks_per_seq, int num_pages, float scale, float* lse,
                                 const float* rotary_cos, const float* rotary_sin,
                                 int rotary_max_pos, int rotary_dim, int rotary_interleaved,
                                 void* workspace, size_t workspace_bytes) {
  if (!q || !k_new || !v_new || !k_pages || !v_pages || !block_table || !cache_seqlens || !o)
    return FA_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || page_size < 1 || num_splits < 0 ||
      max_blocks_per_seq < 1 || num_pages < 0)
    return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_pages, 16) ||
      !aligned(v_pages, 16) || !aligned(o, 16) || !aligned(block_table, 4) ||
      !aligned(cache_seqlens, 4) || (lse && !aligned(lse, 4)) ||
      (workspace && !aligned(workspace, 256)))
    return FA_ERR_INVALID_ARG;
  if ((rotary_cos == nullptr) != (rotary_sin == nullptr)) return FA_ERR_INVALID_ARG;
  if (rotary_cos && (rotary_dim < 2 || rotary_dim > d || rotary_dim % 2 != 0 ||
                     rotary_max_pos < 1 || !aligned(rotary_cos, 4) || !aligned(rotary_sin, 4)))
    return FA_ERR_INVALID_ARG;
  // the attention step has the limits of fa_decode_paged
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if ((long long)num_pages * page_size > 0x7fffffffLL ||
      (long long)max_blocks_per_seq * page_size > 0x7fffffffLL)
    return FA_ERR_UNSUPPORTED;
  if ((long long)B * Hq > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  if (B == 0) return FA_OK;
  const int S = num_splits == 0
                    ? fa_decode_auto_splits(B, Hq, Hkv, max_blocks_per_seq, page_size, 0)
                    : num_splits;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t q_bytes = round_up((size_t)B * Hq * d * 2, 256);
  const size_t l_bytes = round_up((size_t)B * 4, 256);
  const size_t need = fa_decode_append_workspace_size(B, Hq, d, S);
  void* ws = workspace;
  bool owned = false;
  if (ws) {
    if (workspace_bytes < need) return FA_ERR_INVALID_ARG;
  } else {
    if (cudaMallocAsync(&ws, need, s) != cudaSuccess) return FA_ERR_CUDA;
    owned = true;
  }
  uint8_t* w = static_cast<uint8_t*>(ws);
  fa::append::Params ap;
  ap.q = static_cast<const __nv_bfloat16*>(q);
  ap.k_new = static_cast<const __nv_bfloat16*>(k_new);
  ap.v_new = static_cast<const __nv_bfloat16*>(v_new);
  ap.k_pages = static_cast<__nv_bfloat16*>(k_pages);
  ap.v_pages = static_cast<__nv_bfloat16*>(v_pages);
  ap.block_table = block_table;
  ap.cache_seqlens = cache_seqlens;
  ap.cos = rotary_cos;
  ap.sin = rotary_sin;
  ap.q_rot = reinterpret_cast<__nv_bfloat16*>(w);
  ap.seq_lens_new = reinterpret_cast<int32_t*>(w + q_bytes);
  ap.B = B;
  ap.Hq = Hq;
  ap.Hkv = Hkv;
  ap.d = d;
  ap.page_size = page_size;
  ap.max_blocks = max_blocks_per_seq;
  ap.num_pages = num_pages;
  ap.max_pos = rotary_cos ? rotary_max_pos : 0;
  ap.rd = rotary_cos ? rotary_dim : 0;
  ap.interleaved = rotary_interleaved ? 1 : 0;
  fa::append::append_rope_kernel<<<B, fa::append::THREADS, 0, s>>>(ap);
  fa_status st = cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
  if (st == FA_OK) {
    void* dws = (need > q_bytes + l_bytes) ? static_cast<void*>(w + q_bytes + l_bytes) : nullptr;
    if (d == 64)
      st = launch_decode<64>(ap.q_rot, k_pages, v_pages, block_table, ap.seq_lens_new, page_size,
                             num_splits, o, s, B, Hq, Hkv, max_blocks_per_seq, num_pages, scale,
                             lse, dws);
    else
      st = launch_decode<128>(ap.q_rot, k_pages, v_pages, block_table, ap.seq_lens_new,
                              page_size, num_splits, o, s, B, Hq, Hkv, max_blocks_per_seq,
                              num_pages, scale, lse, dws);
  }
  if (owned && cudaFreeAsync(ws, s) != cudaSuccess && st == FA_OK) st = FA_ERR_CUDA;
  return st;
}

fa_status fa_prefill_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                         const int32_t* cu_seqlens, int B, int Hq, int Hkv, int d, int causal,
                         float scale, fa_stream_t stream, int total_tokens, int max_seqlen) {
  (void)max_seqlen;
  if (!q || !k || !v || !o || !cu_seqlens) return FA_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || total_tokens < 0 || d < 1)
    return FA_ERR_INVALID_ARG;
  if (d > fa::debug::MAX_D) return FA_ERR_UNSUPPORTED;
  if (B == 0 || total_tokens == 0) return FA_OK;
  const long long n = (long long)total_tokens * Hq;
  const long long blocks = (n + 127) / 128;
  if (blocks > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  fa::debug::prefill_f32_kernel<<<(unsigned)blocks, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      q, k, v, o, lse, cu_seqlens, B, Hq, Hkv, d, causal ? 1 : 0, resolve_scale(scale, d),
      total_tokens);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_decode_paged_f32(const float* q, const float* k_pages, const float* v_pages,
                              const int32_t* block_table, const int32_t* seq_lens, int page_size,
                              float* o, fa_stream_t stream, int B, int Hq, int Hkv, int d,
                              int max_blocks_per_seq, int num_pages, float scale, float* lse) {
  if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !o) return FA_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || page_size < 1 || max_blocks_per_seq < 1 ||
      num_pages < 0 || d < 1)
    return FA_ERR_INVALID_ARG;
  if (d > fa::debug::MAX_D) return FA_ERR_UNSUPPORTED;
  if (B == 0) return FA_OK;
  const long long n = (long long)B * Hq;
  fa::debug::decode_f32_kernel<<<(unsigned)((n + 127) / 128), 128, 0,
                                 reinterpret_cast<cudaStream_t>(stream)>>>(
      q, k_pages, v_pages, block_table, seq_lens, page_size, o, lse, B, Hq, Hkv, d,
      max_blocks_per_seq, num_pages, resolve_scale(scale, d));
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_get_device_error(fa_stream_t stream, int* code) {
  if (!code) return FA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_device_error, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(fa::g_device_error, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (v & fa::kDevErrTimeout) *code = FA_ERR_DEVICE_TIMEOUT;
  else if (v & fa::kDevErrBounds) *code = FA_ERR_DEVICE_BOUNDS;
  else *code = FA_OK;
  return FA_OK;
}

const char* fa_get_error_string(fa_status status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration";
    case FA_ERR_CUDA: return "CUDA runtime or launch error";
    case FA_ERR_DEVICE_BOUNDS: return "device-side index out of range";
    case FA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

int fa_version(void) { return 100; }

}  // extern "C"

// --------------------------------------------------------------------------
// Self-test hook: the scalar functions the prefill kernel computes the
// softmax weights with, evaluated element by element on the GPU so a test
// can compare them with an exact reference over their whole input range.
// --------------------------------------------------------------------------
namespace fa {
namespace selftest {

__global__ void math_kernel(int op, const float* __restrict__ x, float* __restrict__ y, int n,
                            float a, float b) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const bool two = i + 1 < n;
  const float x0 = x[i], x1 = two ? x[i + 1] : 0.f;
  float y0 = 0.f, y1 = 0.f;
  if (op == FA_MATH_EXP2_FMA) {
    f2_unpack(exp2_fma_pair(f2_pack(x0, x1)), y0, y1);
  } else if (op == FA_MATH_EXP2_MUFU) {
    y0 = ex2(x0);
    y1 = ex2(x1);
  } else {
    y0 = softcap_log2(x0, a, b);
    y1 = softcap_log2(x1, a, b);
  }
  y[i] = y0;
  if (two) y[i + 1] = y1;
}

}  // namespace selftest
}  // namespace fa

extern "C" fa_status fa_selftest_inject_stall(int which, unsigned long long wait_limit_ns) {
  if (which != 0 && which != FA_STALL_PREFILL && which != FA_STALL_DECODE) return FA_ERR_INVALID_ARG;
  const unsigned long long limit = wait_limit_ns ? wait_limit_ns : fa::kWaitLimitNs;
  if (cudaMemcpyToSymbol(fa::g_stall_test, &which, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(fa::g_wait_limit_ns, &limit, sizeof(limit)) != cudaSuccess)
    return FA_ERR_CUDA;
  return FA_OK;
}

extern "C" fa_status fa_selftest_math(int op, const float* x, float* y, int n, float a, float b,
                                      fa_stream_t stream) {
  if (op != FA_MATH_EXP2_FMA && op != FA_MATH_EXP2_MUFU && op != FA_MATH_SOFTCAP_LOG2)
    return FA_ERR_INVALID_ARG;
  if (n < 0 || (n > 0 && (!x || !y)) || !aligned(x, 4) || !aligned(y, 4)) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  const int pairs = (n + 1) / 2;
  fa::selftest::math_kernel<<<(pairs + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      op, x, y, n, a, b);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// --------------------------------------------------------------------------
// Paged decode without any allocation (fa_decode_paged_noalloc).
//
// Some callers cannot allocate device memory at the point where they run a
// decode step: a serving engine that has already handed nearly all of HBM to
// its KV-cache pool, or a step loop that must not block in, or fail inside,
// the allocator once it is running.  This entry point takes its split
// scratch from a fixed array compiled into the library instead.  Every GPU
// that loads the library holds the array until the process exits.
// --------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB per device

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

// Device address of g_decode_scratch on the current device.  The first call
// on each device looks it up (cudaGetSymbolAddress with that device current)
// and caches it; later calls only read the cache.
void* decode_scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) return nullptr;
    addr[dev] = ptr;
  }
  return addr[dev];
}

}  // namespace

extern "C" fa_status fa_decode_paged_noalloc(const void* q, const void* k_pages,
                                             const void* v_pages, const int32_t* block_table,
                                             const int32_t* seq_lens, int page_size,
                                             int num_splits, void* o, fa_stream_t stream, int B,
                                             int Hq, int Hkv, int d, int max_blocks_per_seq,
                                             int num_pages, float scale, float* lse) {
  if (num_splits < 0 || B < 0 || Hq <= 0 || d <= 0) return FA_ERR_INVALID_ARG;
  const int S = num_splits == 0
                    ? fa_decode_auto_splits(B, Hq, Hkv, max_blocks_per_seq, page_size, 0)
                    : num_splits;
  const size_t need = fa_decode_workspace_size(B, Hq, d, S);
  if (need > kNoAllocScratchBytes) return FA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (need > 0) {
    scratch = decode_scratch_on_current_device();
    if (!scratch) return FA_ERR_CUDA;
  }
  // num_splits is passed on unchanged, so 0 keeps the automatic page ranges
  return fa_decode_paged(q, k_pages, v_pages, block_table, seq_lens, page_size, num_splits, o,
                         stream, B, Hq, Hkv, d, max_blocks_per_seq, num_pages, scale, lse, scratch,
                         need > 0 ? kNoAllocScratchBytes : 0);
}
