// debug_f32.cuh -- fp32 CUDA-core versions of prefill and paged decode.
//
// One thread per (query row, head) runs the online softmax of the pages
// ("gsyq.cn FA vs FIA" section 1: running row max m and normaliser l with
// rescaling) over every visible key in fp32 with the accurate expf.  Slow on
// purpose; they exist to check layouts, masks, GQA mapping, paging and LSE
// conventions at fp32 precision independently of the tensor-core kernels.
#pragma once

#include "ptx.cuh"

namespace fa {
namespace debug {

constexpr int MAX_D = 256;

__global__ void prefill_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                   const float* __restrict__ v, float* __restrict__ o,
                                   float* __restrict__ lse, const int32_t* __restrict__ cu,
                                   int B, int Hq, int Hkv, int d, int causal, float scale, int T) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)T * Hq) return;
  const int t = (int)(idx / Hq), h = (int)(idx % Hq);
  // sequence of token t (cu is validated here: a bad entry is a bounds error)
  int lo = 0, hi = B - 1, b = -1;
  while (lo <= hi) {
    const int mid = (lo + hi) >> 1;
    const int s = cu[mid], e = cu[mid + 1];
    if (t < s) hi = mid - 1;
    else if (t >= e) lo = mid + 1;
    else { b = mid; break; }
  }
  if (b < 0 || cu[b] < 0 || cu[b + 1] > T) {
    report_error(kDevErrBounds);
    return;
  }
  const int start = cu[b], len = cu[b + 1] - start, i = t - start;
  const int n = causal ? i + 1 : len;
  const int kh = h / (Hq / Hkv);
  const float* qr = q + ((size_t)t * Hq + h) * d;
  float acc[MAX_D];
  for (int c = 0; c < d; ++c) acc[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  for (int j = 0; j < n; ++j) {
    const float* kr = k + ((size_t)(start + j) * Hkv + kh) * d;
    float s = 0.f;
    for (int c = 0; c < d; ++c) s = fmaf(qr[c], kr[c], s);
    s *= scale;
    const float m_new = fmaxf(m, s);
    const float alpha = expf(m - m_new);
    const float pj = expf(s - m_new);
    l = l * alpha + pj;
    const float* vr = v + ((size_t)(start + j) * Hkv + kh) * d;
    for (int c = 0; c < d; ++c) acc[c] = fmaf(pj, vr[c], acc[c] * alpha);
    m = m_new;
  }
  float* orow = o + ((size_t)t * Hq + h) * d;
  for (int c = 0; c < d; ++c) orow[c] = n > 0 ? acc[c] / l : 0.f;
  if (lse) lse[(size_t)h * T + t] = n > 0 ? m + logf(l) : -INFINITY;
}

__global__ void decode_f32_kernel(const float* __restrict__ q, const float* __restrict__ kp,
                                  const float* __restrict__ vp, const int32_t* __restrict__ bt,
                                  const int32_t* __restrict__ seq_lens, int page_size,
                                  float* __restrict__ o, float* __restrict__ lse, int B, int Hq,
                                  int Hkv, int d, int max_blocks, int num_pages, float scale) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * Hq) return;
  const int b = idx / Hq, h = idx % Hq;
  const int kh = h / (Hq / Hkv);
  int n = seq_lens[b];
  if (n < 0 || n > max_blocks * page_size) {
    report_error(kDevErrBounds);
    n = 0;
  }
  const float* qr = q + (size_t)idx * d;
  float acc[MAX_D];
  for (int c = 0; c < d; ++c) acc[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  for (int t = 0; t < n; ++t) {
    const int page = bt[(size_t)b * max_blocks + t / page_size];
    if (page < 0 || page >= num_pages) {
      report_error(kDevErrBounds);
      continue;
    }
    const size_t row = (((size_t)page * page_size + t % page_size) * Hkv + kh) * d;
    float s = 0.f;
    for (int c = 0; c < d; ++c) s = fmaf(qr[c], kp[row + c], s);
    s *= scale;
    const float m_new = fmaxf(m, s);
    const float alpha = expf(m - m_new);
    const float pj = expf(s - m_new);
    l = l * alpha + pj;
    for (int c = 0; c < d; ++c) acc[c] = fmaf(pj, vp[row + c], acc[c] * alpha);
    m = m_new;
  }
  float* orow = o + (size_t)idx * d;
  for (int c = 0; c < d; ++c) orow[c] = l > 0.f ? acc[c] / l : 0.f;
  if (lse) lse[idx] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace debug
}  // namespace fa
