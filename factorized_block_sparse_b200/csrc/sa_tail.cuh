// Column part of the strided pattern for a partial last row.
//
// When N is not a multiple of l the 2-D view of the sequence ("OpenAI Sparse
// Transformer", "Factorized Attention Patterns": the column part attends to
// the positions a whole number of rows l back) has R = N / l whole rows and a
// partial last row of r = N - R l positions.  The tensor-core passes of the
// column view cover the whole rows; a position p = R l + c of the partial row
// (c < r) attends, besides its natural window, to the R earlier positions of
// its column, c + m l for m < R, and it is itself the key of no later
// position.  These r queries per head are few (fewer than l), so they run on
// CUDA cores: one warp per query, D / 32 elements per lane, an online
// softmax over the R keys.
//
// Forward: writes (o, lse) of the partial row's column part, which the
// natural-view pass then merges exactly like the column view's result.
// Backward (after the column view's pass, before the natural view's): adds
// the partial row's contributions to dQ (fp32 accumulator) and to the column
// view's fp32 dK / dV partials of the R keys of its column (each such key
// has exactly one partial-row query, so the adds do not race).
#pragma once

#include "sa_device.cuh"

namespace sa {

template <int D>
__device__ __forceinline__ void tail_load(const __nv_bfloat16* row, int lane, float* x) {
  constexpr int E = D / 32;
  if constexpr (E == 1) {
    x[0] = __bfloat162float(row[lane]);
  } else if constexpr (E == 2) {
    const float2 f = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(row)[lane]);
    x[0] = f.x;
    x[1] = f.y;
  } else {
    const uint2 u = reinterpret_cast<const uint2*>(row)[lane];
    const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    x[0] = f0.x;
    x[1] = f0.y;
    x[2] = f1.x;
    x[3] = f1.y;
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) v += __shfl_xor_sync(0xffffffffu, v, w);
  return v;
}

template <int D>
__global__ void __launch_bounds__(128) sa_tail_fwd_kernel(const __nv_bfloat16* __restrict__ q,
                                                          const __nv_bfloat16* __restrict__ k,
                                                          const __nv_bfloat16* __restrict__ v,
                                                          __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                                                          int BH, int N, int l, int R, float scale_log2) {
  pdl_wait();
  pdl_trigger();
  constexpr int E = D / 32;
  const int r = N - R * l;
  const long long w = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (w >= static_cast<long long>(BH) * r) return;
  const int lane = threadIdx.x & 31;
  const long long bh = w / r;
  const int p = R * l + static_cast<int>(w - bh * r);
  const size_t base = static_cast<size_t>(bh) * N * D;
  float qv[E], acc[E];
  tail_load<D>(q + base + static_cast<size_t>(p) * D, lane, qv);
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qv[e] *= scale_log2;  // scores in the exp2 domain
    acc[e] = 0.f;
  }
  float m = -INFINITY, sum = 0.f;
  for (int j = p - R * l; j < p; j += l) {  // the earlier positions of the column
    float kv[E], vv[E];
    tail_load<D>(k + base + static_cast<size_t>(j) * D, lane, kv);
    tail_load<D>(v + base + static_cast<size_t>(j) * D, lane, vv);
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) part = fmaf(qv[e], kv[e], part);
    const float s = warp_sum(part);
    const float m_new = fmaxf(m, s);
    const float corr = ex2(m - m_new);
    const float pj = ex2(s - m_new);
    sum = sum * corr + pj;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = fmaf(acc[e], corr, pj * vv[e]);
    m = m_new;
  }
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  __nv_bfloat16* orow = o + base + static_cast<size_t>(p) * D;
#pragma unroll
  for (int e = 0; e < E; ++e) orow[lane * E + e] = __float2bfloat16_rn(acc[e] * inv);
  if (lane == 0) lse[bh * N + p] = sum > 0.f ? (m + lg2(sum)) * 0.6931471805599453f : -INFINITY;
}

// ld: the packed [n_pad / 64][2][64] blocks of -lse * log2(e) and -Delta in
// natural order (written by the backward preprocess).
template <int D>
__global__ void __launch_bounds__(128) sa_tail_bwd_kernel(const __nv_bfloat16* __restrict__ q,
                                                          const __nv_bfloat16* __restrict__ k,
                                                          const __nv_bfloat16* __restrict__ v,
                                                          const __nv_bfloat16* __restrict__ dO,
                                                          const float* __restrict__ ld, float* __restrict__ dq_acc,
                                                          float* __restrict__ dk_part, float* __restrict__ dv_part,
                                                          int BH, int N, int l, int R, int n_pad, float scale,
                                                          float scale_log2) {
  pdl_wait();
  pdl_trigger();
  constexpr int E = D / 32;
  const int r = N - R * l;
  const long long w = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (w >= static_cast<long long>(BH) * r) return;
  const int lane = threadIdx.x & 31;
  const long long bh = w / r;
  const int p = R * l + static_cast<int>(w - bh * r);
  const size_t base = static_cast<size_t>(bh) * N * D;
  const float* ldb = ld + bh * n_pad * 2 + (p / 64) * 128 + (p % 64);
  const float nlse = ldb[0], ndel = ldb[64];
  float qv[E], dov[E], gq[E];
  tail_load<D>(q + base + static_cast<size_t>(p) * D, lane, qv);
  tail_load<D>(dO + base + static_cast<size_t>(p) * D, lane, dov);
#pragma unroll
  for (int e = 0; e < E; ++e) gq[e] = 0.f;
  for (int j = p - R * l; j < p; j += l) {
    float kv[E], vv[E];
    tail_load<D>(k + base + static_cast<size_t>(j) * D, lane, kv);
    tail_load<D>(v + base + static_cast<size_t>(j) * D, lane, vv);
    float ps = 0.f, pd = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      ps = fmaf(qv[e], kv[e], ps);
      pd = fmaf(dov[e], vv[e], pd);
    }
    const float s = warp_sum(ps), dp = warp_sum(pd);
    const float pj = ex2(fmaf(s, scale_log2, nlse));  // P = exp(S - lse)
    const float ds = pj * (dp + ndel);                 // dS = P (dP - Delta)
    float* dkr = dk_part + base + static_cast<size_t>(j) * D + lane * E;
    float* dvr = dv_part + base + static_cast<size_t>(j) * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      gq[e] = fmaf(ds, kv[e], gq[e]);
      dkr[e] += scale * ds * qv[e];
      dvr[e] += pj * dov[e];
    }
  }
  float* dqr = dq_acc + base + static_cast<size_t>(p) * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; ++e) dqr[e] += scale * gq[e];
}

}  // namespace sa
