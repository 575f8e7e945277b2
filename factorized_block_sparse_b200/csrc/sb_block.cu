// The Sparse Transformer block around the attention op: layer norms, the
// GELU feed-forward, the residual stream and the head layout in CUDA kernels
// of this file, the projections as cuBLAS GEMMs (bf16 in, fp32 accumulation;
// cuBLASLt where the residual input and the output differ) and the attention
// through libsparse_attn's C ABI.
//
// The block ("[논문 리뷰] Generating Long Sequences with Sparse Transformers",
// "제안 방법", third and fourth items; pcnews translation, "Глубокое
// внимание"): pre-activation residual sub-blocks with layer normalisation,
// recomputed in the backward pass from the block input.  Formulas and
// readings: include/sparse_block.h.
//
// Data layout: activations [M = B*N rows][C = H*D] bf16 row-major; the
// attention's q, k, v, o in its own [B, H, N, D] layout (head h = columns
// h*D .. h*D+D-1 of a C-wide row), converted by to_heads / from_heads.
#include <cublasLt.h>
#include <cublas_v2.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "sparse_block.h"

namespace sb {

constexpr float kEps = 1e-5f;
constexpr int kMaxC = 6144;  // model width limit (the layer-norm backward's 4 warps x 2 C float sums, 192 KiB)

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) v += __shfl_xor_sync(0xffffffffu, v, w);
  return v;
}

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* f) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* f) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}

// A C-wide bf16 row as seen by one lane: chunks of 8 consecutive channels at
// lane*8 + 256 j.  NCH > 0: the row is held in registers (C <= 256 NCH);
// NCH == 0: any C, the row is read again for each pass.
template <int NCH>
struct Row {
  float v[NCH > 0 ? NCH * 8 : 1];
};

template <int NCH>
__device__ __forceinline__ void row_load(Row<NCH>& r, const __nv_bfloat16* p, int C, int lane) {
  if constexpr (NCH > 0) {
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
      const int i = lane * 8 + 256 * j;
      if (i < C) load8(p + i, r.v + 8 * j);
      else
#pragma unroll
        for (int u = 0; u < 8; ++u) r.v[8 * j + u] = 0.f;
    }
  }
}

// Mean and 1/sqrt(var + eps) of the row (the deviations summed about the mean).
template <int NCH>
__device__ __forceinline__ void row_stats(const Row<NCH>& r, const __nv_bfloat16* xr, int C, int lane, float& mean,
                                          float& rstd) {
  float s = 0.f;
  if constexpr (NCH > 0) {
#pragma unroll
    for (int k = 0; k < NCH * 8; ++k) s += r.v[k];
  } else {
    for (int i = lane * 8; i < C; i += 256) {
      float f[8];
      load8(xr + i, f);
#pragma unroll
      for (int u = 0; u < 8; ++u) s += f[u];
    }
  }
  mean = warp_sum(s) / C;
  float v = 0.f;
  if constexpr (NCH > 0) {
#pragma unroll
    for (int j = 0; j < NCH; ++j)
      if (lane * 8 + 256 * j < C)
#pragma unroll
        for (int u = 0; u < 8; ++u) v += (r.v[8 * j + u] - mean) * (r.v[8 * j + u] - mean);
  } else {
    for (int i = lane * 8; i < C; i += 256) {
      float f[8];
      load8(xr + i, f);
#pragma unroll
      for (int u = 0; u < 8; ++u) v += (f[u] - mean) * (f[u] - mean);
    }
  }
  rstd = rsqrtf(warp_sum(v) / C + kEps);
}

// body(i, j, f) for each of the lane's chunks of the row (first channel i,
// chunk j, the 8 values f), from registers (unrolled) or read again.
template <int NCH, typename Body>
__device__ __forceinline__ void for_chunks(const Row<NCH>& r, const __nv_bfloat16* p, int C, int lane, Body body) {
  if constexpr (NCH > 0) {
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
      const int i = lane * 8 + 256 * j;
      if (i < C) body(i, j, r.v + 8 * j);
    }
  } else {
    for (int i = lane * 8; i < C; i += 256) {
      float f[8];
      load8(p + i, f);
      body(i, 0, f);
    }
  }
}

// The lane's channels of a float32 per-channel parameter, into registers.
template <int NCH>
__device__ __forceinline__ void row_load_f32(Row<NCH>& r, const float* p, int C, int lane) {
  if constexpr (NCH > 0) {
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
      const int i = lane * 8 + 256 * j;
#pragma unroll
      for (int u = 0; u < 8; u += 4) {
        const float4 t = i < C ? *reinterpret_cast<const float4*>(p + i + u) : make_float4(0.f, 0.f, 0.f, 0.f);
        r.v[8 * j + u] = t.x;
        r.v[8 * j + u + 1] = t.y;
        r.v[8 * j + u + 2] = t.z;
        r.v[8 * j + u + 3] = t.w;
      }
    }
  }
}

// Channel i + u (chunk j) of a per-channel parameter: from registers, or memory.
template <int NCH>
__device__ __forceinline__ float param(const Row<NCH>& r, const float* p, int i, int j, int u) {
  if constexpr (NCH > 0) return r.v[8 * j + u];
  else return p[i + u];
}

// A lane's chunks of a bf16 row kept as raw 16-byte words (half the
// registers of floats), zero beyond C.
template <int NCH>
struct Raw {
  uint4 v[NCH > 0 ? NCH : 1];
};

template <int NCH>
__device__ __forceinline__ void raw_load(Raw<NCH>& r, const __nv_bfloat16* p, int C, int lane) {
#pragma unroll
  for (int j = 0; j < NCH; ++j) {
    const int i = lane * 8 + 256 * j;
    r.v[j] = i < C ? *reinterpret_cast<const uint4*>(p + i) : make_uint4(0u, 0u, 0u, 0u);
  }
}

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// y = (x - mean) * rstd * g + b per row; one warp per row.
template <int NCH>
__global__ void __launch_bounds__(256) ln_fwd_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ g,
                                                     const float* __restrict__ b, __nv_bfloat16* __restrict__ y,
                                                     long long M, int C) {
  const int lane = threadIdx.x & 31;
  const long long w0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  // a lane owns the same channels in every row: their gains and biases stay in registers
  Row<NCH> gv, bv;
  row_load_f32(gv, g, C, lane);
  row_load_f32(bv, b, C, lane);
  if constexpr (NCH > 0 && NCH <= 2) {
    // short rows: the warp requests its next row before it works on this one
    Raw<NCH> xa, xn;
    if (w0 < M) raw_load(xa, x + w0 * C, C, lane);
    for (long long r = w0; r < M; r += nw) {
      if (r + nw < M) raw_load(xn, x + (r + nw) * C, C, lane);
      Row<NCH> row;
#pragma unroll
      for (int j = 0; j < NCH; ++j) unpack8(xa.v[j], row.v + 8 * j);
      float mean, rstd;
      row_stats(row, x + r * C, C, lane, mean, rstd);
      for_chunks(row, x + r * C, C, lane, [&](int i, int j, const float* f) {
        float o[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) o[u] = (f[u] - mean) * rstd * gv.v[8 * j + u] + bv.v[8 * j + u];
        store8(y + r * C + i, o);
      });
      xa = xn;
    }
  } else {
    for (long long r = w0; r < M; r += nw) {
      const __nv_bfloat16* xr = x + r * C;
      Row<NCH> row;
      row_load(row, xr, C, lane);
      float mean, rstd;
      row_stats(row, xr, C, lane, mean, rstd);
      for_chunks(row, xr, C, lane, [&](int i, int j, const float* f) {
        float o[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          o[u] = (f[u] - mean) * rstd * param(gv, g, i, j, u) + param(bv, b, i, j, u);
        store8(y + r * C + i, o);
      });
    }
  }
}

// Layer-norm backward with the residual added:
//   dx = resid + rstd (dxh - mean(dxh) - xh mean(dxh xh)),  dxh = dy g,
//   dg += sum_rows dy xh,  db += sum_rows dy  (float32, zeroed by the caller).
// One warp per row.  A lane owns the same channels in every row it visits, so
// each warp sums dg/db into its own shared-memory slice with plain adds; the
// block adds its warps' slices to global memory once.  For short rows
// (NCH <= 2) a warp requests the x, dy and residual rows of its next row
// before it works on the current one (kept as raw bf16 words), so that the
// loads of a row overlap the arithmetic of the one before.
template <int NCH>
__global__ void __launch_bounds__(128) ln_bwd_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ g,
                                                     const __nv_bfloat16* __restrict__ dy,
                                                     const __nv_bfloat16* __restrict__ resid,
                                                     __nv_bfloat16* __restrict__ dx, float* __restrict__ dg,
                                                     float* __restrict__ db, long long M, int C) {
  extern __shared__ float acc[];  // [warps][2][C]
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  float* mine = acc + wid * 2 * C;
  for (int i = lane; i < 2 * C; i += 32) mine[i] = 0.f;
  __syncwarp();
  // the lane's gains in registers; its dg/db sums in registers too when the
  // row is short (NCH <= 2), else in the warp's shared slice
  constexpr bool REG_SUMS = NCH > 0 && NCH <= 2;
  Row<NCH> gv;
  row_load_f32(gv, g, C, lane);
  Row<REG_SUMS ? NCH : 0> sg{}, sb{};
  const long long w0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  if constexpr (NCH > 0 && NCH <= 2) {
    Raw<NCH> xa, da, ra;
    auto load3 = [&](long long r, Raw<NCH>& xr, Raw<NCH>& dr, Raw<NCH>& rr) {
      raw_load(xr, x + r * C, C, lane);
      raw_load(dr, dy + r * C, C, lane);
      raw_load(rr, resid + r * C, C, lane);
    };
    if (w0 < M) load3(w0, xa, da, ra);
    for (long long r = w0; r < M; r += nw) {
      Raw<NCH> xn, dn, rn;  // the next row of this warp, requested before this one is worked on
      if (r + nw < M) load3(r + nw, xn, dn, rn);
      float xs[NCH * 8];
#pragma unroll
      for (int jc = 0; jc < NCH; ++jc) unpack8(xa.v[jc], xs + 8 * jc);
      float sum = 0.f;
#pragma unroll
      for (int k = 0; k < NCH * 8; ++k) sum += xs[k];
      const float mean = warp_sum(sum) / C;
      float var = 0.f;
#pragma unroll
      for (int jc = 0; jc < NCH; ++jc)
        if (lane * 8 + 256 * jc < C)
#pragma unroll
          for (int u = 0; u < 8; ++u) var += (xs[8 * jc + u] - mean) * (xs[8 * jc + u] - mean);
      const float rstd = rsqrtf(warp_sum(var) / C + kEps);
      float s1 = 0.f, s2 = 0.f;
#pragma unroll
      for (int jc = 0; jc < NCH; ++jc) {
        const int i = lane * 8 + 256 * jc;
        if (i >= C) continue;
        float d[8];
        unpack8(da.v[jc], d);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int k = 8 * jc + u;
          const float xh = (xs[k] - mean) * rstd;
          const float dxh = d[u] * gv.v[k];
          s1 += dxh;
          s2 += dxh * xh;
          if constexpr (REG_SUMS) {
            sg.v[k] += d[u] * xh;
            sb.v[k] += d[u];
          } else {
            mine[i + u] += d[u] * xh;
            mine[C + i + u] += d[u];
          }
        }
      }
      s1 = warp_sum(s1) / C;
      s2 = warp_sum(s2) / C;
#pragma unroll
      for (int jc = 0; jc < NCH; ++jc) {
        const int i = lane * 8 + 256 * jc;
        if (i >= C) continue;
        float d[8], o[8];
        unpack8(da.v[jc], d);
        unpack8(ra.v[jc], o);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int k = 8 * jc + u;
          const float xh = (xs[k] - mean) * rstd;
          o[u] += rstd * (d[u] * gv.v[k] - s1 - xh * s2);
        }
        store8(dx + r * C + i, o);
      }
      xa = xn;
      da = dn;
      ra = rn;
    }
  } else {
    for (long long r = w0; r < M; r += nw) {
      const __nv_bfloat16* xr = x + r * C;
      const __nv_bfloat16* dr = dy + r * C;
      Row<NCH> row;
      row_load(row, xr, C, lane);
      float mean, rstd;
      row_stats(row, xr, C, lane, mean, rstd);
      float s1 = 0.f, s2 = 0.f;
      for_chunks(row, xr, C, lane, [&](int i, int j, const float* f) {
        float d[8];
        load8(dr + i, d);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float xh = (f[u] - mean) * rstd;
          const float dxh = d[u] * param(gv, g, i, j, u);
          s1 += dxh;
          s2 += dxh * xh;
          mine[i + u] += d[u] * xh;
          mine[C + i + u] += d[u];
        }
      });
      s1 = warp_sum(s1) / C;
      s2 = warp_sum(s2) / C;
      for_chunks(row, xr, C, lane, [&](int i, int j, const float* f) {
        float d[8], o[8];
        load8(dr + i, d);
        load8(resid + r * C + i, o);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float xh = (f[u] - mean) * rstd;
          o[u] += rstd * (d[u] * param(gv, g, i, j, u) - s1 - xh * s2);
        }
        store8(dx + r * C + i, o);
      });
    }
  }
  if constexpr (REG_SUMS) {
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
      const int i = lane * 8 + 256 * j;
      if (i < C)
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          mine[i + u] = sg.v[8 * j + u];
          mine[C + i + u] = sb.v[8 * j + u];
        }
    }
  }
  __syncthreads();
  const int nwb = blockDim.x >> 5;
  for (int i = threadIdx.x; i < 2 * C; i += blockDim.x) {
    float t = 0.f;
    for (int w = 0; w < nwb; ++w) t += acc[w * 2 * C + i];
    atomicAdd(i < C ? &dg[i] : &db[i - C], t);
  }
}

// Phi(u) and the standard normal density phi(u) from one exponential, by
// the rational approximation of the complementary error function in
// Abramowitz and Stegun, Handbook of Mathematical Functions, eq. 7.1.26
// (absolute error below 1.5e-7 for z >= 0):
//   erfc(z) ~ t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-z^2),  t = 1 / (1 + p z),
// with z = |u| / sqrt 2, so that exp(-z^2) = sqrt(2 pi) phi(u) and
// Phi(-|u|) = erfc(z) / 2.
__device__ __forceinline__ void normal_cdf_pdf(float u, float& cdf, float& pdf) {
  const float z = fabsf(u) * 0.70710678118654752f;
  const float t = __fdividef(1.f, fmaf(0.3275911f, z, 1.f));
  const float e = __expf(-z * z);
  const float poly =
      t * fmaf(t, fmaf(t, fmaf(t, fmaf(t, 1.061405429f, -1.453152027f), 1.421413741f), -0.284496736f), 0.254829592f);
  const float tail = 0.5f * poly * e;  // Phi(-|u|)
  cdf = u >= 0.f ? 1.f - tail : tail;
  pdf = 0.3989422804014327f * e;
}

// gelu(u) = u Phi(u), 8 elements a thread; with GRAD also its derivative
// Phi(u) + u phi(u) (phi the standard normal density), for the backward
// pass's recomputation.
template <bool GRAD>
__global__ void __launch_bounds__(256) gelu_kernel(const __nv_bfloat16* __restrict__ u, __nv_bfloat16* __restrict__ out,
                                                   __nv_bfloat16* __restrict__ grad, long long n8) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float f[8], o[8], gd[8];
    load8(u + i * 8, f);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float cdf, pdf;
      normal_cdf_pdf(f[k], cdf, pdf);
      o[k] = f[k] * cdf;
      if (GRAD) gd[k] = cdf + f[k] * pdf;
    }
    store8(out + i * 8, o);
    if (GRAD) store8(grad + i * 8, gd);
  }
}

// du = dg gelu'(u) elementwise (bf16, 8 elements a thread), gelu'(u) computed
// again from u (one exponential and one reciprocal an element are cheaper than
// writing gelu'(u) in the recomputation and reading it back here).
__global__ void __launch_bounds__(256) dgelu_mul_kernel(const __nv_bfloat16* __restrict__ u,
                                                        const __nv_bfloat16* __restrict__ dg,
                                                        __nv_bfloat16* __restrict__ du, long long n8) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float x[8], y[8];
    load8(u + i * 8, x);
    load8(dg + i * 8, y);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float cdf, pdf;
      normal_cdf_pdf(x[k], cdf, pdf);
      y[k] *= cdf + x[k] * pdf;
    }
    store8(du + i * 8, y);
  }
}

// [M][S*C] rows <-> S tensors [B, H, N, D], 16 bytes (8 of D) a thread: a
// thread keeps its place in the row (tensor s, head h, d) for every row the
// block visits.
template <bool TO_HEADS>
__global__ void __launch_bounds__(256) heads_kernel(__nv_bfloat16* __restrict__ rows, __nv_bfloat16* __restrict__ h0,
                                                    __nv_bfloat16* __restrict__ h1, __nv_bfloat16* __restrict__ h2,
                                                    int B, int N, int H, int D, int S) {
  const int C = H * D;
  const int per_row = S * C / 8;
  const long long M = static_cast<long long>(B) * N;
  for (int v = threadIdx.x; v < per_row; v += blockDim.x) {
    const int col = v * 8;
    const int s = col / C, c = col - s * C;
    const int h = c / D, d = c - h * D;
    __nv_bfloat16* hs = s == 0 ? h0 : (s == 1 ? h1 : h2);
    hs += static_cast<long long>(h) * N * D + d;
    for (long long row = blockIdx.x; row < M; row += gridDim.x) {
      const long long b = row / N, t = row - b * N;
      uint4* hp = reinterpret_cast<uint4*>(hs + (b * H * N + t) * D);
      uint4* rp = reinterpret_cast<uint4*>(rows + row * S * C + col);
      if (TO_HEADS) *hp = *rp;
      else *rp = *hp;
    }
  }
}

// ------------------------------------------------------------------ host side
int grid_for(long long items, int per_block) {
  long long b = (items + per_block - 1) / per_block;
  if (b < 1) b = 1;
  if (b > 148 * 8) b = 148 * 8;
  return static_cast<int>(b);
}

int last_launch() { return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA; }

// heads_kernel: a block per row (grid-stride), a thread per 16 bytes of it.
int heads_grid(long long M) { return static_cast<int>(std::min<long long>(M, 148 * 16)); }
int heads_block(int width) { return std::min(256, std::max(32, (width / 8 + 31) / 32 * 32)); }

// Layer-norm launches: the row in registers up to C = 1024, read again per
// pass above that; for C <= 512 each warp requests its next row ahead.
int ln_fwd(const __nv_bfloat16* x, const float* g, const float* b, __nv_bfloat16* y, long long M, int C,
           cudaStream_t s) {
  auto go = [&](auto kernel, bool one_wave) -> int {
    int grid = grid_for(M * 32, 256);
    if (one_wave) {  // rows requested ahead: one wave of resident blocks, each warp several rows
      int dev = 0, sms = 0, per_sm = 0;
      if (cudaGetDevice(&dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
          cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, 0) != cudaSuccess)
        return SA_ERR_CUDA;
      grid = static_cast<int>(std::min<long long>(grid, static_cast<long long>(sms) * std::max(per_sm, 1)));
    }
    kernel<<<grid, 256, 0, s>>>(x, g, b, y, M, C);
    return last_launch();
  };
  if (C <= 256) return go(ln_fwd_kernel<1>, true);
  if (C <= 512) return go(ln_fwd_kernel<2>, true);
  if (C <= 1024) return go(ln_fwd_kernel<4>, false);
  return go(ln_fwd_kernel<0>, false);
}

int ln_bwd(const __nv_bfloat16* x, const float* g, const __nv_bfloat16* dy, const __nv_bfloat16* resid,
           __nv_bfloat16* dx, float* dg, float* db, long long M, int C, cudaStream_t s) {
  constexpr int kThreads = 128;  // 4 warps, each with its own dg/db slice
  const size_t smem = 4 * 2 * static_cast<size_t>(C) * sizeof(float);
  auto go = [&](auto kernel) -> int {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
            cudaSuccess)
      return SA_ERR_CUDA;
    // one wave of resident blocks (at most 4 a SM: each adds 2 C sums to dg/db)
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem) != cudaSuccess)
      return SA_ERR_CUDA;
    per_sm = std::max(1, std::min(per_sm, 4));
    const int grid = static_cast<int>(std::min<long long>((M + 3) / 4, static_cast<long long>(sms) * per_sm));
    kernel<<<grid, kThreads, smem, s>>>(x, g, dy, resid, dx, dg, db, M, C);
    return last_launch();
  };
  if (C <= 256) return go(ln_bwd_kernel<1>);
  if (C <= 512) return go(ln_bwd_kernel<2>);
  if (C <= 1024) return go(ln_bwd_kernel<4>);
  return go(ln_bwd_kernel<0>);
}

// Serialises the host side of the block calls: the per-device cuBLAS handle
// is bound to the caller's stream for the duration of one call's enqueue.
std::mutex g_call_mu;

// One cuBLAS handle per device, created on first use.
cublasHandle_t handle_for_current_device() {
  static std::mutex mu;
  static cublasHandle_t handles[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!handles[dev] && cublasCreate(&handles[dev]) != CUBLAS_STATUS_SUCCESS) handles[dev] = nullptr;
  return handles[dev];
}

cublasLtHandle_t lt_handle_for_current_device() {
  static std::mutex mu;
  static cublasLtHandle_t handles[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!handles[dev] && cublasLtCreate(&handles[dev]) != CUBLAS_STATUS_SUCCESS) handles[dev] = nullptr;
  return handles[dev];
}

// Row-major Out[M][Nn] = A[M][K] W[K][Nn] + R[M][Nn], all bf16, float32
// accumulation; R and Out distinct buffers (cuBLASLt, no workspace).
int mm_residual(cublasLtHandle_t lt, const void* A, const void* W, const void* R, void* Out, int M, int K, int Nn,
                cudaStream_t s) {
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  int st = SA_ERR_CUDA;
  const float one = 1.f;
  size_t ws = 0;
  cublasLtMatmulHeuristicResult_t res{};
  int n_res = 0;
  if (cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F) == CUBLAS_STATUS_SUCCESS &&
      cublasLtMatrixLayoutCreate(&la, CUDA_R_16BF, Nn, K, Nn) == CUBLAS_STATUS_SUCCESS &&
      cublasLtMatrixLayoutCreate(&lb, CUDA_R_16BF, K, M, K) == CUBLAS_STATUS_SUCCESS &&
      cublasLtMatrixLayoutCreate(&lc, CUDA_R_16BF, Nn, M, Nn) == CUBLAS_STATUS_SUCCESS &&
      cublasLtMatmulPreferenceCreate(&pref) == CUBLAS_STATUS_SUCCESS &&
      cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws, sizeof(ws)) ==
          CUBLAS_STATUS_SUCCESS &&
      cublasLtMatmulAlgoGetHeuristic(lt, op, la, lb, lc, lc, pref, 1, &res, &n_res) == CUBLAS_STATUS_SUCCESS &&
      n_res > 0 &&
      cublasLtMatmul(lt, op, &one, W, la, A, lb, &one, R, lc, Out, lc, &res.algo, nullptr, 0, s) ==
          CUBLAS_STATUS_SUCCESS)
    st = SA_OK;
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (lc) cublasLtMatrixLayoutDestroy(lc);
  if (lb) cublasLtMatrixLayoutDestroy(lb);
  if (la) cublasLtMatrixLayoutDestroy(la);
  if (op) cublasLtMatmulDescDestroy(op);
  return st;
}

// A second stream per device, with a cuBLAS handle of its own, for the
// weight gradients of the backward pass: they run beside the chain of data
// gradients and join it before the call returns.  Created on first use,
// under the call lock.
struct Side {
  cudaStream_t s = nullptr;
  cublasHandle_t h = nullptr;
  cudaEvent_t ev[5] = {};
};

Side* side_for_current_device() {
  static Side sides[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  Side& sd = sides[dev];
  if (sd.s) return &sd;
  Side n;
  bool ok = cudaStreamCreateWithFlags(&n.s, cudaStreamNonBlocking) == cudaSuccess &&
            cublasCreate(&n.h) == CUBLAS_STATUS_SUCCESS && cublasSetStream(n.h, n.s) == CUBLAS_STATUS_SUCCESS;
  for (auto& e : n.ev) ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    for (auto& e : n.ev)
      if (e) cudaEventDestroy(e);
    if (n.h) cublasDestroy(n.h);
    if (n.s) cudaStreamDestroy(n.s);
    return nullptr;
  }
  sd = n;
  return &sd;
}

struct Gemm {
  cublasHandle_t h;
  // Row-major Out[M][Nn] = A[M][K] W[K][Nn] + beta Out (bf16 out).
  int mm(const void* A, const void* W, void* Out, int M, int K, int Nn, float beta) const {
    const float one = 1.f;
    return cublasGemmEx(h, CUBLAS_OP_N, CUBLAS_OP_N, Nn, M, K, &one, W, CUDA_R_16BF, Nn, A, CUDA_R_16BF, K, &beta,
                        Out, CUDA_R_16BF, Nn, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) == CUBLAS_STATUS_SUCCESS
               ? SA_OK
               : SA_ERR_CUDA;
  }
  // Row-major Out[M][K] = dOut[M][Nn] W[K][Nn]^T (bf16 out).
  int mm_nt(const void* dOut, const void* W, void* Out, int M, int K, int Nn) const {
    const float one = 1.f, zero = 0.f;
    return cublasGemmEx(h, CUBLAS_OP_T, CUBLAS_OP_N, K, M, Nn, &one, W, CUDA_R_16BF, Nn, dOut, CUDA_R_16BF, Nn,
                        &zero, Out, CUDA_R_16BF, K, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) == CUBLAS_STATUS_SUCCESS
               ? SA_OK
               : SA_ERR_CUDA;
  }
  // Row-major dW[K][Nn] = A[M][K]^T dOut[M][Nn] (float32 out).
  int mm_tn(const void* A, const void* dOut, float* dW, int M, int K, int Nn) const {
    const float one = 1.f, zero = 0.f;
    return cublasGemmEx(h, CUBLAS_OP_N, CUBLAS_OP_T, Nn, K, M, &one, dOut, CUDA_R_16BF, Nn, A, CUDA_R_16BF, K,
                        &zero, dW, CUDA_R_32F, Nn, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) == CUBLAS_STATUS_SUCCESS
               ? SA_OK
               : SA_ERR_CUDA;
  }
};

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

// Workspace regions (bytes from the start), in units of M*C bf16 elements.
struct Ws {
  size_t a, qkv, q, k, v, o, lse, o2, h, f, u, g;               // forward (and recomputation)
  size_t dg, du, df, dh, do2, dO, dq, dk, dv, dqkv, da, attn;  // backward
  size_t attn_bytes, total;
};

Ws layout_ws(int B, int N, int H, int D, const sa_layout* L) {
  const size_t mc = static_cast<size_t>(B) * N * H * D * 2;  // bytes of one [M][C] bf16 tensor
  Ws w{};
  size_t at = 0;
  auto take = [&](size_t bytes) {
    const size_t r = at;
    at += align256(bytes);
    return r;
  };
  w.a = take(mc);
  w.qkv = take(3 * mc);
  w.q = take(mc);
  w.k = take(mc);
  w.v = take(mc);
  w.o = take(mc);
  w.lse = take(static_cast<size_t>(B) * H * N * 4);
  w.o2 = take(mc);
  w.h = take(mc);
  w.f = take(mc);
  w.u = take(4 * mc);
  w.g = take(4 * mc);
  w.dg = take(4 * mc);
  w.du = take(4 * mc);
  w.df = take(mc);
  w.dh = take(mc);
  w.do2 = take(mc);
  w.dO = take(mc);
  w.dq = take(mc);
  w.dk = take(mc);
  w.dv = take(mc);
  w.dqkv = take(3 * mc);
  w.da = take(mc);
  w.attn_bytes = sparse_attn_bwd_workspace_size(B, H, N, D, L);
  w.attn = take(w.attn_bytes);
  w.total = at;
  return w;
}

int check_args(int B, int N, int H, int D, const sa_layout* L, void* ws, size_t ws_bytes) {
  if (B < 1 || N < 1 || H < 1 || !L) return SA_ERR_INVALID_ARG;
  if (D != 32 && D != 64 && D != 128) return SA_ERR_UNSUPPORTED;
  if (H * D > kMaxC) return SA_ERR_UNSUPPORTED;  // the layer-norm backward's shared sums
  const Ws w = layout_ws(B, N, H, D, L);
  if (w.attn_bytes == 0) return SA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < w.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SA_ERR_WORKSPACE;
  return SA_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// The forward chain into the workspace: a, q, k, v, o, lse, o2, h, f, u, g
// (when y is given, h is built in y and y = h + g W2 follows).
int forward_chain(const __nv_bfloat16* x, const sb_params* p, __nv_bfloat16* y, int B, int N, int H, int D,
                  const sa_layout* L, void* ws, cudaStream_t s, const Gemm& G) {
  const Ws w = layout_ws(B, N, H, D, L);
  const long long M = static_cast<long long>(B) * N;
  const int C = H * D;
  auto* a = at<__nv_bfloat16>(ws, w.a);
  auto* qkv = at<__nv_bfloat16>(ws, w.qkv);
  auto* q = at<__nv_bfloat16>(ws, w.q);
  auto* k = at<__nv_bfloat16>(ws, w.k);
  auto* v = at<__nv_bfloat16>(ws, w.v);
  auto* o = at<__nv_bfloat16>(ws, w.o);
  auto* lse = at<float>(ws, w.lse);
  auto* o2 = at<__nv_bfloat16>(ws, w.o2);
  auto* h = at<__nv_bfloat16>(ws, w.h);
  auto* f = at<__nv_bfloat16>(ws, w.f);
  auto* u = at<__nv_bfloat16>(ws, w.u);
  auto* g = at<__nv_bfloat16>(ws, w.g);
  int st;
  if ((st = ln_fwd(x, p->ln1_g, p->ln1_b, a, M, C, s))) return st;
  if ((st = G.mm(a, p->w_qkv, qkv, static_cast<int>(M), C, 3 * C, 0.f))) return st;
  heads_kernel<true><<<heads_grid(M), heads_block(3 * C), 0, s>>>(qkv, q, k, v, B, N, H, D, 3);
  if ((st = last_launch())) return st;
  if ((st = sparse_attn_fwd(q, k, v, o, lse, B, H, N, D, L, s))) return st;
  heads_kernel<false><<<heads_grid(M), heads_block(C), 0, s>>>(o2, o, nullptr, nullptr, B, N, H, D, 1);
  if ((st = last_launch())) return st;
  // h = x + o Wo, the residual added by the GEMM itself (cuBLASLt reads x
  // and writes h, so no copy of x); the forward proper builds h in y itself
  // (y = h + ff then needs no copy of h), the recomputation in the workspace
  __nv_bfloat16* hb = y ? y : h;
  {
    cublasLtHandle_t lt = lt_handle_for_current_device();
    if (!lt) return SA_ERR_CUDA;
    if ((st = mm_residual(lt, o2, p->w_o, x, hb, static_cast<int>(M), C, C, s))) return st;
  }
  if ((st = ln_fwd(hb, p->ln2_g, p->ln2_b, f, M, C, s))) return st;
  if ((st = G.mm(f, p->w_1, u, static_cast<int>(M), C, 4 * C, 0.f))) return st;
  gelu_kernel<false><<<grid_for(M * 4 * C / 8, 256), 256, 0, s>>>(u, g, nullptr, M * 4 * C / 8);
  if ((st = last_launch())) return st;
  if (y && (st = G.mm(g, p->w_2, y, static_cast<int>(M), 4 * C, C, 1.f))) return st;
  return SA_OK;
}

bool params_ok(const sb_params* p) {
  return p && p->ln1_g && p->ln1_b && p->w_qkv && p->w_o && p->ln2_g && p->ln2_b && p->w_1 && p->w_2;
}

}  // namespace sb

using namespace sb;

extern "C" {

int sparse_block_gelu(const void* u, void* g, void* dgelu, size_t n, void* stream) {
  if (!u || !g || n % 8 || ((reinterpret_cast<uintptr_t>(u) | reinterpret_cast<uintptr_t>(g) |
                             reinterpret_cast<uintptr_t>(dgelu)) & 15u))
    return SA_ERR_INVALID_ARG;
  if (dgelu && (dgelu == u || dgelu == g)) return SA_ERR_INVALID_ARG;
  if (n == 0) return SA_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long n8 = static_cast<long long>(n / 8);
  const auto* ub = static_cast<const __nv_bfloat16*>(u);
  auto* gb = static_cast<__nv_bfloat16*>(g);
  if (dgelu) gelu_kernel<true><<<grid_for(n8, 256), 256, 0, s>>>(ub, gb, static_cast<__nv_bfloat16*>(dgelu), n8);
  else gelu_kernel<false><<<grid_for(n8, 256), 256, 0, s>>>(ub, gb, nullptr, n8);
  return last_launch();
}

size_t sparse_block_workspace_size(int B, int N, int H, int D, const sa_layout* layout) {
  if (B < 1 || N < 1 || H < 1 || !layout || (D != 32 && D != 64 && D != 128) || H * D > kMaxC) return 0;
  const Ws w = layout_ws(B, N, H, D, layout);
  return w.attn_bytes ? w.total : 0;
}

int sparse_block_fwd(const void* x, const sb_params* p, void* y, int B, int N, int H, int D,
                     const sa_layout* layout, void* workspace, size_t ws_bytes, void* stream) {
  if (!x || !y || x == y || !params_ok(p)) return SA_ERR_INVALID_ARG;
  int st = check_args(B, N, H, D, layout, workspace, ws_bytes);
  if (st) return st;
  std::lock_guard<std::mutex> lock(g_call_mu);
  Gemm G{handle_for_current_device()};
  if (!G.h) return SA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cublasSetStream(G.h, s) != CUBLAS_STATUS_SUCCESS) return SA_ERR_CUDA;
  return forward_chain(static_cast<const __nv_bfloat16*>(x), p, static_cast<__nv_bfloat16*>(y), B, N, H, D, layout,
                       workspace, s, G);
}

int sparse_block_bwd(const void* x, const void* dy, const sb_params* p, void* dx, const sb_grads* gr, int B, int N,
                     int H, int D, const sa_layout* layout, void* workspace, size_t ws_bytes, void* stream) {
  if (!x || !dy || !dx || !params_ok(p) || !gr || !gr->ln1_g || !gr->ln1_b || !gr->w_qkv || !gr->w_o ||
      !gr->ln2_g || !gr->ln2_b || !gr->w_1 || !gr->w_2)
    return SA_ERR_INVALID_ARG;
  int st = check_args(B, N, H, D, layout, workspace, ws_bytes);
  if (st) return st;
  std::lock_guard<std::mutex> lock(g_call_mu);
  Gemm G{handle_for_current_device()};
  if (!G.h) return SA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cublasSetStream(G.h, s) != CUBLAS_STATUS_SUCCESS) return SA_ERR_CUDA;
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  const auto* dyb = static_cast<const __nv_bfloat16*>(dy);
  // the recomputation: every activation again from x
  const Ws w = layout_ws(B, N, H, D, layout);
  if ((st = forward_chain(xb, p, nullptr, B, N, H, D, layout, workspace, s, G)))
    return st;
  const long long M = static_cast<long long>(B) * N;
  const int C = H * D, Mi = static_cast<int>(M);
  void* ws = workspace;
  auto* a = at<__nv_bfloat16>(ws, w.a);
  auto* q = at<__nv_bfloat16>(ws, w.q);
  auto* k = at<__nv_bfloat16>(ws, w.k);
  auto* v = at<__nv_bfloat16>(ws, w.v);
  auto* o = at<__nv_bfloat16>(ws, w.o);
  auto* lse = at<float>(ws, w.lse);
  auto* o2 = at<__nv_bfloat16>(ws, w.o2);
  auto* h = at<__nv_bfloat16>(ws, w.h);
  auto* f = at<__nv_bfloat16>(ws, w.f);
  auto* g = at<__nv_bfloat16>(ws, w.g);
  auto* dg = at<__nv_bfloat16>(ws, w.dg);
  auto* du = at<__nv_bfloat16>(ws, w.du);
  auto* df = at<__nv_bfloat16>(ws, w.df);
  auto* dh = at<__nv_bfloat16>(ws, w.dh);
  auto* do2 = at<__nv_bfloat16>(ws, w.do2);
  auto* dO = at<__nv_bfloat16>(ws, w.dO);
  auto* dq = at<__nv_bfloat16>(ws, w.dq);
  auto* dk = at<__nv_bfloat16>(ws, w.dk);
  auto* dv = at<__nv_bfloat16>(ws, w.dv);
  auto* dqkv = at<__nv_bfloat16>(ws, w.dqkv);
  auto* da = at<__nv_bfloat16>(ws, w.da);
  // The weight gradients go to the side stream as soon as their operands
  // exist (fork k: an event on the caller's stream that the side stream
  // waits for); the side stream joins the caller's stream at the end, on
  // every path that forked.
  Side* sd = side_for_current_device();
  if (!sd) return SA_ERR_CUDA;
  const Gemm GS{sd->h};
  bool forked = false;
  auto fork = [&](int k) {
    forked = true;
    return cudaEventRecord(sd->ev[k], s) == cudaSuccess && cudaStreamWaitEvent(sd->s, sd->ev[k], 0) == cudaSuccess
               ? SA_OK
               : SA_ERR_CUDA;
  };
  auto chain = [&]() -> int {
    // feed-forward: y = h + gelu(f W1) W2
    if ((st = fork(0)) || (st = GS.mm_tn(g, dyb, gr->w_2, Mi, 4 * C, C))) return st;
    if ((st = G.mm_nt(dyb, p->w_2, dg, Mi, 4 * C, C))) return st;
    dgelu_mul_kernel<<<grid_for(M * 4 * C / 8, 256), 256, 0, s>>>(at<__nv_bfloat16>(ws, w.u), dg, du, M * 4 * C / 8);
    if ((st = last_launch())) return st;
    if ((st = fork(1)) || (st = GS.mm_tn(f, du, gr->w_1, Mi, C, 4 * C))) return st;
    if ((st = G.mm_nt(du, p->w_1, df, Mi, C, 4 * C))) return st;
    if (cudaMemsetAsync(gr->ln2_g, 0, C * sizeof(float), s) != cudaSuccess ||
        cudaMemsetAsync(gr->ln2_b, 0, C * sizeof(float), s) != cudaSuccess)
      return SA_ERR_CUDA;
    if ((st = ln_bwd(h, p->ln2_g, df, dyb, dh, gr->ln2_g, gr->ln2_b, M, C, s))) return st;
    // attention: h = x + o Wo
    if ((st = fork(2)) || (st = GS.mm_tn(o2, dh, gr->w_o, Mi, C, C))) return st;
    if ((st = G.mm_nt(dh, p->w_o, do2, Mi, C, C))) return st;
    heads_kernel<true><<<heads_grid(M), heads_block(C), 0, s>>>(do2, dO, nullptr, nullptr, B, N, H, D, 1);
    if ((st = last_launch())) return st;
    if ((st = sparse_attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, D, layout, at<void>(ws, w.attn),
                              w.attn_bytes, s)))
      return st;
    heads_kernel<false><<<heads_grid(M), heads_block(3 * C), 0, s>>>(dqkv, dq, dk, dv, B, N, H, D, 3);
    if ((st = last_launch())) return st;
    if ((st = fork(3)) || (st = GS.mm_tn(a, dqkv, gr->w_qkv, Mi, C, 3 * C))) return st;
    if ((st = G.mm_nt(dqkv, p->w_qkv, da, Mi, C, 3 * C))) return st;
    if (cudaMemsetAsync(gr->ln1_g, 0, C * sizeof(float), s) != cudaSuccess ||
        cudaMemsetAsync(gr->ln1_b, 0, C * sizeof(float), s) != cudaSuccess)
      return SA_ERR_CUDA;
    return ln_bwd(xb, p->ln1_g, da, dh, static_cast<__nv_bfloat16*>(dx), gr->ln1_g, gr->ln1_b, M, C, s);
  };
  st = chain();
  if (forked && (cudaEventRecord(sd->ev[4], sd->s) != cudaSuccess || cudaStreamWaitEvent(s, sd->ev[4], 0) != cudaSuccess))
    st = st ? st : SA_ERR_CUDA;
  return st;
}

}  // extern "C"
