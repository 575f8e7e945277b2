// Backward kernels: recompute-based gradient of block-sparse attention.
//
// The backward pass rebuilds P from the saved log-sum-exp instead of keeping
// the attention matrix, the recomputation of "Generating Long Sequences with
// Sparse Transformers" (ABSTRACT, item b) and of the pcnews translation
// ("Глубокое внимание").  With Delta_i = sum_d dO_id O_id:
//   P = exp(S - lse), dV = P^T dO, dP = dO V^T, dS = P (dP - Delta),
//   dK = s dS^T Q, dQ = s dS K.
//
// sa_bwd_kernel: one CTA = one 128-key tile of one (batch, head), in the
// view order of its table; it walks the 128-query tiles that see it.
//   ST  = K Q^T      (keys on TMEM lanes)          -> P^T   (bf16, smem)
//   dPT = V dO^T                                    -> dS^T  (bf16, smem)
//   dV += P^T dO,  dK += dS^T Q   (TMEM accumulators for the whole CTA)
//   dQ  = dS K       (queries on TMEM lanes, reusing the ST columns), then
//                    added to an fp32 workspace with vector reductions.
// Roles: warp 0 lane 0 TMA producer; warp 1 TMEM allocation and lane 0 MMA
// issue; warps 2..5 elementwise work, thread t of warp w owns TMEM lane
// 32*(w%4)+t (a key row for ST/dPT/dV/dK, a query row for dQ).
// TMEM columns: ST/dQ [0,128), dPT [128,256), dV [256,256+D), dK [256+D,256+2D).
#pragma once

#include "sa_device.cuh"
#include "sa_fwd.cuh"

namespace sa {

struct BwdArgs {
  const int32_t* row_ptr;
  const int32_t* ent;
  const int32_t* order;
  const float* lse;      // [BH, N] natural log
  const float* delta;    // [BH, N]
  float* dq_acc;         // [BH, N, D] fp32, scaled
  __nv_bfloat16* dk;     // final outputs (main pass)
  __nv_bfloat16* dv;
  float* dk_part;        // secondary partials [BH, N, D] fp32 at natural key positions
  float* dv_part;
  int N, l, c, R;
  int pattern;
  int key_view;  // SRC_N, SRC_T or SRC_S
  int add_part;  // main pass: add secondary partials (1 strided: all keys; 2 fixed: summary keys)
  float scale;       // 1/sqrt(D)
  float scale_log2;  // log2(e)/sqrt(D)
};

template <int D>
struct BwdCfg {
  static constexpr int TK = 128, TQ = 128;
  static constexpr int STAGES = (D >= 128) ? 1 : 2;
  static constexpr int ROWB = (D >= 64) ? 128 : 64;
  static constexpr int PANELS = (D >= 64) ? D / 64 : 1;
  static constexpr uint64_t SWZ = (D >= 64) ? kSwizzle128 : kSwizzle64;
  static constexpr int SBO = 8 * ROWB;
  static constexpr int T_BYTES = 128 * D * 2;   // one 128-row tile of D
  static constexpr int PT_BYTES = 128 * 128 * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + T_BYTES;
  static constexpr int OFF_Q = OFF_V + T_BYTES;
  static constexpr int OFF_DO = OFF_Q + STAGES * T_BYTES;
  static constexpr int OFF_PT = OFF_DO + STAGES * T_BYTES;
  static constexpr int OFF_DST = OFF_PT + PT_BYTES;
  static constexpr int OFF_LSE = OFF_DST + PT_BYTES;        // float [2][128]
  static constexpr int OFF_DELTA = OFF_LSE + 2 * 128 * 4;   // float [2][128]
  static constexpr int OFF_BAR = OFF_DELTA + 2 * 128 * 4;
  static constexpr int N_BARS = 1 + 2 * STAGES + 8;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int COL_ST = 0, COL_DPT = 128, COL_DV = 256, COL_DK = 256 + D;
};

template <int D>
__device__ __forceinline__ uint64_t bwd_kdesc(uint32_t base, int kk) {  // K-major, 128 rows, K = D
  using C = BwdCfg<D>;
  constexpr int spp = C::ROWB / 32;
  return make_desc(base + (kk / spp) * 128 * C::ROWB + (kk % spp) * 32, 16, C::SBO, C::SWZ);
}
template <int D>
__device__ __forceinline__ uint64_t bwd_mndesc(uint32_t base, int kk) {  // MN-major, N = D, K = 128 rows
  using C = BwdCfg<D>;
  return make_desc(base + kk * 16 * C::ROWB, 128 * C::ROWB, C::SBO, C::SWZ);
}
// P^T / dS^T buffers: [128 rows][128 cols] bf16 as 2 panels of [128][64], 128B swizzle.
__device__ __forceinline__ uint64_t pt_kdesc(uint32_t base, int kk) {  // K-major (K = cols)
  return make_desc(base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kSwizzle128);
}
__device__ __forceinline__ uint64_t pt_mndesc(uint32_t base, int kk) {  // MN-major (M = cols, K = rows)
  return make_desc(base + kk * 2048, 16384, 1024, kSwizzle128);
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int D>
__global__ void __launch_bounds__(192, 1)
    sa_bwd_kernel(const __grid_constant__ CUtensorMap mq_nat, const __grid_constant__ CUtensorMap mq_col,
                  const __grid_constant__ CUtensorMap mdo_nat, const __grid_constant__ CUtensorMap mdo_col,
                  const __grid_constant__ CUtensorMap mk_nat, const __grid_constant__ CUtensorMap mk_col,
                  const __grid_constant__ CUtensorMap mk_sum, const __grid_constant__ CUtensorMap mv_nat,
                  const __grid_constant__ CUtensorMap mv_col, const __grid_constant__ CUtensorMap mv_sum,
                  const BwdArgs a) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sDO = smem + C::OFF_DO;
  uint8_t* sPT = smem + C::OFF_PT;
  uint8_t* sDST = smem + C::OFF_DST;
  float* sLse = reinterpret_cast<float*>(smem + C::OFF_LSE);
  float* sDelta = reinterpret_cast<float*>(smem + C::OFF_DELTA);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_kv = bars;
  uint64_t* bar_qdo_full = bars + 1;
  uint64_t* bar_qdo_empty = bar_qdo_full + C::STAGES;
  uint64_t* bar_st_full = bar_qdo_empty + C::STAGES;
  uint64_t* bar_dpt_full = bar_st_full + 1;
  uint64_t* bar_pt_full = bar_dpt_full + 1;
  uint64_t* bar_dst_full = bar_pt_full + 1;
  uint64_t* bar_dq_full = bar_dst_full + 1;
  uint64_t* bar_dq_free = bar_dq_full + 1;
  uint64_t* bar_dkv_full = bar_dq_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);

  const int bh = blockIdx.x;
  const int kt = a.order[blockIdx.y];
  const int e0 = a.row_ptr[kt];
  const int n = a.row_ptr[kt + 1] - e0;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q_src = (a.key_view == SRC_T) ? SRC_T : SRC_N;

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_qdo_full + s, 1);
      mbar_init(bar_qdo_empty + s, 1);
    }
    mbar_init(bar_st_full, 1);
    mbar_init(bar_dpt_full, 1);
    mbar_init(bar_pt_full, 128);
    mbar_init(bar_dst_full, 128);
    mbar_init(bar_dq_full, 1);
    mbar_init(bar_dq_free, 128);
    mbar_init(bar_dkv_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc<C::TMEM_COLS>(tmem_slot);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0 && n > 0) {
      // ------------------------------------------------------------ producer
      mbar_arrive_expect_tx(bar_kv, 2 * C::T_BYTES);
      load_rows<D>(sK, a.key_view, kt * C::TK, C::TK, bh, &mk_nat, &mk_col, &mk_sum, bar_kv, a.R, a.l, a.c);
      load_rows<D>(sV, a.key_view, kt * C::TK, C::TK, bh, &mv_nat, &mv_col, &mv_sum, bar_kv, a.R, a.l, a.c);
      for (int j = 0; j < n; ++j) {
        const int st = j % C::STAGES;
        if (j >= C::STAGES && !mbar_wait(bar_qdo_empty + st, ((j / C::STAGES) - 1) & 1, abort_flag)) break;
        const int qpos = (a.ent[e0 + j] >> 3) * C::TQ;
        mbar_arrive_expect_tx(bar_qdo_full + st, 2 * C::T_BYTES);
        load_rows<D>(sQ + st * C::T_BYTES, q_src, qpos, C::TQ, bh, &mq_nat, &mq_col, &mq_col,
                     bar_qdo_full + st, a.R, a.l, a.c);
        load_rows<D>(sDO + st * C::T_BYTES, q_src, qpos, C::TQ, bh, &mdo_nat, &mdo_col, &mdo_col,
                     bar_qdo_full + st, a.R, a.l, a.c);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && n > 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t id_s = make_idesc_bf16(128, 128, false, false);  // ST, dPT
      constexpr uint32_t id_kv = make_idesc_bf16(128, D, false, true);    // dV, dK
      constexpr uint32_t id_q = make_idesc_bf16(128, D, true, true);      // dQ
      const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
      const uint32_t pt_base = smem_u32(sPT), dst_base = smem_u32(sDST);
      bool ok = mbar_wait(bar_kv, 0, abort_flag);
      for (int j = 0; ok && j < n; ++j) {
        const int st = j % C::STAGES;
        ok = mbar_wait(bar_qdo_full + st, (j / C::STAGES) & 1, abort_flag);
        if (ok && j > 0) ok = mbar_wait(bar_dq_free, (j - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t q_base = smem_u32(sQ + st * C::T_BYTES);
        const uint32_t do_base = smem_u32(sDO + st * C::T_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tmem + C::COL_ST, bwd_kdesc<D>(k_base, kk), bwd_kdesc<D>(q_base, kk), id_s, kk > 0);
        mma_commit(bar_st_full);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tmem + C::COL_DPT, bwd_kdesc<D>(v_base, kk), bwd_kdesc<D>(do_base, kk), id_s, kk > 0);
        mma_commit(bar_dpt_full);
        if (!mbar_wait(bar_pt_full, j & 1, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + C::COL_DV, pt_kdesc(pt_base, kk), bwd_mndesc<D>(do_base, kk), id_kv, (j > 0 || kk > 0));
        if (!mbar_wait(bar_dst_full, j & 1, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + C::COL_DK, pt_kdesc(dst_base, kk), bwd_mndesc<D>(q_base, kk), id_kv, (j > 0 || kk > 0));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + C::COL_ST, pt_mndesc(dst_base, kk), bwd_mndesc<D>(k_base, kk), id_q, kk > 0);
        mma_commit(bar_dq_full);
        mma_commit(bar_qdo_empty + st);
      }
      mma_commit(bar_dkv_full);
    }
  } else {
    // ------------------------------------------------------------ elementwise
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int ctid = threadIdx.x - 64;  // 0..127
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    // this thread's key: view position y, natural position
    const int y = kt * C::TK + row;
    const int nkeys = (a.key_view == SRC_S) ? a.R * a.c : a.N;
    const bool kvalid = y < nkeys;
    int knat;
    if (a.key_view == SRC_T) knat = (y % a.R) * a.l + y / a.R;
    else if (a.key_view == SRC_S) knat = (y / a.c) * a.l + (a.l - a.c) + y % a.c;
    else knat = y;
    // queries (view order) that see this key: [qlo, qhi]
    int qlo, qhi;
    if (a.key_view == SRC_T) {
      qlo = y + 1;
      qhi = (y / a.R) * a.R + a.R - 1;
    } else if (a.key_view == SRC_S) {
      qlo = (y / a.c + 1) * a.l;
      qhi = a.N - 1;
    } else {
      qlo = y;
      if (a.pattern == SA_ALL) qhi = a.N - 1;
      else if (a.pattern == SA_FIXED) qhi = (y / a.l) * a.l + a.l - 1;
      else qhi = y + a.l - 1;
    }
    if (qhi > a.N - 1) qhi = a.N - 1;
    if (!kvalid) qhi = qlo - 1;

    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int e = a.ent[e0 + j];
      const int qt = e >> 3;
      const bool partial = e & 1;
      const int buf = j & 1;
      // lse (log2 units) and Delta of this tile's queries
      {
        const int x = qt * C::TQ + ctid;
        float lv = INFINITY, dv = 0.f;
        if (x < a.N) {
          const int qn = (q_src == SRC_T) ? (x % a.R) * a.l + x / a.R : x;
          lv = a.lse[static_cast<size_t>(bh) * a.N + qn] * 1.4426950408889634f;
          dv = a.delta[static_cast<size_t>(bh) * a.N + qn];
        }
        sLse[buf * 128 + ctid] = lv;
        sDelta[buf * 128 + ctid] = dv;
      }
      named_bar_sync(1, 128);
      const float* lse_t = sLse + buf * 128;
      const float* del_t = sDelta + buf * 128;
      const int x0 = qt * C::TQ;

      // ---- P^T row (this key against 128 queries)
      ok = ok && mbar_wait(bar_st_full, j & 1, abort_flag);
      tc_fence_after();
      float p[128];
#pragma unroll
      for (int i = 0; i < 8; ++i) tmem_ld16(tmem + lane_base + C::COL_ST + i * 16, p + i * 16);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        float v = ex2(fmaf(p[i], a.scale_log2, -lse_t[i]));
        if (partial) {
          const int x = x0 + i;
          if (x < qlo || x > qhi) v = 0.f;
        }
        p[i] = v;
      }
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        uint4 w;
        w.x = pack_bf16(p[ch * 8 + 0], p[ch * 8 + 1]);
        w.y = pack_bf16(p[ch * 8 + 2], p[ch * 8 + 3]);
        w.z = pack_bf16(p[ch * 8 + 4], p[ch * 8 + 5]);
        w.w = pack_bf16(p[ch * 8 + 6], p[ch * 8 + 7]);
        *reinterpret_cast<uint4*>(sPT + (ch >> 3) * 16384 + sw128_offset(row, ch & 7)) = w;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_pt_full);

      // ---- dS^T row
      ok = ok && mbar_wait(bar_dpt_full, j & 1, abort_flag);
      tc_fence_after();
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float dp[16];
        tmem_ld16(tmem + lane_base + C::COL_DPT + i * 16, dp);
        tmem_wait_ld();
        float ds[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) ds[u] = p[i * 16 + u] * (dp[u] - del_t[i * 16 + u]);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int ch = i * 2 + h;
          uint4 w;
          w.x = pack_bf16(ds[h * 8 + 0], ds[h * 8 + 1]);
          w.y = pack_bf16(ds[h * 8 + 2], ds[h * 8 + 3]);
          w.z = pack_bf16(ds[h * 8 + 4], ds[h * 8 + 5]);
          w.w = pack_bf16(ds[h * 8 + 6], ds[h * 8 + 7]);
          *reinterpret_cast<uint4*>(sDST + (ch >> 3) * 16384 + sw128_offset(row, ch & 7)) = w;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_dst_full);

      // ---- dQ rows: this thread now owns query row `row` of the tile
      ok = ok && mbar_wait(bar_dq_full, j & 1, abort_flag);
      tc_fence_after();
      {
        const int x = x0 + row;
        const bool qvalid = x < a.N;
        const int qn = (q_src == SRC_T) ? (x % a.R) * a.l + x / a.R : x;
        float* dst = a.dq_acc + (static_cast<size_t>(bh) * a.N + (qvalid ? qn : 0)) * D;
#pragma unroll
        for (int i = 0; i < D / 16; ++i) {
          float g[16];
          tmem_ld16(tmem + lane_base + C::COL_ST + i * 16, g);
          tmem_wait_ld();
          if (qvalid) {
#pragma unroll
            for (int u = 0; u < 16; u += 4)
              red_add_v4(dst + i * 16 + u, g[u] * a.scale, g[u + 1] * a.scale, g[u + 2] * a.scale,
                         g[u + 3] * a.scale);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar_dq_free);
    }

    // ------------------------------------------------------------ epilogue
    if (n > 0) {
      ok = ok && mbar_wait(bar_dkv_full, 0, abort_flag);
      tc_fence_after();
    }
    const size_t off = (static_cast<size_t>(bh) * a.N + (kvalid ? knat : 0)) * D;
    bool add = false;
    if (a.add_part == 1) add = true;
    else if (a.add_part == 2) add = (knat % a.l) >= (a.l - a.c);
#pragma unroll
    for (int which = 0; which < 2; ++which) {  // 0: dV, 1: dK
      const uint32_t col = which ? C::COL_DK : C::COL_DV;
      const float mul = which ? a.scale : 1.f;
#pragma unroll
      for (int i = 0; i < D / 16; ++i) {
        float g[16];
        if (n > 0) {
          tmem_ld16(tmem + lane_base + col + i * 16, g);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int u = 0; u < 16; ++u) g[u] = 0.f;
        }
        if (!kvalid) continue;
#pragma unroll
        for (int u = 0; u < 16; ++u) g[u] *= mul;
        if (a.key_view != SRC_N) {
          float* dstp = (which ? a.dk_part : a.dv_part) + off + i * 16;
#pragma unroll
          for (int u = 0; u < 16; u += 4)
            *reinterpret_cast<float4*>(dstp + u) = make_float4(g[u], g[u + 1], g[u + 2], g[u + 3]);
        } else {
          if (add) {
            const float* srcp = (which ? a.dk_part : a.dv_part) + off + i * 16;
#pragma unroll
            for (int u = 0; u < 16; u += 4) {
              const float4 t = *reinterpret_cast<const float4*>(srcp + u);
              g[u] += t.x;
              g[u + 1] += t.y;
              g[u + 2] += t.z;
              g[u + 3] += t.w;
            }
          }
          uint4 w0, w1;
          w0.x = pack_bf16(g[0], g[1]);
          w0.y = pack_bf16(g[2], g[3]);
          w0.z = pack_bf16(g[4], g[5]);
          w0.w = pack_bf16(g[6], g[7]);
          w1.x = pack_bf16(g[8], g[9]);
          w1.y = pack_bf16(g[10], g[11]);
          w1.z = pack_bf16(g[12], g[13]);
          w1.w = pack_bf16(g[14], g[15]);
          uint4* dstp = reinterpret_cast<uint4*>((which ? a.dk : a.dv) + off + i * 16);
          dstp[0] = w0;
          dstp[1] = w1;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<C::TMEM_COLS>(tmem);
  }
}

// Delta[bh, i] = sum_d dO[bh, i, d] * O[bh, i, d] (fp32), and zero the fp32
// dQ accumulator.  D/8 threads per row, 16-byte loads; the row loop is
// warp-uniform so the shuffles always see every lane.
template <int D>
__global__ void __launch_bounds__(256) sa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dO,
                                                         float* __restrict__ delta,
                                                         float* __restrict__ dq_acc, long long rows) {
  constexpr int TPR = D / 8;         // threads per row
  constexpr int RPW = 32 / TPR;      // rows per warp per step
  const int lane = threadIdx.x & 31;
  const int sub = lane % TPR;
  const long long warp_id = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long r0 = warp_id * RPW; r0 < rows; r0 += n_warps * RPW) {
    const long long r = r0 + lane / TPR;
    const bool valid = r < rows;
    float acc = 0.f;
    if (valid) {
      const uint4 a = *reinterpret_cast<const uint4*>(o + r * D + sub * 8);
      const uint4 b = *reinterpret_cast<const uint4*>(dO + r * D + sub * 8);
      const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 fa = __bfloat1622float2(ha[u]);
        const float2 fb = __bfloat1622float2(hb[u]);
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
      }
    }
#pragma unroll
    for (int w = TPR / 2; w >= 1; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w, TPR);
    if (valid) {
      if (sub == 0) delta[r] = acc;
      float4* z = reinterpret_cast<float4*>(dq_acc + r * D + sub * 8);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

// dq (bf16) = dq_acc (fp32, already scaled).
__global__ void __launch_bounds__(256) sa_bwd_final_kernel(const float* __restrict__ acc,
                                                           __nv_bfloat16* __restrict__ dq,
                                                           long long n8) {
  const long long nthreads = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += nthreads) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    uint4 w;
    w.x = pack_bf16(a.x, a.y);
    w.y = pack_bf16(a.z, a.w);
    w.z = pack_bf16(b.x, b.y);
    w.w = pack_bf16(b.z, b.w);
    reinterpret_cast<uint4*>(dq)[i] = w;
  }
}

}  // namespace sa
