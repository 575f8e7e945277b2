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
// view order of its table; it walks the 64-query steps that see it.  Per
// step j:
//   ST_j  = K Q_j^T, dPT_j = V dO_j^T  (keys on TMEM lanes, 64 columns each,
//                                       double-buffered so step j+1's products
//                                       overlap step j's elementwise work)
//   P^T_j (bf16, smem), dS^T_j (bf16, smem) by the elementwise warps
//   dV += P^T_j dO_j,  dK += dS^T_j Q_j   (TMEM accumulators for the CTA)
//   every second step: dQ = dS_pair K for the two steps' 128 queries
//                      (M = 128), read by the dQ warps and added to an fp32
//                      workspace with vector reductions.
// Roles (480 threads): warp 0 producer (TMA for K, V, Q, dO; bulk copy of
// the packed lse/Delta), warp 1 TMEM allocation and lane 0 issue of ST/dPT,
// warps 2..9 elementwise (two groups of four, one warp per TMEM lane quarter
// each, taking alternate steps), warps 10..13 dQ reduction, warp 14 lane 0 issue of dV/dK/dQ.  Two
// issuing threads keep the S products of later steps flowing while dV/dK/dQ
// of earlier steps wait on the elementwise warps.  Warp w may only touch TMEM lanes
// 32*(w%4)..32*(w%4)+31, so every role picks its rows by w%4.
// TMEM columns (NBUF = 2 for D <= 64, 1 for D = 128):
//   ST[b] = b*64, dPT[b] = NBUF*64 + b*64, dV = 2*NBUF*64, dK = dV + D,
//   dQ[b] = dK + D + b*D (two dQ buffers for D <= 64, one for D = 128).
#pragma once

#include "sa_device.cuh"
#include "sa_fwd.cuh"

namespace sa {

struct BwdArgs {
  const int32_t* row_ptr;
  const int32_t* ent;
  const int32_t* order;
  const float2* ld_nat;  // [BH, n_pad] (lse * log2(e), Delta) in natural query order
  const float2* ld_col;  // [BH, n_pad] the same in column-major order (strided)
  int n_pad;             // N rounded up to the 64-query step, padded with (+inf, 0)
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
  static constexpr int TK = 128, TQ = 64;
  static constexpr int NBUF = (D >= 128) ? 1 : 2;      // ST/dPT buffers in TMEM
  // Q/dO ring.  At least 2: the MMA issuer asks for step j's Q/dO before it
  // releases step j-1's (it issues S_j ahead of dV/dK of step j-1).
  static constexpr int STAGES = (D >= 128) ? 2 : 4;
  static constexpr int DST_BUFS = (D >= 128) ? 1 : 2;  // dS^T pair buffers
  static constexpr int ROWB = (D >= 64) ? 128 : 64;
  static constexpr uint64_t SWZ = (D >= 64) ? kSwizzle128 : kSwizzle64;
  static constexpr int SBO = 8 * ROWB;
  static constexpr int KV_BYTES = TK * D * 2;          // 128-key tile
  static constexpr int QS_BYTES = TQ * D * 2;          // 64-query tile
  static constexpr int PT_BYTES = TK * TQ * 2;         // [128 keys][64 queries] bf16 = 16 KiB
  static constexpr int DST_BYTES = 2 * PT_BYTES;       // a pair of steps (2 panels)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_Q = OFF_V + KV_BYTES;
  static constexpr int OFF_DO = OFF_Q + STAGES * QS_BYTES;
  static constexpr int OFF_PT = OFF_DO + STAGES * QS_BYTES;
  static constexpr int OFF_DST = OFF_PT + 2 * PT_BYTES;
  static constexpr int OFF_LD = OFF_DST + DST_BUFS * DST_BYTES;  // float2 [STAGES][64]
  static constexpr int LD_BYTES = TQ * 8;
  static constexpr int OFF_ENT = OFF_LD + STAGES * LD_BYTES;
  static constexpr int OFF_BAR = OFF_ENT + kMaxStagedEnt * 4;
  static constexpr int DQBUF = (D >= 128) ? 1 : 2;       // dQ TMEM buffers
  static constexpr int N_BARS = 1 + 2 * STAGES + 2 * 2 + 2 * 2 + 2 + DST_BUFS + 2 * DQBUF + 1;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int COL_DPT = NBUF * 64;
  static constexpr int COL_DV = 2 * NBUF * 64;
  static constexpr int COL_DK = COL_DV + D;
  static constexpr int COL_DQ = COL_DK + D;
  static constexpr int THREADS = 480;
  static_assert(COL_DQ + DQBUF * D <= TMEM_COLS, "TMEM budget");
  static_assert(STAGES >= 2, "the software-pipelined MMA loop needs two Q/dO stages");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

// K-major operand (rows x D) for k-step kk (16 elements of D).
template <int D>
__device__ __forceinline__ uint64_t bwd_kdesc(uint32_t base, int rows, int kk) {
  using C = BwdCfg<D>;
  constexpr int spp = C::ROWB / 32;
  return make_desc(base + (kk / spp) * rows * C::ROWB + (kk % spp) * 32, 16, C::SBO, C::SWZ);
}
// MN-major operand: N = D contiguous in panels of rows x ROWB, k-step = 16 rows.
template <int D>
__device__ __forceinline__ uint64_t bwd_mndesc(uint32_t base, int rows, int kk) {
  using C = BwdCfg<D>;
  return make_desc(base + kk * 16 * C::ROWB, rows * C::ROWB, C::SBO, C::SWZ);
}
// [128 keys][64 queries] bf16 panel, 128B swizzle: K-major with K = queries.
__device__ __forceinline__ uint64_t pt_kdesc(uint32_t base, int kk) {
  return make_desc(base + kk * 32, 16, 1024, kSwizzle128);
}
// A pair of panels viewed MN-major: M = 128 queries (2 panels), K = keys.
__device__ __forceinline__ uint64_t pair_mndesc(uint32_t base, int kk) {
  return make_desc(base + kk * 2048, 16384, 1024, kSwizzle128);
}

template <int D>
__global__ void __launch_bounds__(480, 1)
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
  float2* sLD = reinterpret_cast<float2*>(smem + C::OFF_LD);
  int32_t* sEnt = reinterpret_cast<int32_t*>(smem + C::OFF_ENT);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_kv = bars;
  uint64_t* bar_qdo_full = bar_kv + 1;                 // [STAGES]
  uint64_t* bar_qdo_empty = bar_qdo_full + C::STAGES;  // [STAGES]
  // s_full / s_free are indexed by step parity (one per elementwise group),
  // not by TMEM buffer: with a single buffer the two groups alternate on it,
  // and a shared barrier could be waited on two phases ahead.
  uint64_t* bar_s_full = bar_qdo_empty + C::STAGES;    // [2]  ST and dPT of a step
  uint64_t* bar_s_free = bar_s_full + 2;               // [2]  elementwise done reading them
  uint64_t* bar_pt_full = bar_s_free + 2;              // [2]
  uint64_t* bar_pt_free = bar_pt_full + 2;             // [2]
  uint64_t* bar_dst_full = bar_pt_free + 2;            // [2]  per step parity
  uint64_t* bar_dst_free = bar_dst_full + 2;           // [DST_BUFS] per pair
  uint64_t* bar_dq_full = bar_dst_free + C::DST_BUFS;  // [DQBUF]
  uint64_t* bar_dq_free = bar_dq_full + C::DQBUF;      // [DQBUF]
  uint64_t* bar_dkv_full = bar_dq_free + C::DQBUF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);

  const int bh = blockIdx.x;  // all heads of the longest tiles first (longest-first balance)
  const int kt = a.order[blockIdx.y];
  const int e0 = a.row_ptr[kt];
  const int n = a.row_ptr[kt + 1] - e0;  // 64-query steps
  const int32_t* gEnt = a.ent + e0;
  stage_entries(sEnt, gEnt, n);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q_src = (a.key_view == SRC_T) ? SRC_T : SRC_N;

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_qdo_full + s, 1);
      mbar_init(bar_qdo_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_s_full + b, 1);
      mbar_init(bar_s_free + b, 128);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_pt_full + b, 128);
      mbar_init(bar_pt_free + b, 1);
      mbar_init(bar_dst_full + b, 128);
    }
    for (int b = 0; b < C::DST_BUFS; ++b) mbar_init(bar_dst_free + b, 1);
    for (int b = 0; b < C::DQBUF; ++b) {
      mbar_init(bar_dq_full + b, 1);
      mbar_init(bar_dq_free + b, 128);
    }
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
    // ------------------------------------------------------------ producer
    if (n > 0) {
      if (lane == 0) {
        mbar_arrive_expect_tx(bar_kv, 2 * C::KV_BYTES);
        load_rows<D>(sK, a.key_view, kt * C::TK, C::TK, bh, &mk_nat, &mk_col, &mk_sum, bar_kv, a.R, a.l, a.c);
        load_rows<D>(sV, a.key_view, kt * C::TK, C::TK, bh, &mv_nat, &mv_col, &mv_sum, bar_kv, a.R, a.l, a.c);
      }
      if (lane == 0) {
        const float2* ld = (q_src == SRC_T ? a.ld_col : a.ld_nat) + static_cast<size_t>(bh) * a.n_pad;
        for (int j = 0; j < n; ++j) {
          const int st = j % C::STAGES;
          if (j >= C::STAGES && !mbar_wait(bar_qdo_empty + st, ((j / C::STAGES) - 1) & 1, abort_flag)) break;
          const int qpos = (entry_at(sEnt, gEnt, j) >> 3) * C::TQ;
          mbar_arrive_expect_tx(bar_qdo_full + st, 2 * C::QS_BYTES + C::LD_BYTES);
          load_rows<D>(sQ + st * C::QS_BYTES, q_src, qpos, C::TQ, bh, &mq_nat, &mq_col, &mq_col,
                       bar_qdo_full + st, a.R, a.l, a.c);
          load_rows<D>(sDO + st * C::QS_BYTES, q_src, qpos, C::TQ, bh, &mdo_nat, &mdo_col, &mdo_col,
                       bar_qdo_full + st, a.R, a.l, a.c);
          bulk_load(sLD + st * C::TQ, ld + qpos, C::LD_BYTES, bar_qdo_full + st);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer: ST_j, dPT_j
    // Runs up to NBUF steps ahead of the elementwise warps; only waits for
    // the step's Q/dO and for its TMEM buffer to be read out.
    if (lane == 0 && n > 0) {
      constexpr uint32_t id_s = make_idesc_bf16(128, C::TQ, false, false);  // N = 64 queries
      const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
      bool ok = mbar_wait(bar_kv, 0, abort_flag);
      for (int j = 0; ok && j < n; ++j) {
        const int st = j % C::STAGES;
        const int b = j % C::NBUF;
        ok = mbar_wait(bar_qdo_full + st, (j / C::STAGES) & 1, abort_flag);
        if (ok && j >= C::NBUF) {  // buffer b was last used by step j - NBUF
          const int jp = j - C::NBUF;
          ok = mbar_wait(bar_s_free + (jp & 1), (jp >> 1) & 1, abort_flag);
        }
        if (!ok) break;
        tc_fence_after();
        const uint32_t q_base = smem_u32(sQ + st * C::QS_BYTES);
        const uint32_t do_base = smem_u32(sDO + st * C::QS_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tmem + b * 64, bwd_kdesc<D>(k_base, C::TK, kk), bwd_kdesc<D>(q_base, C::TQ, kk), id_s,
                      kk > 0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tmem + C::COL_DPT + b * 64, bwd_kdesc<D>(v_base, C::TK, kk),
                      bwd_kdesc<D>(do_base, C::TQ, kk), id_s, kk > 0);
        mma_commit(bar_s_full + (j & 1));
      }
    }
  } else if (warp == 14) {
    // ------------------------------------------------------------ G issuer: dV, dK, dQ
    // Its commits track only its own MMAs; the S issuer's products of a step
    // are complete before the step's P^T exists, so releasing the Q/dO stage
    // after dK covers both issuers.
    if (lane == 0 && n > 0) {
      constexpr uint32_t id_kv = make_idesc_bf16(128, D, false, true);  // dV, dK
      constexpr uint32_t id_q = make_idesc_bf16(128, D, true, true);    // dQ (pair)
      const uint32_t k_base = smem_u32(sK);
      bool ok = mbar_wait(bar_kv, 0, abort_flag);
      for (int jj = 0; ok && jj < n; ++jj) {
        const int st = jj % C::STAGES;
        const int pb = jj & 1;
        const int pair = jj >> 1;
        const uint32_t q_base = smem_u32(sQ + st * C::QS_BYTES);
        const uint32_t do_base = smem_u32(sDO + st * C::QS_BYTES);
        const uint32_t dst_pair = smem_u32(sDST + (pair % C::DST_BUFS) * C::DST_BYTES);
        if (!mbar_wait(bar_pt_full + pb, (jj >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t pt_base = smem_u32(sPT + pb * C::PT_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::TQ / 16; ++kk)
          mma_bf16_ss(tmem + C::COL_DV, pt_kdesc(pt_base, kk), bwd_mndesc<D>(do_base, C::TQ, kk), id_kv,
                      (jj > 0 || kk > 0));
        mma_commit(bar_pt_free + pb);
        if (!mbar_wait(bar_dst_full + pb, (jj >> 1) & 1, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::TQ / 16; ++kk)
          mma_bf16_ss(tmem + C::COL_DK, pt_kdesc(dst_pair + pb * C::PT_BYTES, kk),
                      bwd_mndesc<D>(q_base, C::TQ, kk), id_kv, (jj > 0 || kk > 0));
        mma_commit(bar_qdo_empty + st);
        if ((jj & 1) || jj == n - 1) {
          const int qb = pair % C::DQBUF;
          if (pair >= C::DQBUF && !mbar_wait(bar_dq_free + qb, ((pair / C::DQBUF) - 1) & 1, abort_flag)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < C::TK / 16; ++kk)
            mma_bf16_ss(tmem + C::COL_DQ + qb * D, pair_mndesc(dst_pair, kk), bwd_mndesc<D>(k_base, C::TK, kk),
                        id_q, kk > 0);
          mma_commit(bar_dq_full + qb);
          mma_commit(bar_dst_free + (pair % C::DST_BUFS));
        }
      }
      mma_commit(bar_dkv_full);
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------ elementwise
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;  // step parity of this group; dV/dK column half in the epilogue
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int y = kt * C::TK + row;  // this thread's key, view order
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

    // Group `half` takes the steps j with j % 2 == half, each thread a whole
    // 64-query row in chunks of 16 columns; the two groups run out of phase,
    // so one group's exp2 (MUFU) work overlaps the other's dS (ALU) work.
    bool ok = true;
    for (int j = half; j < n; j += 2) {
      const int e = entry_at(sEnt, gEnt, j);
      const int st = j % C::STAGES;
      const int b = j % C::NBUF;
      const int pb = j & 1;
      const int pair = j >> 1;
      const bool partial = e & 1;
      const int x0 = (e >> 3) * C::TQ;
      ok = ok && mbar_wait(bar_qdo_full + st, (j / C::STAGES) & 1, abort_flag);
      ok = ok && mbar_wait(bar_s_full + pb, (j >> 1) & 1, abort_flag);
      // P^T buffer pb is free once dV of step j-2 has completed; dS^T pair
      // buffer once dQ of pair - DST_BUFS has completed.
      if (j >= 2) ok = ok && mbar_wait(bar_pt_free + pb, ((j >> 1) - 1) & 1, abort_flag);
      if (pair >= C::DST_BUFS)
        ok = ok && mbar_wait(bar_dst_free + (pair % C::DST_BUFS), ((pair / C::DST_BUFS) - 1) & 1, abort_flag);
      tc_fence_after();
      const float4* ld_t = reinterpret_cast<const float4*>(sLD + st * C::TQ);  // (lse*log2 e, Delta) x 2
      uint8_t* pt = sPT + pb * C::PT_BYTES;
      uint8_t* dst = sDST + (pair % C::DST_BUFS) * C::DST_BYTES + pb * C::PT_BYTES;
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        float p[16], dp[16];
        tmem_ld16(tmem + lane_base + b * 64 + c16 * 16, p);
        tmem_ld16(tmem + lane_base + C::COL_DPT + b * 64 + c16 * 16, dp);
        tmem_wait_ld();
        if (c16 == 3) {  // both TMEM buffers of this step have been read
          tc_fence_before();
          mbar_arrive(bar_s_free + pb);
        }
        float lse2[16], dl[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 t = ld_t[c16 * 8 + i];
          lse2[2 * i] = t.x;
          dl[2 * i] = t.y;
          lse2[2 * i + 1] = t.z;
          dl[2 * i + 1] = t.w;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float v = ex2(fmaf(p[i], a.scale_log2, -lse2[i]));
          if (partial) {
            const int x = x0 + c16 * 16 + i;
            if (x < qlo || x > qhi) v = 0.f;
          }
          p[i] = v;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint4 w;
          w.x = pack_bf16(p[h * 8 + 0], p[h * 8 + 1]);
          w.y = pack_bf16(p[h * 8 + 2], p[h * 8 + 3]);
          w.z = pack_bf16(p[h * 8 + 4], p[h * 8 + 5]);
          w.w = pack_bf16(p[h * 8 + 6], p[h * 8 + 7]);
          *reinterpret_cast<uint4*>(pt + sw128_offset(row, c16 * 2 + h)) = w;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float d8[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) d8[u] = p[h * 8 + u] * (dp[h * 8 + u] - dl[h * 8 + u]);
          uint4 w;
          w.x = pack_bf16(d8[0], d8[1]);
          w.y = pack_bf16(d8[2], d8[3]);
          w.z = pack_bf16(d8[4], d8[5]);
          w.w = pack_bf16(d8[6], d8[7]);
          *reinterpret_cast<uint4*>(dst + sw128_offset(row, c16 * 2 + h)) = w;
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bar_pt_full + pb);
      mbar_arrive(bar_dst_full + pb);
    }

    // ------------------------------------------------------------ epilogue (dV, dK)
    if (n > 0) {
      ok = ok && mbar_wait(bar_dkv_full, 0, abort_flag);
      tc_fence_after();
    }
    const size_t off = (static_cast<size_t>(bh) * a.N + (kvalid ? knat : 0)) * D;
    bool add = false;
    if (a.add_part == 1) add = true;
    else if (a.add_part == 2) add = (knat % a.l) >= (a.l - a.c);
    constexpr int HC = D / 2;  // columns per half
#pragma unroll
    for (int which = 0; which < 2; ++which) {  // 0: dV, 1: dK
      const uint32_t col = (which ? C::COL_DK : C::COL_DV) + half * HC;
      const float mul = which ? a.scale : 1.f;
#pragma unroll
      for (int i = 0; i < HC / 16; ++i) {
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
        const size_t eo = off + half * HC + i * 16;
        if (a.key_view != SRC_N) {
          float* dstp = (which ? a.dk_part : a.dv_part) + eo;
#pragma unroll
          for (int u = 0; u < 16; u += 4)
            *reinterpret_cast<float4*>(dstp + u) = make_float4(g[u], g[u + 1], g[u + 2], g[u + 3]);
        } else {
          if (add) {
            const float* srcp = (which ? a.dk_part : a.dv_part) + eo;
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
          uint4* dstp = reinterpret_cast<uint4*>((which ? a.dk : a.dv) + eo);
          dstp[0] = w0;
          dstp[1] = w1;
        }
      }
    }
  } else if (warp < 14) {
    // ------------------------------------------------------------ dQ reduction
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // query row of the pair: step 2p + row / 64
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int n_pairs = (n + 1) >> 1;
    bool ok = true;
    for (int p = 0; p < n_pairs; ++p) {
      const int qb = p % C::DQBUF;
      ok = ok && mbar_wait(bar_dq_full + qb, (p / C::DQBUF) & 1, abort_flag);
      tc_fence_after();
      const int s = 2 * p + (row >> 6);
      bool qvalid = false;
      float* dstp = a.dq_acc;
      if (s < n) {
        const int x = (entry_at(sEnt, gEnt, s) >> 3) * C::TQ + (row & 63);
        qvalid = x < a.N;
        const int qn = (q_src == SRC_T) ? (x % a.R) * a.l + x / a.R : x;
        dstp = a.dq_acc + (static_cast<size_t>(bh) * a.N + (qvalid ? qn : 0)) * D;
      }
#pragma unroll
      for (int i = 0; i < D / 16; ++i) {
        float g[16];
        tmem_ld16(tmem + lane_base + C::COL_DQ + qb * D + i * 16, g);
        tmem_wait_ld();
        if (qvalid) {
#pragma unroll
          for (int u = 0; u < 16; u += 4)
            red_add_v4(dstp + i * 16 + u, g[u] * a.scale, g[u + 1] * a.scale, g[u + 2] * a.scale,
                       g[u + 3] * a.scale);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_dq_free + qb);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<C::TMEM_COLS>(tmem);
  }
}

// Backward preprocess, one row per D/8 threads (16-byte loads; the row loop
// is warp-uniform so the shuffles always see every lane):
//   Delta_i = sum_d dO_id O_id (fp32); writes (lse_i * log2 e, Delta_i) to the
//   natural-order array and, for the strided pattern, at the row's
//   column-major position t = (i mod l) * R + i / l; pads positions
//   [N, n_pad) of both with (+inf, 0); zeroes the fp32 dQ accumulator.
template <int D>
__global__ void __launch_bounds__(256) sa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dO,
                                                         const float* __restrict__ lse,
                                                         float2* __restrict__ ld_nat, float2* __restrict__ ld_col,
                                                         float* __restrict__ dq_acc, int BH, int N, int n_pad,
                                                         int l, int R) {
  constexpr int TPR = D / 8;         // threads per row
  constexpr int RPW = 32 / TPR;      // rows per warp per step
  const long long rows = static_cast<long long>(BH) * N;
  const int lane = threadIdx.x & 31;
  const int sub = lane % TPR;
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long nthr = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long warp_id = tid >> 5;
  const long long n_warps = nthr >> 5;
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
      if (sub == 0) {
        const long long bh = r / N;
        const int i = static_cast<int>(r - bh * N);
        const float2 v = make_float2(lse[r] * 1.4426950408889634f, acc);
        ld_nat[bh * n_pad + i] = v;
        if (ld_col) ld_col[bh * n_pad + (i % l) * R + i / l] = v;
      }
      float4* z = reinterpret_cast<float4*>(dq_acc + r * D + sub * 8);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  const int pad = n_pad - N;
  for (long long k = tid; k < static_cast<long long>(BH) * pad; k += nthr) {
    const long long bh = k / pad;
    const long long i = N + (k - bh * pad);
    ld_nat[bh * n_pad + i] = make_float2(INFINITY, 0.f);
    if (ld_col) ld_col[bh * n_pad + i] = make_float2(INFINITY, 0.f);
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
