// Forward kernel: fused online-softmax block-sparse attention on tcgen05.
//
// Persistent: each CTA walks a zig-zag share of the items (128-row query
// tile, batch*head) of its table, longest tiles first; an item is a query
// tile in the view order of its table (natural, or column-major for the
// strided column view) and its list of 64-key tiles.  The loads of the next
// item's tiles run while the current one finishes.  Per key tile:
//   S = Q K^T            tcgen05.mma, bf16 in smem -> fp32 in TMEM
//   mask (PARTIAL only), running max, P = exp2(S*scale*log2e - m) -> bf16,
//                        written back into TMEM over its own S columns
//   O += P V             tcgen05.mma with A = P read from TMEM
// This is masked softmax attention restricted to the nonzero blocks of the
// layout ("OpenAI Sparse Transformer", "Sparse Attention and Algorithmic
// Complexity" and "Implementation and Limitations").
//
// Roles (224 threads):
//   warp 0 lane 0 : TMA producer (Q once, K/V through a STAGES-deep ring)
//   warp 1        : allocates TMEM; lane 0 issues S = Q K^T
//   warps 2..5    : softmax; thread t of warp w owns query row
//                   32*(w%4)+t, which is TMEM lane 32*(w%4)+t
//   warp 6 lane 0 : issues O += P V (a second issuing thread, so S of the
//                   next tiles never waits behind PV of earlier ones)
// TMEM columns: S double buffer [0,64) and [64,128) (P of a tile occupies the
// first 32 columns of its S buffer, two bf16 per column); two O accumulators
// [128,128+D) and [128+D,128+2D) taken by item parity, so the next item's PV
// products run while the epilogue reads the previous O.  An S buffer is
// reused once PV of its tile has completed.
//
// The running max is only moved when it grows by more than 2^8 (in the
// exp2 domain), so O is rescaled rarely; the final normalisation uses the
// same max, so the result is exact up to rounding.
#pragma once

#include "sa_device.cuh"

namespace sa {

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

struct FwdArgs {
  const int32_t* row_ptr;
  const int32_t* ent;
  const int32_t* order;
  __nv_bfloat16* o;
  float* lse;
  int N, l, c, R;
  int pattern;  // sa_pattern
  int q_col;    // 1: query tiles are in column-major (T) order
  int merge;    // 1: combine with the partial (o, lse) already stored
  int t_open;   // column view: 1 when it excludes the diagonal (SA_STRIDED), 0 when it stands alone
  int n_rows, BH;  // items = n_rows * BH, slot-major (all heads of a launch slot together)
  float scale_log2;
  BoxSet box;  // column / summary TMA boxes per tile height
  const uint32_t* bits;  // sub-block bits per entry (caller block masks with blocks below a tile)
  int blk;               // their block size (16, 32 or 64), else 0
};

template <int D>
struct FwdCfg {
  static constexpr int TQ = 128, TK = 64;
  static constexpr int STAGES = (D >= 128) ? 3 : ((D == 64) ? 4 : 6);
  static constexpr int ROWB = (D >= 64) ? 128 : 64;     // bytes per row per panel
  static constexpr int PANELS = (D >= 64) ? D / 64 : 1;
  static constexpr int BOXW = (D >= 64) ? 64 : D;       // TMA box inner width (elements)
  static constexpr uint64_t SWZ = (D >= 64) ? kSwizzle128 : kSwizzle64;
  static constexpr int SBO = 8 * ROWB;
  static constexpr int Q_BYTES = TQ * D * 2;
  static constexpr int KV_BYTES = TK * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_STG = OFF_V + STAGES * KV_BYTES;  // epilogue: 32 output rows per softmax warp
  static constexpr int OFF_BAR = OFF_STG + TQ * D * 2;
  static constexpr int N_BARS = 2 + 3 * STAGES + 8 + 2 + 4 + 2;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
  static constexpr int TMEM_COLS = (128 + 2 * D <= 256) ? 256 : 512;
  static constexpr int COL_O = 128;  // + (item parity) * D
  static constexpr int THREADS = 224;
};

// Loads a tile of `rows` positions starting at view position `pos0` into
// `dst` (PANELS panels of rows x ROWB bytes).
//   src N: natural order, 3-D map {D, N, BH}, box {BOXW, rows, 1}
//   src T: column-major order, 4-D map {D, l, R, BH}, box {BOXW, 1, RB, 1}
//          with RB = gcd(R, rows): one load per RB rows of a column
//   src S: summary order, 4-D map {D, l, R, BH}, box {BOXW, CB, GB, 1} from
//          summary_box(c, rows): whole blocks, or runs inside one block
template <int D>
__device__ __forceinline__ void load_rows(uint8_t* dst, int src, int pos0, int rows, int bh,
                                          const CUtensorMap* m_nat, const CUtensorMap* m_col,
                                          const CUtensorMap* m_sum, uint64_t* bar, int R, int l,
                                          int c, const BoxGeo& bg) {
  using C = FwdCfg<D>;
  const int panel_bytes = rows * C::ROWB;
#pragma unroll
  for (int p = 0; p < C::PANELS; ++p) {
    uint8_t* d = dst + p * panel_bytes;
    const int x = p * 64;
    if (src == SRC_N) {
      tma_load_3d(d, m_nat, bar, x, pos0, bh);
    } else if (src == SRC_T) {
      const int rb = bg.rb_t;
      for (int s = 0; s < rows; s += rb) {
        const int t = pos0 + s;
        tma_load_4d(d + s * C::ROWB, m_col, bar, x, t / R, t % R, bh);
      }
    } else {
      const int cb = bg.cb_s;
      if (bg.gb_s > 1 || cb == c) {  // whole blocks
        tma_load_4d(d, m_sum, bar, x, l - c, pos0 / c, bh);
      } else {  // runs of cb keys inside one block
        for (int s = 0; s < rows; s += cb) {
          const int y = pos0 + s;
          tma_load_4d(d + s * C::ROWB, m_sum, bar, x, l - c + y % c, y / c, bh);
        }
      }
    }
  }
}

// K-major operand descriptor for k-step kk (16 elements of K) of a tile with
// PANELS panels of `rows` rows.
template <int D>
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int rows, int kk) {
  using C = FwdCfg<D>;
  constexpr int steps_per_panel = C::ROWB / 32;
  const int panel = kk / steps_per_panel;
  const int within = (kk % steps_per_panel) * 32;
  return make_desc(base + panel * rows * C::ROWB + within, 16, C::SBO, C::SWZ);
}

// MN-major operand descriptor (N = D contiguous in panels of rows x ROWB),
// for k-step kk = 16 rows of K.
template <int D>
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t base, int rows, int kk) {
  using C = FwdCfg<D>;
  return make_desc(base + kk * 16 * C::ROWB, rows * C::ROWB, C::SBO, C::SWZ);
}

// Item k of a CTA's share: zig-zag rounds over the items (launch slots sorted
// longest first, all heads of a slot together), so long and short tiles pair up.
__device__ __forceinline__ int fwd_item(int k, int cta, int n_ctas) {
  return k * n_ctas + ((k & 1) ? (n_ctas - 1 - cta) : cta);
}

struct FwdItem {
  int bh, qt, e0, n;
};

__device__ __forceinline__ FwdItem fwd_item_of(const FwdArgs& a, int item) {
  const int slot = item / a.BH;
  const int qt = a.order[slot];
  const int e0 = a.row_ptr[qt];
  return FwdItem{item - slot * a.BH, qt, e0, a.row_ptr[qt + 1] - e0};
}

// BLK: a caller block mask whose blocks are smaller than a tile (the
// entries' sub-block bits are applied on PARTIAL tiles).
template <int D, bool BLK = false>
__global__ void __launch_bounds__(224, (D <= 64) ? 2 : 1)
    sa_fwd_kernel(const __grid_constant__ CUtensorMap mq_nat, const __grid_constant__ CUtensorMap mq_col,
                  const __grid_constant__ CUtensorMap mk_nat, const __grid_constant__ CUtensorMap mk_col,
                  const __grid_constant__ CUtensorMap mk_sum, const __grid_constant__ CUtensorMap mv_nat,
                  const __grid_constant__ CUtensorMap mv_col, const __grid_constant__ CUtensorMap mv_sum,
                  const __grid_constant__ CUtensorMap mo_nat, const __grid_constant__ CUtensorMap mo_col,
                  const FwdArgs a) {
  using C = FwdCfg<D>;
#ifdef SA_TEST_HOOKS
  pdl_wait();  // the range check of the tables (previous kernel) has completed
  if (*(volatile int*)&g_status == kStatusLut) return;  // a table failed it: touch nothing
#endif
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_q = bars;                           // Q of an item landed
  uint64_t* bar_q_free = bars + 1;                  // every S product of the item has completed
  uint64_t* bar_k_full = bars + 2;
  uint64_t* bar_v_full = bar_k_full + C::STAGES;
  uint64_t* bar_kv_empty = bar_v_full + C::STAGES;
  uint64_t* bar_s_full = bar_kv_empty + C::STAGES;  // [2]
  uint64_t* bar_s_empty = bar_s_full + 2;           // [2]  PV of the buffer's tile done
  uint64_t* bar_p_full = bar_s_empty + 2;           // [2]  P written into TMEM
  uint64_t* bar_pv_done = bar_p_full + 2;           // [2]
  uint64_t* bar_o_free = bar_pv_done + 2;           // [2]  the epilogue has read O of the buffer's item
  uint64_t* bar_epi = bar_o_free + 2;               // [4]  old O rows of a merge landed (per warp)
  uint64_t* bar_drain = bar_epi + 4;                // [2]  each issuer's last commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = a.n_rows * a.BH;
  const int cta = blockIdx.x, n_ctas = gridDim.x;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_q_free, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_k_full + s, 1);
      mbar_init(bar_v_full + s, 1);
      mbar_init(bar_kv_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_s_full + s, 1);
      mbar_init(bar_s_empty + s, 1);
      mbar_init(bar_p_full + s, 128);
      mbar_init(bar_pv_done + s, 1);
      mbar_init(bar_o_free + s, 128);
    }
    for (int w = 0; w < 4; ++w) mbar_init(bar_epi + w, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_drain + 1, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc<C::TMEM_COLS>(tmem_slot);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  // Every role walks the same items in the same order; tile and item
  // counters (jg: key tiles, ta: items with at least one tile) continue
  // across items, so barrier phases follow them.
  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      const CUtensorMap* mq = a.q_col ? &mq_col : &mq_nat;
      bool ok = true;
      int jg = 0, ta = 0;
      for (int k = 0, item = cta; ok && item < n_items; item = fwd_item(++k, cta, n_ctas)) {
        const FwdItem it = fwd_item_of(a, item);
        if (it.n == 0) continue;
        // Q of this item once every S product of the previous one has completed
        if (ta >= 1 && !mbar_wait(bar_q_free, (ta - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
        load_rows<D>(sQ, a.q_col ? SRC_T : SRC_N, it.qt * C::TQ, C::TQ, it.bh, mq, mq, mq, bar_q, a.R,
                     a.l, a.c, a.box.b[box_index(C::TQ)]);
        ++ta;
        for (int j = 0; j < it.n; ++j, ++jg) {
          const int st = jg % C::STAGES;
          if (jg >= C::STAGES && !mbar_wait(bar_kv_empty + st, ((jg / C::STAGES) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int e = a.ent[it.e0 + j];
          const int src = (e >> 1) & 3;
          const int kpos = (e >> 3) * C::TK;
          mbar_arrive_expect_tx(bar_k_full + st, C::KV_BYTES);
          load_rows<D>(sK + st * C::KV_BYTES, src, kpos, C::TK, it.bh, &mk_nat, &mk_col, &mk_sum,
                       bar_k_full + st, a.R, a.l, a.c, a.box.b[box_index(C::TK)]);
          mbar_arrive_expect_tx(bar_v_full + st, C::KV_BYTES);
          load_rows<D>(sV + st * C::KV_BYTES, src, kpos, C::TK, it.bh, &mv_nat, &mv_col, &mv_sum,
                       bar_v_full + st, a.R, a.l, a.c, a.box.b[box_index(C::TK)]);
        }
      }
      // After an abort, wait (bounded) for the loads still in flight, so that
      // no copy lands in shared memory after the CTA has exited.
      if (*(volatile int*)abort_flag) {
        if (ta >= 1) mbar_wait_drain(bar_q, (ta - 1) & 1);
        for (int h = jg > C::STAGES ? jg - C::STAGES : 0; h < jg; ++h) {
          mbar_wait_drain(bar_k_full + h % C::STAGES, (h / C::STAGES) & 1);
          mbar_wait_drain(bar_v_full + h % C::STAGES, (h / C::STAGES) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer: S_j = Q K_j^T
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc_bf16(128, C::TK, false, false);
      const uint32_t q_base = smem_u32(sQ);
      bool ok = true;
      int jg = 0, ta = 0;
      for (int k = 0, item = cta; ok && item < n_items; item = fwd_item(++k, cta, n_ctas)) {
        const FwdItem it = fwd_item_of(a, item);
        if (it.n == 0) continue;
        ok = mbar_wait(bar_q, ta & 1, abort_flag);
        for (int j = 0; ok && j < it.n; ++j, ++jg) {
          const int st = jg % C::STAGES;
          const int sb = jg & 1;
          ok = mbar_wait(bar_k_full + st, (jg / C::STAGES) & 1, abort_flag);
          if (ok && jg >= 2) ok = mbar_wait(bar_s_empty + sb, ((jg >> 1) - 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t k_base = smem_u32(sK + st * C::KV_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(tmem + sb * C::TK, kmajor_desc<D>(q_base, C::TQ, kk), kmajor_desc<D>(k_base, C::TK, kk),
                        idesc_qk, kk > 0);
          mma_commit(bar_s_full + sb);
        }
        mma_commit(bar_q_free);  // Q may be replaced once these products have completed
        ++ta;
      }
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ PV issuer: O += P_j V_j
    // S_j has completed before P_j exists, so this thread's commit after PV_j
    // also releases the K half of the stage and the S/P buffer of the tile.
    if (lane == 0) {
      constexpr uint32_t idesc_pv = make_idesc_bf16(128, D, false, true);
      bool ok = true;
      int jg = 0, ta = 0;
      for (int k = 0, item = cta; ok && item < n_items; item = fwd_item(++k, cta, n_ctas)) {
        const FwdItem it = fwd_item_of(a, item);
        if (it.n == 0) continue;
        const int ob = ta & 1;
        // O buffer ob once the epilogue of the item two before has read it
        if (ta >= 2) ok = mbar_wait(bar_o_free + ob, ((ta >> 1) - 1) & 1, abort_flag);
        for (int j = 0; ok && j < it.n; ++j, ++jg) {
          const int st = jg % C::STAGES;
          const int pb = jg & 1;
          ok = mbar_wait(bar_p_full + pb, (jg >> 1) & 1, abort_flag) &&
               mbar_wait(bar_v_full + st, (jg / C::STAGES) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t v_base = smem_u32(sV + st * C::KV_BYTES);
#pragma unroll
          for (int kk = 0; kk < C::TK / 16; ++kk)  // 16 keys of P = 8 TMEM columns per k-step
            mma_bf16_ts(tmem + C::COL_O + ob * D, tmem + pb * C::TK + kk * 8, mnmajor_desc<D>(v_base, C::TK, kk),
                        idesc_pv, (j > 0 || kk > 0));
          mma_commit(bar_pv_done + pb);
          mma_commit(bar_s_empty + pb);
          mma_commit(bar_kv_empty + st);
        }
        ++ta;
      }
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(bar_drain + 1);
      mbar_wait_drain(bar_drain + 1, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    uint8_t* stg = smem + C::OFF_STG + quarter * (32 * D * 2);  // this warp's 32 output rows
    constexpr int PB = 32 * C::ROWB;                            // one 32-row panel
    bool ok = true;
    int jg = 0, ta = 0, epi_n = 0;
    for (int k = 0, item = cta; ok && item < n_items; item = fwd_item(++k, cta, n_ctas)) {
      const FwdItem it = fwd_item_of(a, item);
      const int x = it.qt * C::TQ + row;  // view position of this query
      const bool valid = x < (a.q_col ? a.R * a.l : a.N);  // the column view covers whole rows
      const int nat = a.q_col ? (x % a.R) * a.l + x / a.R : x;
      const int ob = ta & 1;
      const uint32_t col_o = C::COL_O + ob * D;

      float m_used = -INFINITY;
      float l_sum = 0.f;
      int e_next = it.n > 0 ? a.ent[it.e0] : 0;
      for (int j = 0; j < it.n; ++j, ++jg) {
        const int sb = jg & 1;
        const int e = e_next;
        if (j + 1 < it.n) e_next = a.ent[it.e0 + j + 1];
        ok = ok && mbar_wait(bar_s_full + sb, (jg >> 1) & 1, abort_flag);
        tc_fence_after();
        float s[C::TK];
#pragma unroll
        for (int i = 0; i < C::TK / 16; ++i) tmem_ld16(tmem + lane_base + sb * C::TK + i * 16, s + i * 16);
        tmem_wait_ld();

        if (e & 1) {
          // the row's key interval in the tile's source view (inclusive)
          const int src = (e >> 1) & 3;
          const int k0 = (e >> 3) * C::TK;
          int lo, hi;
          if (src == SRC_T) {
            lo = (x / a.R) * a.R;
            hi = x - a.t_open;
          } else if (src == SRC_S) {
            lo = 0;
            hi = (nat / a.l) * a.c - 1;
          } else {
            lo = (a.pattern == SA_ALL) ? 0 : (a.pattern == SA_FIXED ? (nat / a.l) * a.l : max(0, nat - a.l + 1));
            hi = nat;
          }
          static_assert(C::TK == 64, "interval mask of 64 keys");
          if constexpr (BLK) {
            const int nj = C::TK / a.blk;
            const uint32_t nib = (a.bits[it.e0 + j] >> ((row / a.blk) * nj)) & ((1u << nj) - 1u);
            mask_bits64(s, interval_bits64(lo - k0, hi - k0) & sub_block_cols(nib, a.blk), -INFINITY);
          } else {
            mask_interval64(s, lo - k0, hi - k0, -INFINITY);
          }
        }
        // row max as a tree of three-input maxima (short dependency chains)
        float m21[21];
#pragma unroll
        for (int u = 0; u < 21; ++u) m21[u] = max3f(s[3 * u], s[3 * u + 1], s[3 * u + 2]);
        float m7[7];
#pragma unroll
        for (int u = 0; u < 7; ++u) m7[u] = max3f(m21[3 * u], m21[3 * u + 1], m21[3 * u + 2]);
        const float mx = max3f(max3f(m7[0], m7[1], m7[2]), max3f(m7[3], m7[4], m7[5]), fmaxf(m7[6], s[63]));
        const float m_tile = mx * a.scale_log2;
        float factor = 1.f;
        if (m_tile > m_used + 8.f) {
          factor = (m_used == -INFINITY) ? 0.f : ex2(m_used - m_tile);
          m_used = m_tile;
        }
        // Rescale the O accumulator (only after the item's first tile, only if needed).
        if (j > 0 && __any_sync(0xffffffffu, factor != 1.f)) {
          const int jp = jg - 1;
          ok = ok && mbar_wait(bar_pv_done + (jp & 1), (jp >> 1) & 1, abort_flag);
          tc_fence_after();
#pragma unroll
          for (int i = 0; i < D / 16; ++i) {
            float ov[16];
            tmem_ld16(tmem + lane_base + col_o + i * 16, ov);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 16; ++u) ov[u] *= factor;
            tmem_st16(tmem + lane_base + col_o + i * 16, ov);
          }
          tmem_wait_st();
        }
        const float neg = (m_used == -INFINITY) ? 0.f : -m_used;
        uint64_t rs2[4] = {0, 0, 0, 0};  // partial row sums, fp32 pairs
        const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2), ng2 = f2_pack(neg, neg);
        uint32_t pk[C::TK / 2];
#pragma unroll
        for (int ch = 0; ch < C::TK / 8; ++ch) {
          float p[8];
#pragma unroll
          for (int u = 0; u < 8; u += 2) {
            const float2 t = f2_unpack(f2_fma(f2_pack(s[ch * 8 + u], s[ch * 8 + u + 1]), sc2, ng2));
            p[u] = ex2(t.x);
            p[u + 1] = ex2(t.y);
            rs2[u / 2] = f2_add(rs2[u / 2], f2_pack(p[u], p[u + 1]));
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) pk[ch * 4 + u] = pack_bf16(p[2 * u], p[2 * u + 1]);
        }
        float rs8[8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 t = f2_unpack(rs2[u]);
          rs8[2 * u] = t.x;
          rs8[2 * u + 1] = t.y;
        }
        // P over the first TK/2 columns of its own S buffer (the S values are in registers)
        tmem_st32(tmem + lane_base + sb * C::TK, pk);
        tmem_wait_st();
        const float rsum = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
        l_sum = l_sum * factor + rsum;
        tc_fence_before();
        mbar_arrive(bar_p_full + sb);
      }

      // ------------------------------------------------------------ epilogue of the item
      float inv = 0.f, lse_row = -INFINITY;
      if (l_sum > 0.f) {
        inv = 1.f / l_sum;
        lse_row = (m_used + lg2(l_sum)) * 0.6931471805599453f;
      }
      if (it.n > 0) {
        const int jl = jg - 1;
        ok = ok && mbar_wait(bar_pv_done + (jl & 1), (jl >> 1) & 1, abort_flag);
        tc_fence_after();
      }
      float w_new = 1.f, w_old = 0.f, lse_out = lse_row;
      if (a.merge && valid) {
        const float lse_old = a.lse[static_cast<size_t>(it.bh) * a.N + nat];
        const float mm = fmaxf(lse_row, lse_old);
        if (mm == -INFINITY) {
          w_new = 0.f;
          w_old = 0.f;
        } else {
          const float en = ex2((lse_row - mm) * 1.4426950408889634f);
          const float eo = ex2((lse_old - mm) * 1.4426950408889634f);
          const float tot = en + eo;
          w_new = en / tot;
          w_old = eo / tot;
          lse_out = mm + lg2(tot) * 0.6931471805599453f;
        }
      }
      // Rows go out through this warp's staging buffer: a merge first brings
      // the stored O rows in by TMA, each thread blends its own row in place,
      // and one TMA store per warp (per 64-column panel) writes the 32 rows in
      // the tile's view order.
      const int xw = it.qt * C::TQ + quarter * 32;  // view position of the warp's first row
      if (lane == 0) bulk_wait_read_all();         // the previous item's store has read the staging
      __syncwarp();
      if (a.merge) {
        if (lane == 0) {
          mbar_arrive_expect_tx(bar_epi + quarter, 32 * D * 2);
#pragma unroll
          for (int p = 0; p < C::PANELS; ++p)
            tma_load_3d(stg + p * PB, &mo_nat, bar_epi + quarter, p * 64, xw, it.bh);
        }
        ok = ok && mbar_wait(bar_epi + quarter, epi_n & 1, abort_flag);
        ++epi_n;
      }
#pragma unroll
      for (int i = 0; i < D / 16; ++i) {
        float ov[16];
        if (it.n > 0) {
          tmem_ld16(tmem + lane_base + col_o + i * 16, ov);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int u = 0; u < 16; ++u) ov[u] = 0.f;
        }
        if (it.n > 0 && i == D / 16 - 1) {
          tc_fence_before();
          mbar_arrive(bar_o_free + ob);  // O of this item has been read
        }
        // the two 16-byte chunks of columns [16i, 16i + 16) in the swizzled row
        const int ch = (i * 2) % (C::ROWB / 16);
        const int pnl = (i * 16) / 64;
        uint8_t* c0 = stg + (D >= 64 ? pnl * PB + sw128_offset(lane, ch) : sw64_offset(lane, ch));
        uint8_t* c1 = stg + (D >= 64 ? pnl * PB + sw128_offset(lane, ch + 1) : sw64_offset(lane, ch + 1));
        float r[16];
        if (a.merge) {
          const uint4 o0 = *reinterpret_cast<const uint4*>(c0), o1 = *reinterpret_cast<const uint4*>(c1);
          const __nv_bfloat162* h0 = reinterpret_cast<const __nv_bfloat162*>(&o0);
          const __nv_bfloat162* h1 = reinterpret_cast<const __nv_bfloat162*>(&o1);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 f0 = __bfloat1622float2(h0[u]);
            const float2 f1 = __bfloat1622float2(h1[u]);
            r[2 * u] = w_new * ov[2 * u] * inv + w_old * f0.x;
            r[2 * u + 1] = w_new * ov[2 * u + 1] * inv + w_old * f0.y;
            r[8 + 2 * u] = w_new * ov[8 + 2 * u] * inv + w_old * f1.x;
            r[8 + 2 * u + 1] = w_new * ov[8 + 2 * u + 1] * inv + w_old * f1.y;
          }
        } else {
#pragma unroll
          for (int u = 0; u < 16; ++u) r[u] = ov[u] * inv;
        }
        *reinterpret_cast<uint4*>(c0) =
            make_uint4(pack_bf16(r[0], r[1]), pack_bf16(r[2], r[3]), pack_bf16(r[4], r[5]), pack_bf16(r[6], r[7]));
        *reinterpret_cast<uint4*>(c1) = make_uint4(pack_bf16(r[8], r[9]), pack_bf16(r[10], r[11]),
                                                   pack_bf16(r[12], r[13]), pack_bf16(r[14], r[15]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int p = 0; p < C::PANELS; ++p) {
          if (a.q_col) {
            const int rb = a.box.b[0].rb_t;
            for (int s0 = 0; s0 < 32; s0 += rb) {
              const int t = xw + s0;
              tma_store_4d(&mo_col, stg + p * PB + s0 * C::ROWB, p * 64, t / a.R, t % a.R, it.bh);
            }
          } else {
            tma_store_3d(&mo_nat, stg + p * PB, p * 64, xw, it.bh);
          }
        }
        bulk_commit_group();
      }
      if (valid) a.lse[static_cast<size_t>(it.bh) * a.N + nat] = lse_out;
      if (it.n > 0) ++ta;
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<C::TMEM_COLS>(tmem);
  }
}

}  // namespace sa
