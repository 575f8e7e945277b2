// Wide-step backward kernel (D = 64) for tables whose key tiles see many
// query steps: the recompute-based gradient of block-sparse attention
// ("Generating Long Sequences with Sparse Transformers", ABSTRACT, item b;
// pcnews translation, "Глубокое внимание"), the same mathematics as
// sa_bwd_kernel:
//   P = exp(S - lse), dV = P^T dO, dP = dO V^T, dS = P (dP - Delta),
//   dK = s dS^T Q, dQ = s dS K.
//
// Persistent: one CTA per SM walks a zig-zag share of the (128-key tile,
// batch*head) items of its table, longest first.  Each item walks its
// 128-query steps.  Per step g:
//   S^T_g  = K Q_g^T   and  dP^T_g = V dO_g^T      (tcgen05, M128 N128)
//   P^T_g, dS^T_g                                  (elementwise warps)
//   dV += P^T_g dO_g,  dK += dS^T_g Q_g             (M128 N64 K128)
//   dQ_g = dS_g K                                  (M128 N64 K128, then a
//                                                   bulk reduce-add into the
//                                                   fp32 accumulator)
// The products of the 128-query step run at the tensor cores' full N = 128
// rate for S^T and dP^T.
//
// Roles (512 threads, four warpgroups, registers rebalanced by setmaxnreg):
//   warpgroup 0 (56 registers): warp 0 lane 0 TMA producer (K/V per item into
//     one of two buffers, Q/dO and the packed -lse*log2e / -Delta blocks per
//     step through a STAGES-deep ring); warp 1 allocates TMEM and lane 0
//     issues every MMA; warps 2-3 idle.
//   warpgroups 1 and 2 (176 registers): elementwise.  Warpgroup 1+h takes the
//     64 query columns [64h, 64h + 64) of every step; thread = key row =
//     TMEM lane (warp w touches lanes 32*(w%4) .. +31).  A thread holds its
//     whole S^T and dP^T half-row in registers.
//   warpgroup 3 (104 registers): dQ read-out and reduce-add per step, and
//     the dV / dK epilogue per item (through the item's K/V buffer, which is
//     idle by then).
// TMEM (512 columns): S^T [0, 128), dP^T [128, 256) (the bf16 P^T of column
// half h is written over dP^T columns 128 + 64h + [32, 64) once that half-row
// is in registers, and dV reads it from there), dV [256, 320), dK [320, 384),
// two dQ buffers [384, 448) and [448, 512).
//
// MMA issue order per step g: S^T_g (once the elementwise warps have read
// S^T_{g-1}), dV_{g-1} (once P^T_{g-1} is written), dP^T_g (once dV_{g-1} has
// completed: P^T_{g-1} lives in its columns), then dK_{g-1} and dQ_{g-1}.
#pragma once

#include "sa_bwd.cuh"

namespace sa {

struct WideCfg {
  static constexpr int D = 64;
  static constexpr int TK = 128, TQ = 128, HQ = 64;
  static constexpr int KVB = 2;     // K/V buffers (the next item's tiles load early)
  static constexpr int STAGES = 3;  // Q/dO ring
  static constexpr int DSTB = 1;    // dS^T buffers
  static constexpr int KV_BYTES = TK * D * 2;    // 16 KiB
  static constexpr int QS_BYTES = TQ * D * 2;    // 16 KiB
  static constexpr int PANEL = TK * HQ * 2;      // [128 keys][64 queries] bf16, 16 KiB
  static constexpr int DST_BYTES = 2 * PANEL;    // one step: two panels
  static constexpr int LD_BYTES = TQ * 8;        // two [2][64] float blocks
  static constexpr int DQS_WARP = 32 * 32 * 4;   // 32 query rows x 32 fp32 (one reduce box)
  static constexpr int EPI_WARP = 32 * D * 4;    // 32 key rows x D fp32, inside the K/V buffer
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KVB * KV_BYTES;
  static constexpr int OFF_Q = OFF_V + KVB * KV_BYTES;
  static constexpr int OFF_DO = OFF_Q + STAGES * QS_BYTES;
  static constexpr int OFF_DST = OFF_DO + STAGES * QS_BYTES;
  static constexpr int OFF_DQS = OFF_DST + DSTB * DST_BYTES;
  static constexpr int OFF_LD = OFF_DQS + 4 * DQS_WARP;
  static constexpr int OFF_BAR = OFF_LD + STAGES * LD_BYTES;
  static constexpr int N_BARS = 2 * KVB + 2 * STAGES + 7 + 2 * DSTB + 4 + 2 + 4;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int COL_ST = 0, COL_DPT = 128, COL_DV = 256, COL_DK = 320, COL_DQ = 384;
  static constexpr int THREADS = 512;
  static constexpr int REG_CTRL = 56, REG_EW = 176, REG_DQ = 104;
  static_assert(REG_CTRL + 2 * REG_EW + REG_DQ == 4 * 128, "register split of the 4 warpgroups");
  static_assert(2 * KV_BYTES >= 4 * EPI_WARP, "epilogue staging fits the K and V tiles of an item");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(KV_BYTES % 1024 == 0 && QS_BYTES % 1024 == 0 && DQS_WARP % 1024 == 0, "1 KiB alignment");
};

template <int N>
__device__ __forceinline__ void regs_raise() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_lower() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Bounded wait used only to drain in-flight asynchronous work after an
// abort: it ignores the abort flag and gives up after about 2^26 cycles.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > (1LL << 26)) return;
  }
}

// S^T = K Q^T or dP^T = V dO^T of one 128-query step (M128 N128, K = D).
__device__ __forceinline__ void wide_issue_s(uint32_t d_tmem, uint32_t a_base, uint32_t b_base) {
  using C = WideCfg;
  constexpr uint32_t id_s = make_idesc_bf16(128, C::TQ, false, false);
#pragma unroll
  for (int kk = 0; kk < C::D / 16; ++kk)
    mma_bf16_ss(d_tmem, bwd_kdesc<C::D>(a_base, C::TK, kk), bwd_kdesc<C::D>(b_base, C::TQ, kk), id_s, kk > 0);
}

// dV += P^T_g dO_g for step g (j: its index in the item; ne: the item's
// index among this CTA's non-empty items).  P^T sits in TMEM over the second
// half of each 64-column half of dP^T.  The first step of an item first waits
// until the epilogue has read the previous item's dV / dK.
__device__ __forceinline__ bool wide_issue_dv(uint32_t tmem, uint32_t do_base, int j, int g, int ne,
                                              uint64_t* bar_pt_full, uint64_t* bar_pt_free,
                                              uint64_t* bar_dkv_free, int* abort_flag) {
  using C = WideCfg;
  constexpr uint32_t id_kv = make_idesc_bf16(128, C::D, false, true);
  if (!mbar_wait(bar_pt_full, g & 1, abort_flag)) return false;
  if (j == 0 && ne >= 1 && !mbar_wait(bar_dkv_free, (ne - 1) & 1, abort_flag)) return false;
  tc_fence_after();
#pragma unroll
  for (int kk = 0; kk < C::TQ / 16; ++kk) {
    const uint32_t pt = tmem + C::COL_DPT + (kk >> 2) * 64 + 32 + (kk & 3) * 8;
    mma_bf16_ts(tmem + C::COL_DV, pt, bwd_mndesc<C::D>(do_base, C::TQ, kk), id_kv, (j > 0 || kk > 0));
  }
  mma_commit(bar_pt_free);
  return true;
}

// dK += dS^T_g Q_g, then dQ_g = dS_g K into dQ buffer qi % 2; releases the
// Q/dO stage, the dS^T buffer and (last step of the item) the dV / dK
// accumulators.
__device__ __forceinline__ bool wide_issue_dk_dq(uint32_t tmem, uint32_t q_base, uint32_t k_base, uint32_t dst0,
                                                 int j, int last, int g, int qi, uint64_t* bar_dst_full,
                                                 uint64_t* bar_dst_free, uint64_t* bar_stage_empty,
                                                 uint64_t* bar_dq_full, uint64_t* bar_dq_free,
                                                 uint64_t* bar_dkv_full, int* abort_flag) {
  using C = WideCfg;
  constexpr uint32_t id_kv = make_idesc_bf16(128, C::D, false, true);
  constexpr uint32_t id_q = make_idesc_bf16(128, C::D, true, true);
  const int db = g % C::DSTB;
  if (!mbar_wait(bar_dst_full + db, (g / C::DSTB) & 1, abort_flag)) return false;
  tc_fence_after();
  const uint32_t dst = dst0 + db * C::DST_BYTES;
#pragma unroll
  for (int kk = 0; kk < C::TQ / 16; ++kk)
    mma_bf16_ss(tmem + C::COL_DK, pt_kdesc(dst + (kk >> 2) * C::PANEL, kk & 3), bwd_mndesc<C::D>(q_base, C::TQ, kk),
                id_kv, (j > 0 || kk > 0));
  mma_commit(bar_stage_empty);
  const int qb = qi & 1;
  if (qi >= 2 && !mbar_wait(bar_dq_free + qb, ((qi >> 1) - 1) & 1, abort_flag)) return false;
  tc_fence_after();
#pragma unroll
  for (int kk = 0; kk < C::TK / 16; ++kk)
    mma_bf16_ss(tmem + C::COL_DQ + qb * C::D, pair_mndesc(dst, kk), bwd_mndesc<C::D>(k_base, C::TK, kk), id_q,
                kk > 0);
  mma_commit(bar_dq_full + qb);
  mma_commit(bar_dst_free + db);
  if (last) mma_commit(bar_dkv_full);  // every product of the item has been issued
  return true;
}

template <bool FINAL_T>
__global__ void __launch_bounds__(512, 1)
    sa_bwd_wide_kernel(const __grid_constant__ CUtensorMap mq_nat, const __grid_constant__ CUtensorMap mq_col,
                       const __grid_constant__ CUtensorMap mdo_nat, const __grid_constant__ CUtensorMap mdo_col,
                       const __grid_constant__ CUtensorMap mk_nat, const __grid_constant__ CUtensorMap mk_col,
                       const __grid_constant__ CUtensorMap mk_sum, const __grid_constant__ CUtensorMap mv_nat,
                       const __grid_constant__ CUtensorMap mv_col, const __grid_constant__ CUtensorMap mv_sum,
                       const __grid_constant__ CUtensorMap mdq_nat, const __grid_constant__ CUtensorMap mdq_col,
                       const __grid_constant__ CUtensorMap mdk_out, const __grid_constant__ CUtensorMap mdv_out,
                       const __grid_constant__ CUtensorMap mdk_part, const __grid_constant__ CUtensorMap mdv_part,
                       const BwdArgs a) {
  using C = WideCfg;
  constexpr int D = C::D;
#ifdef SA_TEST_HOOKS
  pdl_wait();  // the range check of the tables (previous kernel) has completed
  if (*(volatile int*)&g_status == kStatusLut) return;  // a table failed it: touch nothing
#endif
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sDO = smem + C::OFF_DO;
  uint8_t* sDST = smem + C::OFF_DST;
  float* sLD = reinterpret_cast<float*>(smem + C::OFF_LD);  // [STAGES][2 halves][2][64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_kv_full = bars;                        // [KVB]
  uint64_t* bar_kv_empty = bar_kv_full + C::KVB;       // [KVB] the item's epilogue is done with it
  uint64_t* bar_qdo_full = bar_kv_empty + C::KVB;      // [STAGES]
  uint64_t* bar_qdo_empty = bar_qdo_full + C::STAGES;  // [STAGES]
  uint64_t* bar_st_full = bar_qdo_empty + C::STAGES;   // S^T_g in TMEM
  uint64_t* bar_st_free = bar_st_full + 1;             // S^T_g read by the elementwise warps
  uint64_t* bar_dpt_full = bar_st_free + 1;            // dP^T_g in TMEM
  uint64_t* bar_pt_full = bar_dpt_full + 1;            // P^T_g written into TMEM
  uint64_t* bar_pt_free = bar_pt_full + 1;             // dV_g completed (dP^T columns free)
  uint64_t* bar_dkv_full = bar_pt_free + 1;            // the item's dV / dK complete
  uint64_t* bar_dkv_free = bar_dkv_full + 1;           // ... and read out
  uint64_t* bar_dst_full = bar_dkv_free + 1;           // [DSTB]
  uint64_t* bar_dst_free = bar_dst_full + C::DSTB;     // [DSTB]
  uint64_t* bar_dq_full = bar_dst_free + C::DSTB;      // [2]
  uint64_t* bar_dq_free = bar_dq_full + 2;             // [2]
  uint64_t* bar_drain = bar_dq_free + 2;               // the issuer's last commit
  uint64_t* bar_spare = bar_drain + 1;
  uint64_t* bar_epi = bar_spare + 1;                   // [4] partial rows landed (epilogue warp)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int wg = warp >> 2;
  const int q_src = (a.key_view == SRC_T) ? SRC_T : SRC_N;
  const int n_items = a.n_slots * a.BH;
  const int cta = blockIdx.x, n_ctas = gridDim.x;

  if (threadIdx.x == 0) {
    for (int b = 0; b < C::KVB; ++b) {
      mbar_init(bar_kv_full + b, 1);
      mbar_init(bar_kv_empty + b, 4);
    }
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_qdo_full + s, 1);
      mbar_init(bar_qdo_empty + s, 1);
    }
    mbar_init(bar_st_full, 1);
    mbar_init(bar_st_free, 256);
    mbar_init(bar_dpt_full, 1);
    mbar_init(bar_pt_full, 256);
    mbar_init(bar_pt_free, 1);
    mbar_init(bar_dkv_full, 1);
    mbar_init(bar_dkv_free, 128);
    for (int b = 0; b < C::DSTB; ++b) {
      mbar_init(bar_dst_full + b, 256);
      mbar_init(bar_dst_free + b, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_dq_full + b, 1);
      mbar_init(bar_dq_free + b, 128);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_spare, 1);
    for (int w = 0; w < 4; ++w) mbar_init(bar_epi + w, 1);
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

  if (wg == 0) {
    regs_lower<C::REG_CTRL>();
    if (warp == 0 && lane == 0) {
      // -------------------------------------------------------------- producer
      bool ok = true;
      int gs = 0, ne = 0;  // Q/dO loads and K/V loads issued
      BwdItem nxt = (cta < n_items) ? bwd_item(a, cta) : BwdItem{0, 0, 0, 0};
      for (int k = 0, item = cta; ok && item < n_items;) {
        const BwdItem it = nxt;
        item = zigzag_item(++k, cta, n_ctas);
        if (item < n_items) nxt = bwd_item(a, item);
        if (it.n == 0) continue;
        const int kb = ne % C::KVB;
        if (ne >= C::KVB && !mbar_wait(bar_kv_empty + kb, ((ne / C::KVB) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar_kv_full + kb, 2 * C::KV_BYTES);
        load_rows<D>(sK + kb * C::KV_BYTES, a.key_view, it.kt * C::TK, C::TK, it.bh, &mk_nat, &mk_col, &mk_sum,
                     bar_kv_full + kb, a.R, a.l, a.c);
        load_rows<D>(sV + kb * C::KV_BYTES, a.key_view, it.kt * C::TK, C::TK, it.bh, &mv_nat, &mv_col, &mv_sum,
                     bar_kv_full + kb, a.R, a.l, a.c);
        ++ne;
        const float* ld = (q_src == SRC_T ? a.ld_col : a.ld_nat) + static_cast<size_t>(it.bh) * a.n_pad * 2;
        int e_next = a.ent[it.e0];
        for (int j = 0; j < it.n; ++j) {
          const int st = gs % C::STAGES;
          const int e = e_next;
          if (j + 1 < it.n) e_next = a.ent[it.e0 + j + 1];
          if (gs >= C::STAGES && !mbar_wait(bar_qdo_empty + st, ((gs / C::STAGES) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
#ifdef SA_TEST_HOOKS
          if (gs == 0 && *(volatile int*)&g_test_withhold) {  // the first step's tiles never arrive
            ++gs;
            continue;
          }
#endif
          const int qpos = (e >> 3) * C::TQ;
          mbar_arrive_expect_tx(bar_qdo_full + st, 2 * C::QS_BYTES + C::LD_BYTES);
          load_rows<D>(sQ + st * C::QS_BYTES, q_src, qpos, C::TQ, it.bh, &mq_nat, &mq_col, &mq_col,
                       bar_qdo_full + st, a.R, a.l, a.c);
          load_rows<D>(sDO + st * C::QS_BYTES, q_src, qpos, C::TQ, it.bh, &mdo_nat, &mdo_col, &mdo_col,
                       bar_qdo_full + st, a.R, a.l, a.c);
          bulk_load(sLD + st * 2 * C::TQ, ld + 2 * qpos, C::LD_BYTES, bar_qdo_full + st);
          ++gs;
        }
      }
      // After an abort, wait (bounded) for the loads still in flight, so that
      // no copy lands in shared memory after the CTA has exited.
      if (*(volatile int*)abort_flag) {
        for (int h = ne > C::KVB ? ne - C::KVB : 0; h < ne; ++h)
          mbar_wait_drain(bar_kv_full + h % C::KVB, (h / C::KVB) & 1);
        for (int h = gs > C::STAGES ? gs - C::STAGES : 0; h < gs; ++h)
          mbar_wait_drain(bar_qdo_full + h % C::STAGES, (h / C::STAGES) & 1);
      }
    } else if (warp == 1 && lane == 0) {
      // -------------------------------------------------------------- MMA issuer
      bool ok = true;
      int g = 0, ne = 0, qi = 0;
      // the previous step, whose dV / dK / dQ products are issued after this
      // step's S^T (dV) and dP^T (dK, dQ)
      bool have_prev = false;
      int p_st = 0, p_j = 0, p_last = 0, p_kb = 0, p_ne = 0;
      BwdItem nxt = (cta < n_items) ? bwd_item(a, cta) : BwdItem{0, 0, 0, 0};
      for (int k = 0, item = cta; ok && item < n_items;) {
        const BwdItem it = nxt;
        item = zigzag_item(++k, cta, n_ctas);
        if (item < n_items) nxt = bwd_item(a, item);
        if (it.n == 0) continue;
        const int kb = ne % C::KVB;
        ok = mbar_wait(bar_kv_full + kb, (ne / C::KVB) & 1, abort_flag);
        const uint32_t k_base = smem_u32(sK + kb * C::KV_BYTES), v_base = smem_u32(sV + kb * C::KV_BYTES);
        for (int j = 0; ok && j < it.n; ++j) {
          const int st = g % C::STAGES;
          ok = mbar_wait(bar_qdo_full + st, (g / C::STAGES) & 1, abort_flag);
          if (ok && g > 0) ok = mbar_wait(bar_st_free, (g - 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t q_base = smem_u32(sQ + st * C::QS_BYTES);
          const uint32_t do_base = smem_u32(sDO + st * C::QS_BYTES);
          wide_issue_s(tmem + C::COL_ST, k_base, q_base);  // S^T_g = K Q_g^T
          mma_commit(bar_st_full);
          if (have_prev) {
            ok = wide_issue_dv(tmem, smem_u32(sDO + p_st * C::QS_BYTES), p_j, g - 1, p_ne, bar_pt_full, bar_pt_free,
                               bar_dkv_free, abort_flag) &&
                 mbar_wait(bar_pt_free, (g - 1) & 1, abort_flag);  // dV_{g-1} done: its P^T columns are free
            if (!ok) break;
            tc_fence_after();
          }
          wide_issue_s(tmem + C::COL_DPT, v_base, do_base);  // dP^T_g = V dO_g^T
          mma_commit(bar_dpt_full);
          if (have_prev) {
            ok = wide_issue_dk_dq(tmem, smem_u32(sQ + p_st * C::QS_BYTES), smem_u32(sK + p_kb * C::KV_BYTES),
                                  smem_u32(sDST), p_j, p_last, g - 1, qi, bar_dst_full, bar_dst_free,
                                  bar_qdo_empty + p_st, bar_dq_full, bar_dq_free, bar_dkv_full, abort_flag);
            ++qi;
            if (!ok) break;
          }
          have_prev = true;
          p_st = st;
          p_j = j;
          p_last = (j == it.n - 1);
          p_kb = kb;
          p_ne = ne;
          ++g;
        }
        ++ne;
      }
      if (ok && have_prev) {  // the last step's dV, dK, dQ
        ok = wide_issue_dv(tmem, smem_u32(sDO + p_st * C::QS_BYTES), p_j, g - 1, p_ne, bar_pt_full, bar_pt_free,
                           bar_dkv_free, abort_flag) &&
             wide_issue_dk_dq(tmem, smem_u32(sQ + p_st * C::QS_BYTES), smem_u32(sK + p_kb * C::KV_BYTES),
                              smem_u32(sDST), p_j, p_last, g - 1, qi, bar_dst_full, bar_dst_free,
                              bar_qdo_empty + p_st, bar_dq_full, bar_dq_free, bar_dkv_full, abort_flag);
        ++qi;
      }
      // every MMA issued by this thread has completed before TMEM is released
      mma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0);
    }
  } else if (wg <= 2) {
    regs_raise<C::REG_EW>();
    // -------------------------------------------------------------- elementwise
    const int half = wg - 1;  // query columns [64 half, 64 half + 64) of each step
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t col_s = tmem + lane_base + C::COL_ST + half * C::HQ;
    const uint32_t col_dp = tmem + lane_base + C::COL_DPT + half * C::HQ;
    bool ok = true;
    int gs = 0;
    const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2);
    BwdItem nxt = (cta < n_items) ? bwd_item(a, cta) : BwdItem{0, 0, 0, 0};
    for (int k = 0, item = cta; ok && item < n_items;) {
      const BwdItem it = nxt;
      item = zigzag_item(++k, cta, n_ctas);
      if (item < n_items) nxt = bwd_item(a, item);
      if (it.n == 0) continue;
      const KeyRow kr = key_row<D, FINAL_T>(a, it.kt, row);
      int e_next = a.ent[it.e0];
      for (int j = 0; j < it.n; ++j) {
        const int g = gs + j;
        const int st = g % C::STAGES;
        const int e = e_next;
        if (j + 1 < it.n) e_next = a.ent[it.e0 + j + 1];
        const int x0 = (e >> 3) * C::TQ + half * C::HQ;  // view position of this half's first query
        ok = ok && mbar_wait(bar_qdo_full + st, (g / C::STAGES) & 1, abort_flag);
        ok = ok && mbar_wait(bar_st_full, g & 1, abort_flag);
        tc_fence_after();
        // (1) the S^T half-row: one TMEM round trip, then 64 independent exp2
        float sv[64];
#pragma unroll
        for (int c16 = 0; c16 < 4; ++c16) tmem_ld16(col_s + c16 * 16, sv + c16 * 16);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar_st_free);
        const float4* nlse4 = reinterpret_cast<const float4*>(sLD + st * 2 * C::TQ + half * 128);
        const float4* ndel4 = nlse4 + 16;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float4 t = nlse4[i];
          const float2 x01 = f2_unpack(f2_fma(f2_pack(sv[4 * i], sv[4 * i + 1]), sc2, f2_pack(t.x, t.y)));
          const float2 x23 = f2_unpack(f2_fma(f2_pack(sv[4 * i + 2], sv[4 * i + 3]), sc2, f2_pack(t.z, t.w)));
          sv[4 * i] = ex2(x01.x);
          sv[4 * i + 1] = ex2(x01.y);
          sv[4 * i + 2] = ex2(x23.x);
          sv[4 * i + 3] = ex2(x23.y);
        }
        if (e & 1) mask_interval64(sv, kr.qlo - x0, kr.qhi - x0, 0.f);
        // (2) the dP^T half-row in one round trip; P^T (bf16) over its second
        //     half, where the dV product reads it
        ok = ok && mbar_wait(bar_dpt_full, g & 1, abort_flag);
        tc_fence_after();
        float dp[64];
#pragma unroll
        for (int c16 = 0; c16 < 4; ++c16) tmem_ld16(col_dp + c16 * 16, dp + c16 * 16);
        tmem_wait_ld();
#pragma unroll
        for (int h16 = 0; h16 < 2; ++h16) {
          float pk[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) pk[u] = __uint_as_float(pack_bf16(sv[32 * h16 + 2 * u], sv[32 * h16 + 2 * u + 1]));
          tmem_st16(col_dp + 32 + 16 * h16, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_pt_full);
        // (3) dS = P (dP - Delta), packed to bf16 in registers first (no shared
        //     memory store between the Delta loads, so they need not wait for
        //     one another), then stored into this half's dS^T panel once the
        //     buffer is free
        uint32_t dsk[32];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const float4 d0 = ndel4[2 * ch], d1 = ndel4[2 * ch + 1];
          const int c0 = ch * 8;
          const float2 a01 = f2_unpack(
              f2_mul(f2_pack(sv[c0], sv[c0 + 1]), f2_add(f2_pack(dp[c0], dp[c0 + 1]), f2_pack(d0.x, d0.y))));
          const float2 a23 = f2_unpack(
              f2_mul(f2_pack(sv[c0 + 2], sv[c0 + 3]), f2_add(f2_pack(dp[c0 + 2], dp[c0 + 3]), f2_pack(d0.z, d0.w))));
          const float2 a45 = f2_unpack(
              f2_mul(f2_pack(sv[c0 + 4], sv[c0 + 5]), f2_add(f2_pack(dp[c0 + 4], dp[c0 + 5]), f2_pack(d1.x, d1.y))));
          const float2 a67 = f2_unpack(
              f2_mul(f2_pack(sv[c0 + 6], sv[c0 + 7]), f2_add(f2_pack(dp[c0 + 6], dp[c0 + 7]), f2_pack(d1.z, d1.w))));
          dsk[4 * ch] = pack_bf16(a01.x, a01.y);
          dsk[4 * ch + 1] = pack_bf16(a23.x, a23.y);
          dsk[4 * ch + 2] = pack_bf16(a45.x, a45.y);
          dsk[4 * ch + 3] = pack_bf16(a67.x, a67.y);
        }
        const int db = g % C::DSTB;
        if (g >= C::DSTB) ok = ok && mbar_wait(bar_dst_free + db, ((g / C::DSTB) - 1) & 1, abort_flag);
        uint8_t* dst = sDST + db * C::DST_BYTES + half * C::PANEL;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          *reinterpret_cast<uint4*>(dst + sw128_offset(row, ch)) =
              make_uint4(dsk[4 * ch], dsk[4 * ch + 1], dsk[4 * ch + 2], dsk[4 * ch + 3]);
        fence_proxy_async_smem();
        mbar_arrive(bar_dst_full + db);
      }
      gs += it.n;
    }
  } else {
    regs_lower<C::REG_DQ>();
    // -------------------------------------------------------------- dQ reduction + dV/dK epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // query row of a dQ product; key row of the epilogue
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    uint8_t* stq = smem + C::OFF_DQS + quarter * C::DQS_WARP;
    bool ok = true;
    int gs = 0, ne = 0, qi = 0, epi_n = 0;
    BwdItem nxt = (cta < n_items) ? bwd_item(a, cta) : BwdItem{0, 0, 0, 0};
    for (int k = 0, item = cta; ok && item < n_items;) {
      const BwdItem it = nxt;
      item = zigzag_item(++k, cta, n_ctas);
      if (item < n_items) nxt = bwd_item(a, item);
      for (int j = 0; j < it.n; ++j) {
        const int qb = qi & 1;
        ok = ok && mbar_wait(bar_dq_full + qb, (qi >> 1) & 1, abort_flag);
        tc_fence_after();
        const int xw = (a.ent[it.e0 + j] >> 3) * C::TQ + quarter * 32;  // view position of the warp's first row
#pragma unroll
        for (int bx = 0; bx < D / 32; ++bx) {
          float gq[32];
          tmem_ld16(tmem + lane_base + C::COL_DQ + qb * D + bx * 32, gq);
          tmem_ld16(tmem + lane_base + C::COL_DQ + qb * D + bx * 32 + 16, gq + 16);
          tmem_wait_ld();
          if (bx == D / 32 - 1) {
            tc_fence_before();
            mbar_arrive(bar_dq_free + qb);  // the rows are in registers
          }
          if (lane == 0) bulk_wait_read_all();  // the previous reduce has read the staging box
          __syncwarp();
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<float4*>(stq + sw128_offset(lane, ch)) =
                make_float4(gq[ch * 4] * a.scale, gq[ch * 4 + 1] * a.scale, gq[ch * 4 + 2] * a.scale,
                            gq[ch * 4 + 3] * a.scale);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (q_src == SRC_T) {
              const int rb = gcd_int(a.R, 32);
              for (int s0 = 0; s0 < 32; s0 += rb) {
                const int t = xw + s0;
                tma_reduce_add_4d(&mdq_col, stq + s0 * 128, bx * 32, t / a.R, t % a.R, it.bh);
              }
            } else {
              tma_reduce_add_3d(&mdq_nat, stq, bx * 32, xw, it.bh);
            }
            bulk_commit_group();
          }
        }
        ++qi;
      }
      // ---- dV / dK of this item (thread = key row)
      const KeyRow kr = key_row<D, FINAL_T>(a, it.kt, row);
      const bool nat_out = a.key_view == SRC_N || FINAL_T;  // bf16 rows (else fp32 partials)
      if (it.n > 0) {
        const int kb = ne % C::KVB;
        ok = ok && mbar_wait(bar_dkv_full, ne & 1, abort_flag);
        tc_fence_after();
        // staging: this warp's 8 KiB of the item's K/V buffer (no MMA reads it any more)
        uint8_t* stg = (quarter < 2 ? sK + kb * C::KV_BYTES : sV + kb * C::KV_BYTES) + (quarter & 1) * C::EPI_WARP;
        const int y0 = it.kt * C::TK + quarter * 32;  // first view key of the warp
        bool row_add = false;
        if (nat_out && a.add_part == 1) row_add = kr.kvalid && kr.knat < a.R * a.l;  // keys of whole rows
        else if (nat_out && a.add_part == 2) row_add = kr.kvalid && (kr.knat % a.l) >= (a.l - a.c) && kr.knat < a.R * a.l;
        const bool warp_add = __any_sync(0xffffffffu, row_add);
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {  // 0: dV, 1: dK
          if (lane == 0) bulk_wait_read_all();  // earlier stores have read the staging
          __syncwarp();
          if (warp_add && lane == 0) {
            mbar_arrive_expect_tx(bar_epi + quarter, 32 * D * 4);
#pragma unroll
            for (int bx = 0; bx < D / 32; ++bx)
              tma_load_3d(stg + bx * 4096, which ? &mdk_part : &mdv_part, bar_epi + quarter, bx * 32, y0, it.bh);
          }
          const uint32_t col = which ? C::COL_DK : C::COL_DV;
          const float mul = which ? a.scale : 1.f;
#pragma unroll
          for (int h = 0; h < D / 32; ++h) {
            float gv[32];
            tmem_ld16(tmem + lane_base + col + h * 32, gv);
            tmem_ld16(tmem + lane_base + col + h * 32 + 16, gv + 16);
            tmem_wait_ld();
            if (which == 1 && h == D / 32 - 1) {
              tc_fence_before();
              mbar_arrive(bar_dkv_free);  // both accumulators have been read
            }
#pragma unroll
            for (int u = 0; u < 32; ++u) gv[u] *= mul;
            if (h == 0 && warp_add) {
              ok = ok && mbar_wait(bar_epi + quarter, epi_n & 1, abort_flag);
              ++epi_n;
            }
            if (row_add) {
#pragma unroll
              for (int ch = 0; ch < 8; ++ch) {
                const float4 t = *reinterpret_cast<const float4*>(stg + h * 4096 + sw128_offset(lane, ch));
                gv[ch * 4] += t.x;
                gv[ch * 4 + 1] += t.y;
                gv[ch * 4 + 2] += t.z;
                gv[ch * 4 + 3] += t.w;
              }
            }
            if (nat_out) {
              // the bf16 row (128 bytes) lands over the first fp32 box, which
              // every lane of the warp has read by then
              if (h == 0 && warp_add) __syncwarp();
#pragma unroll
              for (int c4 = 0; c4 < 4; ++c4) {
                const int ch = h * 4 + c4;
                const uint4 w = make_uint4(pack_bf16(gv[8 * c4], gv[8 * c4 + 1]), pack_bf16(gv[8 * c4 + 2], gv[8 * c4 + 3]),
                                           pack_bf16(gv[8 * c4 + 4], gv[8 * c4 + 5]),
                                           pack_bf16(gv[8 * c4 + 6], gv[8 * c4 + 7]));
                *reinterpret_cast<uint4*>(stg + sw128_offset(lane, ch)) = w;
              }
            } else {
#pragma unroll
              for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<float4*>(stg + h * 4096 + sw128_offset(lane, ch)) =
                    make_float4(gv[ch * 4], gv[ch * 4 + 1], gv[ch * 4 + 2], gv[ch * 4 + 3]);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if constexpr (FINAL_T) {  // rows of the column runs
              const int rb = gcd_int(a.R, 32);
              for (int s0 = 0; s0 < 32; s0 += rb) {
                const int t = y0 + s0;
                tma_store_4d(which ? &mdk_out : &mdv_out, stg + s0 * (D * 2), 0, t / a.R, t % a.R, it.bh);
              }
            } else if (nat_out) {
              tma_store_3d(which ? &mdk_out : &mdv_out, stg, 0, y0, it.bh);
            } else {
              const CUtensorMap* mp = which ? &mdk_part : &mdv_part;
#pragma unroll
              for (int bx = 0; bx < D / 32; ++bx) {
                if (a.key_view == SRC_T) {
                  const int rb = gcd_int(a.R, 32);
                  for (int s0 = 0; s0 < 32; s0 += rb) {
                    const int t = y0 + s0;
                    tma_store_4d(mp, stg + bx * 4096 + s0 * 128, bx * 32, t / a.R, t % a.R, it.bh);
                  }
                } else {
                  int cb, gb;
                  summary_box(a.c, 32, &cb, &gb);
                  if (gb > 1 || cb == a.c) {  // whole blocks
                    tma_store_4d(mp, stg + bx * 4096, bx * 32, a.l - a.c, y0 / a.c, it.bh);
                  } else {  // runs of cb keys inside one block
                    for (int s0 = 0; s0 < 32; s0 += cb) {
                      const int y = y0 + s0;
                      tma_store_4d(mp, stg + bx * 4096 + s0 * 128, bx * 32, a.l - a.c + y % a.c, y / a.c, it.bh);
                    }
                  }
                }
              }
            }
            bulk_commit_group();
          }
        }
        if (lane == 0) {
          bulk_wait_read_all();  // the K/V buffer may be reloaded once the stores have read it
          mbar_arrive(bar_kv_empty + kb);
        }
        ++ne;
      } else {
        // a key tile that no query sees: zero gradients (plus, in the natural
        // pass, the secondary view's partials), written directly
        const size_t off = (static_cast<size_t>(it.bh) * a.N + (kr.kvalid ? kr.knat : 0)) * D;
        bool add = false;
        if (a.add_part == 1) add = kr.knat < a.R * a.l;
        else if (a.add_part == 2) add = (kr.knat % a.l) >= (a.l - a.c) && kr.knat < a.R * a.l;
        if (kr.kvalid) {
#pragma unroll 1
          for (int which = 0; which < 2; ++which) {
#pragma unroll
            for (int i = 0; i < D / 16; ++i) {
              float gv[16];
#pragma unroll
              for (int u = 0; u < 16; ++u) gv[u] = 0.f;
              store_grad_row<D, 16>(a, which, off, i * 16, gv, !nat_out, add && nat_out);
            }
          }
        }
      }
      gs += it.n;
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
