// Backward kernels: recompute-based gradient of block-sparse attention.
//
// The backward pass rebuilds P from the saved log-sum-exp instead of keeping
// the attention matrix, the recomputation of "Generating Long Sequences with
// Sparse Transformers" (ABSTRACT, item b) and of the pcnews translation
// ("Глубокое внимание").  With Delta_i = sum_d dO_id O_id:
//   P = exp(S - lse), dV = P^T dO, dP = dO V^T, dS = P (dP - Delta),
//   dK = s dS^T Q, dQ = s dS K.
//
// sa_bwd_kernel is persistent: one CTA per SM walks a fixed zig-zag share of
// the (key tile, batch*head) items of its table (longest tiles first), each
// item a 128-key tile in the view order of the table and the 64-query steps
// that see it.  Per step (global step counter g, continued across items):
//   ST_g  = K Q^T, dPT_g = V dO^T  (keys on TMEM lanes, 64 columns each,
//                                   double-buffered)
//   P^T_g, dS^T_g in bf16          (elementwise warps; dS^T in smem, P^T in
//                                   smem or, in the LONG shape, in TMEM)
//   dV += P^T dO, dK += dS^T Q     (TMEM accumulators of the item)
//   dQ = dS K for the 128 queries of the global step pair (g even, g odd),
//   restricted to the item's own steps, then reduced into an fp32 workspace
//   (where each query step meets one key tile of the pass: stored into it by
//   the first pass, or added to the earlier passes' sum and stored as the
//   final bf16 rows by the natural pass).
// In the SHORT shape K/V and dV/dK are double-buffered so the next item's
// tiles load and accumulate during this one; the dV/dK epilogue of an item
// runs in the dQ warps while the next item's steps proceed.  A secondary
// (column or summary) view's pass writes its dK/dV as fp32 partials at the
// keys' natural positions; the natural pass then adds them to its own rows
// and writes bf16 (or, SUM_RED, reduce-adds its rows into the partials and a
// small launch rounds them).
// Roles (480 threads): warp 0 producer (TMA for K, V, Q, dO; bulk copy of
// the packed lse/Delta), warp 1 TMEM allocation and lane 0 issue of ST/dPT,
// warps 2..9 elementwise (two groups of four taking alternate global steps,
// one warp per TMEM lane quarter each), warps 10..13 dQ reduction and the
// dV/dK epilogue, warp 14 lane 0 issue of dV/dK/dQ.  Warp w may only touch
// TMEM lanes 32*(w%4)..32*(w%4)+31, so every role picks its rows by w%4.
// TMEM columns: ST[b] = b*64, dPT[b] = NBUF*64 + b*64 (one buffer each that
// the two elementwise groups take in turn, or one per group in the LONG
// shape), dV[b] = 2*NBUF*64 + b*2D, dK[b] = dV[b] + D with b the item parity
// (two buffers for D <= 64 outside the LONG shape, so an item's dV/dK
// accumulate while the previous item's are read out), then the dQ buffers:
//   dQ[b] = dK + D + b*D (two dQ buffers for D <= 64, one for D = 128).
#pragma once

#include "sa_device.cuh"
#include "sa_fwd.cuh"

namespace sa {

struct BwdArgs {
  const int32_t* sched;  // per launch slot: {tile, first entry, count, 0}
  const int32_t* ent;
  // Per 64-query step of view positions: 64 floats -lse*log2(e), then 64
  // floats -Delta ([BH][n_pad/64][2][64]), natural query order / column-major
  // order (strided).  Padding positions hold (-inf, 0).
  const float* ld_nat;
  const float* ld_col;
  int n_pad;             // N rounded up to the 64-query step, padded with (+inf, 0)
  int n_slots, BH;       // items = n_slots * BH, slot-major (all heads of a slot together)
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
  BoxSet box;        // column / summary TMA boxes per tile height
  const uint32_t* bits;  // sub-block bits per entry (caller block masks with blocks below a tile)
  int blk;               // their block size (16, 32 or 64), else 0
  // kDqFinal passes (below): the final bf16 dQ rows, and whether earlier
  // passes left an fp32 sum in the accumulator to add.
  __nv_bfloat16* dq_out;
  int dq_in;
};

// How a pass hands over its dQ rows (a template argument, so that each form
// is its own instantiation):
//   kDqReduce: reduced into the fp32 accumulator;
//   kDqStore:  stored into it (the first pass, which meets every row once);
//   kDqFinal:  added to the earlier passes' sum and stored as final bf16 rows
//              (the natural pass, which meets every row once and is the last).
enum DqMode : int { kDqReduce = 0, kDqStore = 1, kDqFinal = 2 };

// Two shapes of the same kernel.  LONG is for tables whose items run many
// steps (D <= 64): P^T is written into TMEM over the second half of its
// step's dP^T columns (once the elementwise thread holds that row in
// registers) and dV is a TS-MMA with A read from TMEM; the dP^T buffer then
// stays busy until dV completes, which is off the S^T -> exp -> dV loop
// (S^T is released as soon as it is read).  S^T/dP^T are double-buffered, and
// there is one dV/dK and one K/V buffer (an item boundary costs a short
// stall), so the shared memory of the P^T buffers and of the second K/V
// buffer goes to a deeper Q/dO ring.  The other shape keeps P^T in shared
// memory and double-buffers the per-item state, for items of a few steps.
template <int D, bool LONG = false>
struct BwdCfg {
  static constexpr int TK = 128, TQ = 64;
  static constexpr bool PT_TMEM = LONG;
  static constexpr int NBUF = LONG ? 2 : 1;            // ST/dPT buffers in TMEM
  static constexpr int DKVB = (LONG || D >= 128) ? 1 : 2;  // dV/dK buffers (by item parity)
  // Q/dO ring (>= 2: see the S issuer).  A stage is held from its load
  // until dK of its step is done, which trails the S products by about two
  // steps, so the ring must be deep for the loads to run ahead.
  static constexpr int STAGES = LONG ? ((D == 32) ? 8 : 5) : ((D == 32) ? 3 : 2);
  static constexpr int KVB = (LONG || D >= 128) ? 1 : 2;  // K/V buffers (next item's tiles load early)
  // dQ is added to the fp32 workspace by TMA bulk reduce from a per-warp
  // staging buffer (32 query rows x D fp32, 128B-swizzled 32-column boxes);
  // D = 128 has no shared memory left for it and uses vector reductions.
  static constexpr bool DQ_TMA = (D <= 64);
  static constexpr int DQS_WARP_BYTES = DQ_TMA ? 32 * D * 4 : 0;
  static constexpr int DST_BUFS = (D >= 128) ? 1 : 2;  // dS^T pair buffers
  static constexpr int DQBUF = (D >= 128) ? 1 : 2;     // dQ TMEM buffers
  static constexpr int ROWB = (D >= 64) ? 128 : 64;
  static constexpr uint64_t SWZ = (D >= 64) ? kSwizzle128 : kSwizzle64;
  static constexpr int SBO = 8 * ROWB;
  static constexpr int KV_BYTES = TK * D * 2;          // 128-key tile
  static constexpr int QS_BYTES = TQ * D * 2;          // 64-query tile
  static constexpr int PT_BYTES = TK * TQ * 2;         // [128 keys][64 queries] bf16 = 16 KiB
  static constexpr int DST_BYTES = 2 * PT_BYTES;       // a pair of steps (2 panels)
  static constexpr int LD_BYTES = TQ * 8;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KVB * KV_BYTES;
  static constexpr int OFF_Q = OFF_V + KVB * KV_BYTES;
  static constexpr int OFF_DO = OFF_Q + STAGES * QS_BYTES;
  static constexpr int OFF_PT = OFF_DO + STAGES * QS_BYTES;
  static constexpr int OFF_DST = OFF_PT + (PT_TMEM ? 0 : 2 * PT_BYTES);
  static constexpr int OFF_LD = OFF_DST + DST_BUFS * DST_BYTES;  // float [STAGES][2][64]
  // 4 x DQS_WARP_BYTES; 1 KiB aligned (the 128-byte swizzle pattern is address based)
  static constexpr int OFF_DQS = (OFF_LD + STAGES * LD_BYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_BAR = OFF_DQS + 4 * DQS_WARP_BYTES;
  static constexpr int N_BARS = 2 * KVB + 2 * STAGES + 2 * 7 + DST_BUFS + 2 * DQBUF + 2 * DKVB + 4 + 2;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int COL_DPT = NBUF * 64;
  static constexpr int COL_DV = 2 * NBUF * 64;        // + b * 2D
  static constexpr int COL_DK = COL_DV + D;           // + b * 2D
  static constexpr int COL_DQ = COL_DV + DKVB * 2 * D;
  static constexpr int THREADS = 480;
  static_assert(COL_DQ + DQBUF * D <= TMEM_COLS, "TMEM budget");
  static_assert(STAGES >= 2, "the S issuer needs step j's Q/dO while step j-1's is still in use");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(!LONG || D <= 64, "TMEM budget of the LONG shape");
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

// Item k of this CTA in the zig-zag share: rounds alternate direction so
// that long and short tiles pair up (the slots are sorted longest first).
__device__ __forceinline__ int zigzag_item(int k, int cta, int n_ctas) {
  return k * n_ctas + ((k & 1) ? (n_ctas - 1 - cta) : cta);
}

struct BwdItem {
  int bh, kt, e0, n;
};

__device__ __forceinline__ BwdItem bwd_item(const BwdArgs& a, int item) {
  const int slot = item / a.BH;
  const int4 sc = *reinterpret_cast<const int4*>(a.sched + 4 * slot);
  return BwdItem{item - slot * a.BH, sc.x, sc.y, sc.z};
}

// Key-row facts of an elementwise / epilogue thread for key tile kt.
struct KeyRow {
  int y, knat, qlo, qhi;
  bool kvalid;
};

// T_DIAG: the column view holds the diagonal (SA_COLUMN, whose column view
// stands alone); otherwise it is strict (SA_STRIDED).
template <int D, bool T_DIAG>
__device__ __forceinline__ KeyRow key_row(const BwdArgs& a, int kt, int row) {
  KeyRow k;
  k.y = kt * BwdCfg<D>::TK + row;
  const int nkeys = (a.key_view == SRC_S) ? a.R * a.c : (a.key_view == SRC_T ? a.R * a.l : a.N);
  k.kvalid = k.y < nkeys;
  if (a.key_view == SRC_T) k.knat = (k.y % a.R) * a.l + k.y / a.R;
  else if (a.key_view == SRC_S) k.knat = (k.y / a.c) * a.l + (a.l - a.c) + k.y % a.c;
  else k.knat = k.y;
  if (a.key_view == SRC_T) {
    k.qlo = T_DIAG ? k.y : k.y + 1;
    k.qhi = (k.y / a.R) * a.R + a.R - 1;
  } else if (a.key_view == SRC_S) {
    k.qlo = (k.y / a.c + 1) * a.l;
    k.qhi = a.N - 1;
  } else {
    k.qlo = k.y;
    if (a.pattern == SA_ALL) k.qhi = a.N - 1;
    else if (a.pattern == SA_FIXED) k.qhi = (k.y / a.l) * a.l + a.l - 1;  // also SA_BLOCK (same view)
    else k.qhi = k.y + a.l - 1;
  }
  if (k.qhi > a.N - 1) k.qhi = a.N - 1;
  if (!k.kvalid) k.qhi = k.qlo - 1;
  return k;
}

// dV / dK rows of one key for columns [c0, c0 + NC): add the secondary
// partial (natural pass) and store bf16, or store the fp32 partial
// (secondary pass).  g holds NC fp32 values, already scaled.
template <int D, int NC>
__device__ __forceinline__ void store_grad_row(const BwdArgs& a, int which, size_t off, int c0, float* g,
                                               bool partial_out, bool add) {
  if (partial_out) {
    float* dstp = (which ? a.dk_part : a.dv_part) + off + c0;
#pragma unroll
    for (int u = 0; u < NC; u += 4)
      *reinterpret_cast<float4*>(dstp + u) = make_float4(g[u], g[u + 1], g[u + 2], g[u + 3]);
    return;
  }
  if (add) {
    const float* srcp = (which ? a.dk_part : a.dv_part) + off + c0;
#pragma unroll
    for (int u = 0; u < NC; u += 4) {
      const float4 t = *reinterpret_cast<const float4*>(srcp + u);
      g[u] += t.x;
      g[u + 1] += t.y;
      g[u + 2] += t.z;
      g[u + 3] += t.w;
    }
  }
  uint4* dstp = reinterpret_cast<uint4*>((which ? a.dk : a.dv) + off + c0);
#pragma unroll
  for (int u = 0; u < NC; u += 8) {
    uint4 w;
    w.x = pack_bf16(g[u], g[u + 1]);
    w.y = pack_bf16(g[u + 2], g[u + 3]);
    w.z = pack_bf16(g[u + 4], g[u + 5]);
    w.w = pack_bf16(g[u + 6], g[u + 7]);
    dstp[u / 8] = w;
  }
}

// FINAL_T: the pass writes final bf16 dK/dV in column-major order (the
// column view of SA_COLUMN, which has no natural view).
// BLK: a caller block mask whose blocks are smaller than a tile (the
// entries' sub-block bits are applied on PARTIAL steps).
// DQM: the DqMode of the pass.
// SUM_RED: the natural pass of the fixed pattern adds its dK/dV rows of the
// summary keys to the summary view's fp32 partials by TMA reduce-add (and a
// later launch rounds them to bf16) instead of loading the partials and
// storing the sum itself.
template <int D, bool LONG, bool FINAL_T, bool BLK = false, int DQM = kDqReduce, bool SUM_RED = false>
__global__ void __launch_bounds__(480, 1)
    sa_bwd_kernel(const __grid_constant__ CUtensorMap mq_nat, const __grid_constant__ CUtensorMap mq_col,
                  const __grid_constant__ CUtensorMap mdo_nat, const __grid_constant__ CUtensorMap mdo_col,
                  const __grid_constant__ CUtensorMap mk_nat, const __grid_constant__ CUtensorMap mk_col,
                  const __grid_constant__ CUtensorMap mk_sum, const __grid_constant__ CUtensorMap mv_nat,
                  const __grid_constant__ CUtensorMap mv_col, const __grid_constant__ CUtensorMap mv_sum,
                  const __grid_constant__ CUtensorMap mdq_nat, const __grid_constant__ CUtensorMap mdq_col,
                  const __grid_constant__ CUtensorMap mdk_out, const __grid_constant__ CUtensorMap mdv_out,
                  const __grid_constant__ CUtensorMap mdk_part, const __grid_constant__ CUtensorMap mdv_part,
                  const BwdArgs a) {
  using C = BwdCfg<D, LONG>;
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
  uint8_t* sPT = smem + C::OFF_PT;
  uint8_t* sDST = smem + C::OFF_DST;
  float* sLD = reinterpret_cast<float*>(smem + C::OFF_LD);  // [STAGES][2][64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_kv_full = bars;                          // [KVB]
  uint64_t* bar_kv_empty = bar_kv_full + C::KVB;         // [KVB]
  uint64_t* bar_qdo_full = bar_kv_empty + C::KVB;        // [STAGES]
  uint64_t* bar_qdo_empty = bar_qdo_full + C::STAGES;    // [STAGES]
  // Per global-step-parity barriers (one per elementwise group), so that a
  // barrier is never waited on two phases ahead.
  uint64_t* bar_st_full = bar_qdo_empty + C::STAGES;     // [2]  ST of a step in TMEM
  uint64_t* bar_st_free = bar_st_full + 2;               // [2]  elementwise has read it
  uint64_t* bar_dpt_full = bar_st_free + 2;              // [2]  dPT of a step in TMEM
  uint64_t* bar_dpt_free = bar_dpt_full + 2;             // [2]  elementwise has read it
  uint64_t* bar_pt_full = bar_dpt_free + 2;              // [2]
  uint64_t* bar_pt_free = bar_pt_full + 2;               // [2]
  uint64_t* bar_dst_full = bar_pt_free + 2;              // [2]
  uint64_t* bar_dst_free = bar_dst_full + 2;             // [DST_BUFS] per global pair
  uint64_t* bar_dq_full = bar_dst_free + C::DST_BUFS;    // [DQBUF] per dQ product
  uint64_t* bar_dq_free = bar_dq_full + C::DQBUF;        // [DQBUF]
  uint64_t* bar_dkv_full = bar_dq_free + C::DQBUF;       // [DKVB] per non-empty item
  uint64_t* bar_dkv_free = bar_dkv_full + C::DKVB;       // [DKVB]
  uint64_t* bar_epi = bar_dkv_free + C::DKVB;            // [4] partial rows landed (epilogue warp)
  uint64_t* bar_drain = bar_epi + 4;                     // [2] each issuer's last commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q_src = (a.key_view == SRC_T) ? SRC_T : SRC_N;
  const int n_items = a.n_slots * a.BH;
  const int cta = blockIdx.x, n_ctas = gridDim.x;

  if (threadIdx.x == 0) {
    for (int b = 0; b < C::KVB; ++b) {
      mbar_init(bar_kv_full + b, 1);
      mbar_init(bar_kv_empty + b, 1);
    }
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_qdo_full + s, 1);
      mbar_init(bar_qdo_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_st_full + b, 1);
      mbar_init(bar_st_free + b, 128);
      mbar_init(bar_dpt_full + b, 1);
      mbar_init(bar_dpt_free + b, 128);
      mbar_init(bar_pt_full + b, 128);
      mbar_init(bar_pt_free + b, 1);
      mbar_init(bar_dst_full + b, 128);
    }
    for (int b = 0; b < C::DST_BUFS; ++b) mbar_init(bar_dst_free + b, 1);
    for (int b = 0; b < C::DQBUF; ++b) {
      mbar_init(bar_dq_full + b, 1);
      mbar_init(bar_dq_free + b, 128);
    }
    for (int b = 0; b < C::DKVB; ++b) {
      mbar_init(bar_dkv_full + b, 1);
      mbar_init(bar_dkv_free + b, 128);
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      int gs = 0, ne = 0, issued = 0, kv_issued = 0;
      BwdItem nxt = (cta < n_items) ? bwd_item(a, cta) : BwdItem{0, 0, 0, 0};
      for (int k = 0, item = cta; ok && item < n_items;) {
        const BwdItem it = nxt;
        item = zigzag_item(++k, cta, n_ctas);
        if (item < n_items) nxt = bwd_item(a, item);
        if (it.n == 0) continue;
        const int kb = ne % C::KVB;
        if (ne >= C::KVB && !mbar_wait(bar_kv_empty + kb, ((ne / C::KVB) - 1) & 1, abort_flag)) break;
        ++kv_issued;
        mbar_arrive_expect_tx(bar_kv_full + kb, 2 * C::KV_BYTES);
        load_rows<D>(sK + kb * C::KV_BYTES, a.key_view, it.kt * C::TK, C::TK, it.bh, &mk_nat, &mk_col, &mk_sum,
                     bar_kv_full + kb, a.R, a.l, a.c, a.box.b[box_index(C::TK)]);
        load_rows<D>(sV + kb * C::KV_BYTES, a.key_view, it.kt * C::TK, C::TK, it.bh, &mv_nat, &mv_col, &mv_sum,
                     bar_kv_full + kb, a.R, a.l, a.c, a.box.b[box_index(C::TK)]);
        const float* ld = (q_src == SRC_T ? a.ld_col : a.ld_nat) + static_cast<size_t>(it.bh) * a.n_pad * 2;
        int e_next = a.ent[it.e0];
        for (int j = 0; j < it.n; ++j) {
          const int g = gs + j;
          const int st = g % C::STAGES;
          const int e = e_next;
          if (j + 1 < it.n) e_next = a.ent[it.e0 + j + 1];
          if (g >= C::STAGES && !mbar_wait(bar_qdo_empty + st, ((g / C::STAGES) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          ++issued;
#ifdef SA_TEST_HOOKS
          if (g == 0 && *(volatile int*)&g_test_withhold) continue;  // the first step's tiles never arrive
#endif
          const int qpos = (e >> 3) * C::TQ;
          mbar_arrive_expect_tx(bar_qdo_full + st, 2 * C::QS_BYTES + C::LD_BYTES);
          load_rows<D>(sQ + st * C::QS_BYTES, q_src, qpos, C::TQ, it.bh, &mq_nat, &mq_col, &mq_col,
                       bar_qdo_full + st, a.R, a.l, a.c, a.box.b[box_index(C::TQ)]);
          load_rows<D>(sDO + st * C::QS_BYTES, q_src, qpos, C::TQ, it.bh, &mdo_nat, &mdo_col, &mdo_col,
                       bar_qdo_full + st, a.R, a.l, a.c, a.box.b[box_index(C::TQ)]);
          bulk_load(sLD + st * 2 * C::TQ, ld + 2 * qpos, C::LD_BYTES, bar_qdo_full + st);
        }
        gs += it.n;
        ++ne;
      }
      // After an abort, wait (bounded) for the loads still in flight, so that
      // no copy lands in shared memory after the CTA has exited.
      if (*(volatile int*)abort_flag) {
        for (int h = kv_issued > C::KVB ? kv_issued - C::KVB : 0; h < kv_issued; ++h)
          mbar_wait_drain(bar_kv_full + h % C::KVB, (h / C::KVB) & 1);
        for (int h = issued > C::STAGES ? issued - C::STAGES : 0; h < issued; ++h)
          mbar_wait_drain(bar_qdo_full + h % C::STAGES, (h / C::STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer: ST_g, dPT_g
    // Runs up to NBUF steps ahead of the elementwise warps; waits only for a
    // step's Q/dO and for its TMEM buffer to have been read out.
    if (lane == 0) {
      constexpr uint32_t id_s = make_idesc_bf16(128, C::TQ, false, false);  // N = 64 queries
      bool ok = true;
      int gs = 0, ne = 0;
      BwdItem nxt = (cta < n_items) ? bwd_item(a, cta) : BwdItem{0, 0, 0, 0};
      for (int k = 0, item = cta; ok && item < n_items;) {
        const BwdItem it = nxt;  // the next item's schedule entry is fetched one item ahead
        item = zigzag_item(++k, cta, n_ctas);
        if (item < n_items) nxt = bwd_item(a, item);
        if (it.n == 0) continue;
        const int kb = ne % C::KVB;
        ok = mbar_wait(bar_kv_full + kb, (ne / C::KVB) & 1, abort_flag);
        const uint32_t k_base = smem_u32(sK + kb * C::KV_BYTES), v_base = smem_u32(sV + kb * C::KV_BYTES);
        for (int j = 0; ok && j < it.n; ++j) {
          const int g = gs + j;
          const int st = g % C::STAGES;
          const int b = g % C::NBUF;
          ok = mbar_wait(bar_qdo_full + st, (g / C::STAGES) & 1, abort_flag);
          const int gp = g - C::NBUF;  // last user of TMEM buffer b
          if (ok && gp >= 0) ok = mbar_wait(bar_st_free + (gp & 1), (gp >> 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t q_base = smem_u32(sQ + st * C::QS_BYTES);
          const uint32_t do_base = smem_u32(sDO + st * C::QS_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(tmem + b * 64, bwd_kdesc<D>(k_base, C::TK, kk), bwd_kdesc<D>(q_base, C::TQ, kk), id_s,
                        kk > 0);
          mma_commit(bar_st_full + (g & 1));
          // the dP^T buffer is free once it has been read out or, when it
          // holds P^T (LONG shape), once dV of that step has completed
          if (gp >= 0 &&
              !mbar_wait((C::PT_TMEM ? bar_pt_free : bar_dpt_free) + (gp & 1), (gp >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(tmem + C::COL_DPT + b * 64, bwd_kdesc<D>(v_base, C::TK, kk),
                        bwd_kdesc<D>(do_base, C::TQ, kk), id_s, kk > 0);
          mma_commit(bar_dpt_full + (g & 1));
        }
        gs += it.n;
        ++ne;
      }
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0);
    }
  } else if (warp == 14) {
    // ------------------------------------------------------------ G issuer: dV, dK, dQ
    // Its commits track only its own MMAs; the S issuer's products of a step
    // are complete before the step's P^T exists, so releasing the Q/dO stage
    // after dK (and the K/V buffer after the item's last dQ) covers both.
    if (lane == 0) {
      constexpr uint32_t id_kv = make_idesc_bf16(128, D, false, true);  // dV, dK
      constexpr uint32_t id_q = make_idesc_bf16(128, D, true, true);    // dQ (pair)
      bool ok = true;
      int gs = 0, ne = 0, qi = 0;
      BwdItem nxt = (cta < n_items) ? bwd_item(a, cta) : BwdItem{0, 0, 0, 0};
      for (int k = 0, item = cta; ok && item < n_items;) {
        const BwdItem it = nxt;  // the next item's schedule entry is fetched one item ahead
        item = zigzag_item(++k, cta, n_ctas);
        if (item < n_items) nxt = bwd_item(a, item);
        if (it.n == 0) continue;
        const int kb = ne % C::KVB;
        ok = mbar_wait(bar_kv_full + kb, (ne / C::KVB) & 1, abort_flag);
        // this item's dV/dK buffer must have been read out by the epilogue of
        // the item DKVB before it
        const int vb = ne % C::DKVB;
        if (ok && ne >= C::DKVB) ok = mbar_wait(bar_dkv_free + vb, ((ne / C::DKVB) - 1) & 1, abort_flag);
        const uint32_t k_base = smem_u32(sK + kb * C::KV_BYTES);
        for (int jj = 0; ok && jj < it.n; ++jj) {
          const int g = gs + jj;
          const int st = g % C::STAGES;
          const int pb = g & 1;
          const int P = g >> 1;
          const uint32_t q_base = smem_u32(sQ + st * C::QS_BYTES);
          const uint32_t do_base = smem_u32(sDO + st * C::QS_BYTES);
          const uint32_t dst_pair = smem_u32(sDST + (P % C::DST_BUFS) * C::DST_BYTES);
          if (!mbar_wait(bar_pt_full + pb, (g >> 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          if constexpr (C::PT_TMEM) {
            const uint32_t pt_tmem = tmem + C::COL_DPT + (g % C::NBUF) * 64 + 32;  // 8 columns per k-step
#pragma unroll
            for (int kk = 0; kk < C::TQ / 16; ++kk)
              mma_bf16_ts(tmem + C::COL_DV + vb * 2 * D, pt_tmem + kk * 8, bwd_mndesc<D>(do_base, C::TQ, kk), id_kv,
                          (jj > 0 || kk > 0));
          } else {
            const uint32_t pt_base = smem_u32(sPT + pb * C::PT_BYTES);
#pragma unroll
            for (int kk = 0; kk < C::TQ / 16; ++kk)
              mma_bf16_ss(tmem + C::COL_DV + vb * 2 * D, pt_kdesc(pt_base, kk), bwd_mndesc<D>(do_base, C::TQ, kk),
                          id_kv, (jj > 0 || kk > 0));
          }
          mma_commit(bar_pt_free + pb);
          if (!mbar_wait(bar_dst_full + pb, (g >> 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < C::TQ / 16; ++kk)
            mma_bf16_ss(tmem + C::COL_DK + vb * 2 * D, pt_kdesc(dst_pair + pb * C::PT_BYTES, kk),
                        bwd_mndesc<D>(q_base, C::TQ, kk), id_kv, (jj > 0 || kk > 0));
          mma_commit(bar_qdo_empty + st);
          if ((g & 1) || jj == it.n - 1) {
            // dQ for the item's steps of global pair P (one or two of them)
            const int qb = qi % C::DQBUF;
            if (qi >= C::DQBUF && !mbar_wait(bar_dq_free + qb, ((qi / C::DQBUF) - 1) & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < C::TK / 16; ++kk)
              mma_bf16_ss(tmem + C::COL_DQ + qb * D, pair_mndesc(dst_pair, kk), bwd_mndesc<D>(k_base, C::TK, kk),
                          id_q, kk > 0);
            mma_commit(bar_dq_full + qb);
            // the pair buffer is free once the product covering its odd step is done
            if (g & 1) mma_commit(bar_dst_free + (P % C::DST_BUFS));
            ++qi;
          }
        }
        mma_commit(bar_dkv_full + vb);
        mma_commit(bar_kv_empty + kb);
        gs += it.n;
        ++ne;
      }
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(bar_drain + 1);
      mbar_wait_drain(bar_drain + 1, 0);
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------ elementwise
    // Group `half` takes the global steps g with g % 2 == half, each thread a
    // whole 64-query row in chunks of 16 columns; the two groups run out of
    // phase, so one group's exp2 (MUFU) work overlaps the other's dS work.
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    bool ok = true;
    int gs = 0;
    BwdItem nxt = (cta < n_items) ? bwd_item(a, cta) : BwdItem{0, 0, 0, 0};
    for (int k = 0, item = cta; ok && item < n_items;) {
      const BwdItem it = nxt;  // the next item's schedule entry is fetched one item ahead
      item = zigzag_item(++k, cta, n_ctas);
      if (item < n_items) nxt = bwd_item(a, item);
      if (it.n == 0) continue;
      const KeyRow kr = key_row<D, FINAL_T>(a, it.kt, row);
      for (int j = (half - gs) & 1; j < it.n; j += 2) {
        const int g = gs + j;
        const int e = a.ent[it.e0 + j];
        const int st = g % C::STAGES;
        const int b = g % C::NBUF;
        const int pb = g & 1;
        const int P = g >> 1;
        const bool partial = e & 1;
        const int x0 = (e >> 3) * C::TQ;
        ok = ok && mbar_wait(bar_qdo_full + st, (g / C::STAGES) & 1, abort_flag);
        ok = ok && mbar_wait(bar_st_full + pb, (g >> 1) & 1, abort_flag);
        // P^T buffer pb is free once dV of step g-2 has completed; the dS^T
        // pair buffer once the product over pair P - DST_BUFS has.
        if (!C::PT_TMEM && g >= 2) ok = ok && mbar_wait(bar_pt_free + pb, ((g >> 1) - 1) & 1, abort_flag);
        if (P >= C::DST_BUFS)
          ok = ok && mbar_wait(bar_dst_free + (P % C::DST_BUFS), ((P / C::DST_BUFS) - 1) & 1, abort_flag);
        tc_fence_after();
        const float4* nlse4 = reinterpret_cast<const float4*>(sLD + st * 2 * C::TQ);      // -lse*log2 e
        const float4* ndel4 = reinterpret_cast<const float4*>(sLD + st * 2 * C::TQ + C::TQ);  // -Delta
        uint8_t* pt = sPT + pb * C::PT_BYTES;
        uint8_t* dst = sDST + (P % C::DST_BUFS) * C::DST_BYTES + pb * C::PT_BYTES;
        const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2);
        // (1) the whole S^T row of this key: one TMEM round trip, then 64
        //     independent exp2 back to back (keeps the MUFU pipe busy)
        float sv[64];
#pragma unroll
        for (int c16 = 0; c16 < 4; ++c16) tmem_ld16(tmem + lane_base + b * 64 + c16 * 16, sv + c16 * 16);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar_st_free + pb);
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
        if (partial) {
          if constexpr (BLK) {
            const int nj = C::TQ / a.blk;
            const uint32_t nib = (a.bits[it.e0 + j] >> ((row / a.blk) * nj)) & ((1u << nj) - 1u);
            mask_bits64(sv, interval_bits64(kr.qlo - x0, kr.qhi - x0) & sub_block_cols(nib, a.blk), 0.f);
          } else if constexpr (C::PT_TMEM) {
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const int x = x0 + i;
              if (x < kr.qlo || x > kr.qhi) sv[i] = 0.f;
            }
          } else {
            mask_interval64(sv, kr.qlo - x0, kr.qhi - x0, 0.f);
          }
        }
        if constexpr (!C::PT_TMEM) {
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<uint4*>(pt + sw128_offset(row, ch)) =
                make_uint4(pack_bf16(sv[8 * ch], sv[8 * ch + 1]), pack_bf16(sv[8 * ch + 2], sv[8 * ch + 3]),
                           pack_bf16(sv[8 * ch + 4], sv[8 * ch + 5]), pack_bf16(sv[8 * ch + 6], sv[8 * ch + 7]));
          fence_proxy_async_smem();
          mbar_arrive(bar_pt_full + pb);  // dV of the step may start
        }
        // (2) dP^T row in two halves (its TMEM buffer is released after the
        //     second; in the LONG shape P^T is written over the second half
        //     once both are in registers, and dV releases the buffer);
        //     dS = P (dP - Delta) in fp32 pairs
        ok = ok && mbar_wait(bar_dpt_full + pb, (g >> 1) & 1, abort_flag);
        tc_fence_after();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float dp[32];
          tmem_ld16(tmem + lane_base + C::COL_DPT + b * 64 + hh * 32, dp);
          tmem_ld16(tmem + lane_base + C::COL_DPT + b * 64 + hh * 32 + 16, dp + 16);
          tmem_wait_ld();
          if (hh == 1) {
            if constexpr (C::PT_TMEM) {
              const uint32_t pt_cols = tmem + lane_base + C::COL_DPT + b * 64 + 32;
#pragma unroll
              for (int q8 = 0; q8 < 4; ++q8) {
                uint32_t pk[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) pk[u] = pack_bf16(sv[16 * q8 + 2 * u], sv[16 * q8 + 2 * u + 1]);
                tmem_st8(pt_cols + q8 * 8, pk);
              }
              tmem_wait_st();
              tc_fence_before();
              mbar_arrive(bar_pt_full + pb);  // dV of the step may start
            } else {
              tc_fence_before();
              mbar_arrive(bar_dpt_free + pb);
            }
          }
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const int c0 = hh * 32 + cc * 8;  // first of 8 columns
            const float4 d0 = ndel4[c0 / 4], d1 = ndel4[c0 / 4 + 1];
            const int l0 = cc * 8;
            float2 s01, s23, s45, s67;
            if constexpr (C::PT_TMEM) {
              // scalar form: in this shape it compiles to a faster step than
              // the packed pairs (same arithmetic)
              const float nd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
              float ds[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) ds[u] = sv[c0 + u] * (dp[l0 + u] + nd[u]);
              s01 = make_float2(ds[0], ds[1]);
              s23 = make_float2(ds[2], ds[3]);
              s45 = make_float2(ds[4], ds[5]);
              s67 = make_float2(ds[6], ds[7]);
            } else {
              s01 = f2_unpack(f2_mul(f2_pack(sv[c0], sv[c0 + 1]),
                                     f2_add(f2_pack(dp[l0], dp[l0 + 1]), f2_pack(d0.x, d0.y))));
              s23 = f2_unpack(f2_mul(f2_pack(sv[c0 + 2], sv[c0 + 3]),
                                     f2_add(f2_pack(dp[l0 + 2], dp[l0 + 3]), f2_pack(d0.z, d0.w))));
              s45 = f2_unpack(f2_mul(f2_pack(sv[c0 + 4], sv[c0 + 5]),
                                     f2_add(f2_pack(dp[l0 + 4], dp[l0 + 5]), f2_pack(d1.x, d1.y))));
              s67 = f2_unpack(f2_mul(f2_pack(sv[c0 + 6], sv[c0 + 7]),
                                     f2_add(f2_pack(dp[l0 + 6], dp[l0 + 7]), f2_pack(d1.z, d1.w))));
            }
            *reinterpret_cast<uint4*>(dst + sw128_offset(row, c0 / 8)) =
                make_uint4(pack_bf16(s01.x, s01.y), pack_bf16(s23.x, s23.y), pack_bf16(s45.x, s45.y),
                           pack_bf16(s67.x, s67.y));
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar_dst_full + pb);
      }
      gs += it.n;
    }
  } else if (warp < 14) {
    // ------------------------------------------------------------ dQ reduction + dV/dK epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // query row of a dQ product; key row of the epilogue
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    bool ok = true;
    int gs = 0, ne = 0, qi = 0, epi_n = 0;
    BwdItem nxt = (cta < n_items) ? bwd_item(a, cta) : BwdItem{0, 0, 0, 0};
    for (int k = 0, item = cta; ok && item < n_items;) {
      const BwdItem it = nxt;  // the next item's schedule entry is fetched one item ahead
      item = zigzag_item(++k, cta, n_ctas);
      if (item < n_items) nxt = bwd_item(a, item);
      for (int jj = 0; jj < it.n; ++jj) {
        const int g = gs + jj;
        if (!((g & 1) || jj == it.n - 1)) continue;
        const int qb = qi % C::DQBUF;
        if constexpr (DQM != kDqFinal) {
          ok = ok && mbar_wait(bar_dq_full + qb, (qi / C::DQBUF) & 1, abort_flag);
          tc_fence_after();
        }
        // rows 0..63 belong to global step 2*(g/2), rows 64..127 to the next one
        const int gstep = (g & ~1) + (row >> 6);
        const int js = gstep - gs;
        const bool svalid = js >= 0 && js <= jj;  // the step (and so this warp's 32 rows) is this item's
        const int xw = svalid ? (a.ent[it.e0 + js] >> 3) * C::TQ + (row & 32) : 0;  // warp's first view row
        if constexpr (C::DQ_TMA && DQM == kDqFinal) {
          // The natural pass is the last to reach these rows: dQ = (earlier
          // sum) + s dS K, rounded to bf16 and stored by the lanes (one row
          // each, 16-byte chunks).  The earlier sum is requested into the
          // staging buffer before the product is waited for.
          uint8_t* stg = smem + C::OFF_DQS + quarter * C::DQS_WARP_BYTES;
          const bool fin_in = svalid && a.dq_in;
          if (fin_in) {
            fence_proxy_async_smem();  // earlier reads of the staging come before the load
            __syncwarp();
            if (lane == 0) {
              bulk_wait_read_all();  // earlier stores and reduces have read the staging
              mbar_arrive_expect_tx(bar_epi + quarter, 32 * D * 4);
#pragma unroll
              for (int bx = 0; bx < D / 32; ++bx)
                tma_load_3d(stg + bx * 4096, &mdq_nat, bar_epi + quarter, bx * 32, xw, it.bh);
            }
          }
          ok = ok && mbar_wait(bar_dq_full + qb, (qi / C::DQBUF) & 1, abort_flag);
          tc_fence_after();
          float gq[D];
#pragma unroll
          for (int i = 0; i < D / 16; ++i) tmem_ld16(tmem + lane_base + C::COL_DQ + qb * D + i * 16, gq + i * 16);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar_dq_free + qb);  // the TMEM buffer is free; the rows are in registers
          if (fin_in) {
            if (ok) ok = mbar_wait(bar_epi + quarter, epi_n & 1, abort_flag);
            else mbar_wait_drain(bar_epi + quarter, epi_n & 1);  // the load lands before the kernel ends
            ++epi_n;
          }
          const int x = xw + lane;
          if (svalid && x < a.N) {
            uint4* dst = reinterpret_cast<uint4*>(a.dq_out + (static_cast<size_t>(it.bh) * a.N + x) * D);
#pragma unroll
            for (int bx = 0; bx < D / 32; ++bx)
#pragma unroll
              for (int c8 = 0; c8 < 4; ++c8) {
                float v8[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) v8[u] = gq[bx * 32 + c8 * 8 + u] * a.scale;
                if (fin_in) {
                  const float4 t0 = *reinterpret_cast<const float4*>(stg + bx * 4096 + sw128_offset(lane, 2 * c8));
                  const float4 t1 = *reinterpret_cast<const float4*>(stg + bx * 4096 + sw128_offset(lane, 2 * c8 + 1));
                  v8[0] += t0.x;
                  v8[1] += t0.y;
                  v8[2] += t0.z;
                  v8[3] += t0.w;
                  v8[4] += t1.x;
                  v8[5] += t1.y;
                  v8[6] += t1.z;
                  v8[7] += t1.w;
                }
                dst[bx * 4 + c8] = make_uint4(pack_bf16(v8[0], v8[1]), pack_bf16(v8[2], v8[3]),
                                              pack_bf16(v8[4], v8[5]), pack_bf16(v8[6], v8[7]));
              }
          }
          fence_proxy_async_smem();  // these reads come before the staging's next async write
          __syncwarp();
        } else if constexpr (C::DQ_TMA) {
          float gq[D];
#pragma unroll
          for (int i = 0; i < D / 16; ++i) tmem_ld16(tmem + lane_base + C::COL_DQ + qb * D + i * 16, gq + i * 16);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar_dq_free + qb);  // the TMEM buffer is free; the rows are in registers
          if (svalid) {
            uint8_t* stg = smem + C::OFF_DQS + quarter * C::DQS_WARP_BYTES;
            if (lane == 0) bulk_wait_read_all();  // previous reduce has read the staging buffer
            __syncwarp();
#pragma unroll
            for (int bx = 0; bx < D / 32; ++bx)
#pragma unroll
              for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<float4*>(stg + bx * 4096 + sw128_offset(lane, ch)) =
                    make_float4(gq[bx * 32 + ch * 4] * a.scale, gq[bx * 32 + ch * 4 + 1] * a.scale,
                                gq[bx * 32 + ch * 4 + 2] * a.scale, gq[bx * 32 + ch * 4 + 3] * a.scale);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
#pragma unroll
              for (int bx = 0; bx < D / 32; ++bx) {
                if (q_src == SRC_T) {
                  const int rb = a.box.b[0].rb_t;
                  for (int s0 = 0; s0 < 32; s0 += rb) {
                    const int t = xw + s0;
                    if constexpr (DQM == kDqStore)
                      tma_store_4d(&mdq_col, stg + bx * 4096 + s0 * 128, bx * 32, t / a.R, t % a.R, it.bh);
                    else
                      tma_reduce_add_4d(&mdq_col, stg + bx * 4096 + s0 * 128, bx * 32, t / a.R, t % a.R, it.bh);
                  }
                } else {
                  if constexpr (DQM == kDqStore) tma_store_3d(&mdq_nat, stg + bx * 4096, bx * 32, xw, it.bh);
                  else tma_reduce_add_3d(&mdq_nat, stg + bx * 4096, bx * 32, xw, it.bh);
                }
              }
              bulk_commit_group();
            }
          }
        } else {
          if constexpr (DQM == kDqFinal) {
            ok = ok && mbar_wait(bar_dq_full + qb, (qi / C::DQBUF) & 1, abort_flag);
            tc_fence_after();
          }
          const int x = xw + (row & 31);
          const bool qvalid = svalid && x < a.N;
          const int qn = (q_src == SRC_T) ? (x % a.R) * a.l + x / a.R : x;
          float* dstp = a.dq_acc + (static_cast<size_t>(it.bh) * a.N + (qvalid ? qn : 0)) * D;
#pragma unroll
          for (int i = 0; i < D / 16; ++i) {
            float gq[16];
            tmem_ld16(tmem + lane_base + C::COL_DQ + qb * D + i * 16, gq);
            tmem_wait_ld();
            if (qvalid) {
              if constexpr (DQM == kDqFinal) {  // final dQ row (as in the staged form above)
                float v16[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) v16[u] = gq[u] * a.scale;
                if (a.dq_in) {
#pragma unroll
                  for (int u = 0; u < 16; u += 4) {
                    const float4 t = *reinterpret_cast<const float4*>(dstp + i * 16 + u);
                    v16[u] += t.x;
                    v16[u + 1] += t.y;
                    v16[u + 2] += t.z;
                    v16[u + 3] += t.w;
                  }
                }
                uint4* dst = reinterpret_cast<uint4*>(a.dq_out + (static_cast<size_t>(it.bh) * a.N + qn) * D + i * 16);
#pragma unroll
                for (int u = 0; u < 16; u += 8)
                  dst[u / 8] = make_uint4(pack_bf16(v16[u], v16[u + 1]), pack_bf16(v16[u + 2], v16[u + 3]),
                                          pack_bf16(v16[u + 4], v16[u + 5]), pack_bf16(v16[u + 6], v16[u + 7]));
              } else if constexpr (DQM == kDqStore) {
#pragma unroll
                for (int u = 0; u < 16; u += 4)
                  *reinterpret_cast<float4*>(dstp + i * 16 + u) =
                      make_float4(gq[u] * a.scale, gq[u + 1] * a.scale, gq[u + 2] * a.scale, gq[u + 3] * a.scale);
              } else {
#pragma unroll
                for (int u = 0; u < 16; u += 4)
                  red_add_v4(dstp + i * 16 + u, gq[u] * a.scale, gq[u + 1] * a.scale, gq[u + 2] * a.scale,
                             gq[u + 3] * a.scale);
              }
            }
          }
          tc_fence_before();
          mbar_arrive(bar_dq_free + qb);
        }
        ++qi;
      }
      // ---- dV / dK of this item (thread = key row)
      const KeyRow kr = key_row<D, FINAL_T>(a, it.kt, row);
      if (it.n > 0) {
        ok = ok && mbar_wait(bar_dkv_full + ne % C::DKVB, (ne / C::DKVB) & 1, abort_flag);
        tc_fence_after();
      }
      if constexpr (C::DQ_TMA) {
        // Through this warp's staging buffer: TMEM -> registers (+ the fp32
        // partial rows, fetched by TMA) -> swizzled staging -> one TMA store
        // of the warp's 32 key rows (bf16 dV/dK in the natural pass, fp32
        // partials at the keys' natural positions in a secondary pass).
        uint8_t* stg = smem + C::OFF_DQS + quarter * C::DQS_WARP_BYTES;
        const int y0 = it.kt * C::TK + quarter * 32;  // first view key of the warp
        const bool nat_out = a.key_view == SRC_N || FINAL_T;  // bf16 rows (else fp32 partials)
        bool row_add = false;
        if (nat_out && a.add_part == 1) row_add = kr.kvalid && kr.knat < a.R * a.l;  // keys of whole rows
        else if (nat_out && a.add_part == 2) row_add = kr.kvalid && (kr.knat % a.l) >= (a.l - a.c) && kr.knat < a.R * a.l;
        const bool warp_add = __any_sync(0xffffffffu, row_add);
        if (SUM_RED && warp_add) {
          // Rows of summary keys: their fp32 rows go to the partials by TMA
          // reduce-add (the other rows of the warp are added there too, at
          // positions nothing reads); the warp's rows of other keys are
          // stored as final bf16 rows directly.
          const size_t roff = (static_cast<size_t>(it.bh) * a.N + (kr.kvalid ? kr.knat : 0)) * D;
#pragma unroll 1
          for (int which = 0; which < 2; ++which) {  // 0: dV, 1: dK
            if (lane == 0) bulk_wait_read_all();  // earlier stores and reduces have read the staging
            __syncwarp();
            const uint32_t col = (which ? C::COL_DK : C::COL_DV) + (ne % C::DKVB) * 2 * D;
            const float mul = which ? a.scale : 1.f;
#pragma unroll
            for (int h = 0; h < D / 32; ++h) {
              float gv[32];
              if (it.n > 0) {
                tmem_ld16(tmem + lane_base + col + h * 32, gv);
                tmem_ld16(tmem + lane_base + col + h * 32 + 16, gv + 16);
                tmem_wait_ld();
                if (which == 1 && h == D / 32 - 1) {
                  tc_fence_before();
                  mbar_arrive(bar_dkv_free + ne % C::DKVB);  // both accumulators have been read
                }
              } else {
#pragma unroll
                for (int u = 0; u < 32; ++u) gv[u] = 0.f;
              }
#pragma unroll
              for (int u = 0; u < 32; ++u) gv[u] *= mul;
#pragma unroll
              for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<float4*>(stg + h * 4096 + sw128_offset(lane, ch)) =
                    make_float4(gv[ch * 4], gv[ch * 4 + 1], gv[ch * 4 + 2], gv[ch * 4 + 3]);
              if (!row_add && kr.kvalid) {
                uint4* dstp = reinterpret_cast<uint4*>((which ? a.dk : a.dv) + roff + h * 32);
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4)
                  dstp[c4] = make_uint4(pack_bf16(gv[8 * c4], gv[8 * c4 + 1]), pack_bf16(gv[8 * c4 + 2], gv[8 * c4 + 3]),
                                        pack_bf16(gv[8 * c4 + 4], gv[8 * c4 + 5]),
                                        pack_bf16(gv[8 * c4 + 6], gv[8 * c4 + 7]));
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
#pragma unroll
              for (int bx = 0; bx < D / 32; ++bx)
                tma_reduce_add_3d(which ? &mdk_part : &mdv_part, stg + bx * 4096, bx * 32, y0, it.bh);
              bulk_commit_group();
            }
          }
        } else {
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {  // 0: dV, 1: dK
          if (lane == 0) bulk_wait_read_all();  // earlier stores and reduces have read the staging
          __syncwarp();
          if (warp_add && lane == 0) {
            mbar_arrive_expect_tx(bar_epi + quarter, 32 * D * 4);
#pragma unroll
            for (int bx = 0; bx < D / 32; ++bx)
              tma_load_3d(stg + bx * 4096, which ? &mdk_part : &mdv_part, bar_epi + quarter, bx * 32, y0, it.bh);
          }
          const uint32_t col = (which ? C::COL_DK : C::COL_DV) + (ne % C::DKVB) * 2 * D;
          const float mul = which ? a.scale : 1.f;
          // 32 columns at a time; in the natural pass the bf16 row (D*2 bytes)
          // lands over the first fp32 box, which every lane has read by then
#pragma unroll
          for (int h = 0; h < D / 32; ++h) {
            float gv[32];
            if (it.n > 0) {
              tmem_ld16(tmem + lane_base + col + h * 32, gv);
              tmem_ld16(tmem + lane_base + col + h * 32 + 16, gv + 16);
              tmem_wait_ld();
              if (which == 1 && h == D / 32 - 1) {
                tc_fence_before();
                mbar_arrive(bar_dkv_free + ne % C::DKVB);  // both accumulators have been read
              }
            } else {
#pragma unroll
              for (int u = 0; u < 32; ++u) gv[u] = 0.f;
            }
#pragma unroll
            for (int u = 0; u < 32; ++u) gv[u] *= mul;
            if (h == 0 && warp_add) {  // the partial rows were requested before the TMEM reads
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
              if (h == 0 && warp_add) __syncwarp();
#pragma unroll
              for (int c4 = 0; c4 < 4; ++c4) {
                const int ch = h * 4 + c4;  // 16-byte chunk of the bf16 row
                const uint4 w = make_uint4(pack_bf16(gv[8 * c4], gv[8 * c4 + 1]), pack_bf16(gv[8 * c4 + 2], gv[8 * c4 + 3]),
                                           pack_bf16(gv[8 * c4 + 4], gv[8 * c4 + 5]),
                                           pack_bf16(gv[8 * c4 + 6], gv[8 * c4 + 7]));
                *reinterpret_cast<uint4*>(stg + (D == 64 ? sw128_offset(lane, ch) : sw64_offset(lane, ch))) = w;
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
              const int rb = a.box.b[0].rb_t;
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
                  const int rb = a.box.b[0].rb_t;
                  for (int s0 = 0; s0 < 32; s0 += rb) {
                    const int t = y0 + s0;
                    tma_store_4d(mp, stg + bx * 4096 + s0 * 128, bx * 32, t / a.R, t % a.R, it.bh);
                  }
                } else {
                  const int cb = a.box.b[0].cb_s;
                  if (a.box.b[0].gb_s > 1 || cb == a.c) {  // whole blocks
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
        }
        if (it.n > 0) ++ne;
      } else {
      const size_t off = (static_cast<size_t>(it.bh) * a.N + (kr.kvalid ? kr.knat : 0)) * D;
      bool add = false;
      if (a.add_part == 1) add = kr.knat < a.R * a.l;
      else if (a.add_part == 2) add = (kr.knat % a.l) >= (a.l - a.c) && kr.knat < a.R * a.l;
#pragma unroll
      for (int which = 0; which < 2; ++which) {  // 0: dV, 1: dK
        const uint32_t col = (which ? C::COL_DK : C::COL_DV) + (ne % C::DKVB) * 2 * D;
        const float mul = which ? a.scale : 1.f;
#pragma unroll
        for (int i = 0; i < D / 16; ++i) {
          float gv[16];
          if (it.n > 0) {
            tmem_ld16(tmem + lane_base + col + i * 16, gv);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int u = 0; u < 16; ++u) gv[u] = 0.f;
          }
          if (!kr.kvalid) continue;
#pragma unroll
          for (int u = 0; u < 16; ++u) gv[u] *= mul;
          store_grad_row<D, 16>(a, which, off, i * 16, gv, a.key_view != SRC_N && !FINAL_T, add);
        }
      }
        if (it.n > 0) {
          tc_fence_before();
          mbar_arrive(bar_dkv_free + ne % C::DKVB);
          ++ne;
        }
      }
      gs += it.n;
    }
    if (C::DQ_TMA && lane == 0) bulk_wait_all();
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
//   Delta_i = sum_d dO_id O_id (fp32); writes -lse_i * log2 e and -Delta_i
//   (in [64-step][2][64] blocks) to the natural-order array and, for the
//   strided pattern, at the row's column-major position
//   t = (i mod l) * R + i / l; pads positions [N, n_pad) of both with
//   (-inf, 0); zeroes the fp32 dQ accumulator (null: no pass adds into it).
template <int D>
__global__ void __launch_bounds__(256) sa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dO,
                                                         const float* __restrict__ lse,
                                                         float* __restrict__ ld_nat, float* __restrict__ ld_col,
                                                         float* __restrict__ dq_acc, int BH, int N, int n_pad,
                                                         int l, int R) {
  constexpr int TPR = D / 8;         // threads per row
  constexpr int RPW = 32 / TPR;      // rows per warp per step
  pdl_wait();
  pdl_trigger();
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
        const float nl = -lse[r] * 1.4426950408889634f;
        const long long o = bh * n_pad * 2;
        ld_nat[o + (i / 64) * 128 + (i % 64)] = nl;
        ld_nat[o + (i / 64) * 128 + 64 + (i % 64)] = -acc;
        if (ld_col && i < R * l) {  // rows of a partial last row are not in the column view
          const int t = (i % l) * R + i / l;
          ld_col[o + (t / 64) * 128 + (t % 64)] = nl;
          ld_col[o + (t / 64) * 128 + 64 + (t % 64)] = -acc;
        }
      }
      if (dq_acc) {
        float4* z = reinterpret_cast<float4*>(dq_acc + r * D + sub * 8);
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
  const int pad = n_pad - N;
  for (long long k = tid; k < static_cast<long long>(BH) * pad; k += nthr) {
    const long long bh = k / pad;
    const long long i = N + (k - bh * pad);
    const long long o = bh * n_pad * 2 + (i / 64) * 128 + (i % 64);
    ld_nat[o] = -INFINITY;
    ld_nat[o + 64] = 0.f;
  }
  if (ld_col) {  // the column view covers the R l positions of whole rows
    const int pad_c = n_pad - R * l;
    for (long long k = tid; k < static_cast<long long>(BH) * pad_c; k += nthr) {
      const long long bh = k / pad_c;
      const long long i = static_cast<long long>(R) * l + (k - bh * pad_c);
      const long long o = bh * n_pad * 2 + (i / 64) * 128 + (i % 64);
      ld_col[o] = -INFINITY;
      ld_col[o + 64] = 0.f;
    }
  }
}

// dK, dV (bf16) of the fixed pattern's summary keys = their fp32 partials
// (summary view + the natural view's reduce-adds): positions p with
// p mod l >= l - c of the R whole blocks, 8 channels a thread.
template <int D>
__global__ void __launch_bounds__(256) sa_bwd_summary_final_kernel(const float* __restrict__ dk_part,
                                                                   const float* __restrict__ dv_part,
                                                                   __nv_bfloat16* __restrict__ dk,
                                                                   __nv_bfloat16* __restrict__ dv, int BH, int N,
                                                                   int l, int c, int R) {
  pdl_wait();
  pdl_trigger();
  constexpr int V = D / 8;  // 8-channel vectors per row
  const long long n = static_cast<long long>(BH) * R * c * V;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long key = i / V;
    const int v = static_cast<int>(i - key * V);
    const long long bh = key / (static_cast<long long>(R) * c);
    const int sk = static_cast<int>(key - bh * R * c);  // summary key of the head
    const int p = (sk / c) * l + (l - c) + sk % c;
    const size_t off = (static_cast<size_t>(bh) * N + p) * D + v * 8;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const float4* src = reinterpret_cast<const float4*>((which ? dk_part : dv_part) + off);
      const float4 a0 = src[0], a1 = src[1];
      *reinterpret_cast<uint4*>((which ? dk : dv) + off) =
          make_uint4(pack_bf16(a0.x, a0.y), pack_bf16(a0.z, a0.w), pack_bf16(a1.x, a1.y), pack_bf16(a1.z, a1.w));
    }
  }
}

// dq (bf16) = dq_acc (fp32, already scaled).
__global__ void __launch_bounds__(256) sa_bwd_final_kernel(const float* __restrict__ acc,
                                                           __nv_bfloat16* __restrict__ dq,
                                                           long long n8) {
  pdl_wait();
  pdl_trigger();
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
