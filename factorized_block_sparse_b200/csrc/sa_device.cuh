// Device helpers for sm_100a: mbarriers with bounded waits, TMA tile loads,
// tcgen05 (TMEM allocation, MMA, loads/stores) and shared-memory matrix
// descriptors.  Inline PTX written against the PTX ISA; descriptor bit
// layouts follow the sm100 UMMA descriptor definitions in CUTLASS/CuTe.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sa_internal.h"

namespace sa {

// Status word (one per device).  Kernels record problems here instead of
// trapping; the host reads and clears it in sparse_attn_status().  All
// device code lives in one translation unit (sa_api.cu), which includes
// this header once.
__device__ int g_status = 0;

constexpr int kStatusTimeout = 5;  // == SA_ERR_TIMEOUT
constexpr int kStatusLut = 4;      // == SA_ERR_LUT

#ifdef SA_TEST_HOOKS
// Test build (libsparse_attn_test.so, for the failure-detection tests only):
// device-side waits give up after about 2^22 cycles (a few milliseconds), a
// flag makes the backward producer withhold one load so that a wait runs
// out, and the device tables are range-checked before the kernels use them.
constexpr long long kWaitCycles = 1LL << 22;
__device__ int g_test_withhold = 0;
#else
constexpr long long kWaitCycles = 1LL << 31;
#endif

// Rows per TMA box of the column-major view (runs of R rows) and the summary
// view (runs of c keys per block) for a tile of `rows` view positions that
// starts at a multiple of `rows`: every box stays inside one run.
__host__ __device__ __forceinline__ int gcd_int(int a, int b) {
  while (b) {
    const int t = a % b;
    a = b;
    b = t;
  }
  return a;
}
// Summary-view box for a tile of `rows` keys: {cb rows of a block, gb blocks}.
// Whole blocks when c divides rows, part of one block when rows divides c,
// else boxes of gcd(c, rows) rows.
__host__ __device__ __forceinline__ void summary_box(int c, int rows, int* cb, int* gb) {
  if (rows % c == 0) {
    *cb = c;
    *gb = rows / c;
  } else {
    *cb = gcd_int(c, rows);
    *gb = 1;
  }
}

// TMA box geometry of the column and summary views for tiles of 32, 64 and
// 128 rows (index 0, 1, 2), computed on the host: rb_t rows per box of the
// column view; the summary view moves whole blocks when cb_s == c (gb_s
// blocks per box), else runs of cb_s keys inside one block.
struct BoxGeo {
  int rb_t, cb_s, gb_s;
};
struct BoxSet {
  BoxGeo b[3];
};
__host__ __device__ constexpr int box_index(int rows) { return rows == 32 ? 0 : (rows == 64 ? 1 : 2); }
inline BoxSet make_boxes(int R, int c) {
  BoxSet s;
  for (int i = 0; i < 3; ++i) {
    const int rows = 32 << i;
    s.b[i].rb_t = gcd_int(R, rows);
    summary_box(c, rows, &s.b[i].cb_s, &s.b[i].gb_s);
  }
  return s;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: a waiting thread is parked by the
// hardware until the phase completes or about `hint_ns` nanoseconds pass,
// instead of spinning and taking issue slots from the working warps.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity.  After about 2^31 SM
// cycles (2^22 in the test build) without completion (or once any CTA has already recorded a
// timeout) it records SA_ERR_TIMEOUT in the status word, sets *abort and
// returns false; callers then skip the remaining work and drain.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*(volatile int*)abort) return false;
  const long long t0 = clock64();
  uint32_t spins = 0;
  while (!mbar_try_wait_hint(bar, parity, 20000u)) {
    if (((++spins) & 15u) == 0) {
      if (*(volatile int*)abort || *(volatile int*)&g_status == kStatusTimeout) {
        *(volatile int*)abort = 1;
        return false;
      }
      if (clock64() - t0 > kWaitCycles) {
        atomicExch(&g_status, kStatusTimeout);
        *(volatile int*)abort = 1;
        return false;
      }
    }
  }
  return true;
}

// ------------------------------------------------ programmatic dependent launch
// The library launches its kernels with programmatic stream serialisation:
// a kernel may start (barrier set-up, TMEM allocation, static table reads)
// while the previous kernel in the stream drains.  pdl_wait() blocks until
// that kernel has completed and its writes are visible; every kernel calls it
// before its first access to data another kernel may write or read.  It
// returns at once for an ordinary launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next kernel in the stream begin launching; its CTAs start once
// every CTA of this grid has called this or exited.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Bounded wait used only to drain in-flight asynchronous work (loads, MMAs)
// after an abort: it ignores the abort flag and gives up after about 2^26
// cycles.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > (1LL << 26)) return;
  }
}

// ---------------------------------------------------------------- fences
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* m, uint64_t* bar, int x,
                                            int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

// Untiled bulk copy global -> shared (both 16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Bulk tensor reduce-add (fp32) from shared memory into global memory,
// tracked by bulk async-groups of the issuing thread.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* m, const void* src, int x, int y, int z) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void tma_reduce_add_4d(const CUtensorMap* m, const void* src, int x, int y, int z,
                                                  int w) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}
// Bulk tensor store from shared memory into global memory (elements outside
// the tensor are not written), tracked by bulk async-groups.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* m, const void* src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* m, const void* src, int x, int y, int z, int w) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z), "r"(w)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the sources of all committed bulk groups have been read.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until all committed bulk groups have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ------------------------------------------------------- staged tile lists
// Each CTA copies its row of the tile table into shared memory once, so no
// role pays a global-memory round trip per step.  Longer rows (beyond
// kMaxStagedEnt entries) read the tail from global memory.
constexpr int kMaxStagedEnt = 1024;

__device__ __forceinline__ void stage_entries(int32_t* s_ent, const int32_t* g_ent, int n) {
  const int m = n < kMaxStagedEnt ? n : kMaxStagedEnt;
  for (int i = threadIdx.x; i < m; i += blockDim.x) s_ent[i] = g_ent[i];
}

__device__ __forceinline__ int entry_at(const int32_t* s_ent, const int32_t* g_ent, int j) {
  return j < kMaxStagedEnt ? s_ent[j] : g_ent[j];
}

// ---------------------------------------------------------------- tcgen05
template <int NCOLS>
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "n"(NCOLS)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

template <int NCOLS>
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "n"(NCOLS)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]: A (M x K bf16, K-major) sits in TMEM
// with row m on lane m and two consecutive K elements per 32-bit column.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once) on an mbarrier when all previously issued tcgen05 ops of
// this thread have completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns: thread t gets lane (base + t).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  const uint32_t* r = reinterpret_cast<const uint32_t*>(v);
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32"
      " [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// 32 lanes x 32 bit, 8 consecutive columns from registers.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// 32 lanes x 32 bit, 32 consecutive columns from registers.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32"
      " [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16,"
      " %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
      "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// ------------------------------------------------- matrix descriptors
// Shared-memory matrix descriptor (tcgen05): start address >> 4 in bits
// [0,14), leading-dimension byte offset >> 4 in [16,30), stride-dimension
// byte offset >> 4 in [32,46), version 1 in [46,48), swizzle mode in
// [61,64) (2 = 128-byte, 4 = 64-byte).
constexpr uint64_t kSwizzle128 = 2;
constexpr uint64_t kSwizzle64 = 4;

__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, uint32_t lbo_bytes,
                                              uint32_t sbo_bytes, uint64_t swizzle) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= swizzle << 61;
  return d;
}

// Instruction descriptor, kind::f16 with bf16 A and B, fp32 D:
// D format bits [4,6) = 1 (f32), A format [7,10) = 1 (bf16), B format
// [10,13) = 1 (bf16), A major bit 15, B major bit 16 (1 = MN-major),
// N >> 3 in [17,23), M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t make_idesc_bf16(int M, int N, bool a_mn_major,
                                                       bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// ------------------------------------------------------------- math
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Packed fp32x2 arithmetic (sm_100): two lanes of a 64-bit register pair.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// fp32 vector reduction into global memory (sm_90+).
__device__ __forceinline__ void red_add_v4(float* gptr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(gptr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

// Keeps v[i] for lo <= i <= hi (i in [0, 64)) and sets the others to
// `fill`: the interval becomes one 64-bit mask, then one bit test and one
// select per element.
__device__ __forceinline__ void mask_interval64(float* v, int lo, int hi, float fill) {
  lo = max(lo, 0);
  hi = min(hi, 63);
  uint32_t m0 = 0u, m1 = 0u;
  if (lo <= hi) {
    const uint64_t m = (~0ull << lo) & (~0ull >> (63 - hi));
    m0 = static_cast<uint32_t>(m);
    m1 = static_cast<uint32_t>(m >> 32);
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = ((m0 >> i) & 1u) ? v[i] : fill;
#pragma unroll
  for (int i = 0; i < 32; ++i) v[32 + i] = ((m1 >> i) & 1u) ? v[32 + i] : fill;
}

// Caller block masks with blocks smaller than a tile: the 64-bit mask of the
// columns whose sub-block is listed.  Bit j of `nib` covers columns
// [j * blk, (j + 1) * blk) (blk = 16, 32 or 64).
__device__ __forceinline__ uint64_t sub_block_cols(uint32_t nib, int blk) {
  const uint64_t one = (blk >= 64) ? ~0ull : ((1ull << blk) - 1ull);
  uint64_t m = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (j * blk < 64 && ((nib >> j) & 1u)) m |= one << (j * blk);
  return m;
}

// The interval [lo, hi] of a 64-column tile as a mask (empty when lo > hi).
__device__ __forceinline__ uint64_t interval_bits64(int lo, int hi) {
  lo = max(lo, 0);
  hi = min(hi, 63);
  return (lo <= hi) ? ((~0ull << lo) & (~0ull >> (63 - hi))) : 0ull;
}

// Keeps v[i] where bit i of m is set, sets the others to `fill`.
__device__ __forceinline__ void mask_bits64(float* v, uint64_t m, float fill) {
  const uint32_t m0 = static_cast<uint32_t>(m), m1 = static_cast<uint32_t>(m >> 32);
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = ((m0 >> i) & 1u) ? v[i] : fill;
#pragma unroll
  for (int i = 0; i < 32; ++i) v[32 + i] = ((m1 >> i) & 1u) ? v[32 + i] : fill;
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a K-major tile whose
// rows are 128 bytes (64 bf16) wide, swizzled 128B (8-row atoms of 1 KiB).
__device__ __forceinline__ uint32_t sw128_offset(int row, int chunk) {
  return static_cast<uint32_t>((row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4));
}

// The same for 64-byte rows swizzled 64B (16-byte chunk bits 4..5 XOR
// address bits 7..8, i.e. row bits 1..2).
__device__ __forceinline__ uint32_t sw64_offset(int row, int chunk) {
  return static_cast<uint32_t>(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}

}  // namespace sa
