// C ABI of the factorized sparse attention library (declared in
// include/sparse_attn.h): argument checks, TMA tensor maps, per-device
// copies of the layout tables, kernel launches, the device status word and
// launch instrumentation.  All device code is in this translation unit.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <type_traits>
#include <utility>
#include <new>
#include <vector>

#include "sa_bwd.cuh"
#include "sa_device.cuh"
#include "sa_fwd.cuh"
#include "sa_internal.h"
#include "sa_tail.cuh"
#include "sparse_attn.h"

namespace sa {
namespace {

// ------------------------------------------------------------ instrumentation
enum Kind {
  K_FWD_COL = 0, K_FWD_MAIN, K_BWD_PRE, K_BWD_SEC, K_BWD_MAIN, K_BWD_FINAL, K_FWD_TAIL, K_BWD_TAIL, K_BWD_SUMFIN,
  K_KERNELS
};
const char* const kKernelNames[K_KERNELS] = {"sa_fwd_column_view",  "sa_fwd_natural_view", "sa_bwd_preprocess",
                                             "sa_bwd_secondary_view", "sa_bwd_natural_view", "sa_bwd_finalize_dq",
                                             "sa_fwd_partial_row",  "sa_bwd_partial_row",  "sa_bwd_finalize_summary_dkv"};
constexpr int K_PATTERNS = 7;
const char* const kPatternNames[K_PATTERNS] = {"all", "local", "strided", "fixed", "column", "block", "blocks"};
// Instrumentation kinds: one per (kernel, pattern), kind = kernel * K_PATTERNS + pattern.
constexpr int K_NUM = K_KERNELS * K_PATTERNS;
char g_kind_names[K_NUM][48];
std::once_flag g_names_once;

const char* kind_name(int kind) {
  std::call_once(g_names_once, [] {
    for (int k = 0; k < K_NUM; ++k)
      std::snprintf(g_kind_names[k], sizeof(g_kind_names[k]), "%s.%s", kKernelNames[k / K_PATTERNS],
                    kPatternNames[k % K_PATTERNS]);
  });
  return g_kind_names[kind];
}

struct Pending {
  int kind;
  cudaEvent_t e0, e1;
};

struct Timing {
  std::mutex mu;
  bool on = false;
  std::vector<Pending> pending;
  std::vector<cudaEvent_t> pool;
  double total_ms[K_NUM] = {};
  long long count[K_NUM] = {};
};
Timing g_timing;
std::atomic<long long> g_launches{0};

cudaEvent_t take_event() {
  if (!g_timing.pool.empty()) {
    cudaEvent_t e = g_timing.pool.back();
    g_timing.pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

void drain_timing_locked() {
  for (auto& p : g_timing.pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(p.e1) == cudaSuccess && cudaEventElapsedTime(&ms, p.e0, p.e1) == cudaSuccess) {
      g_timing.total_ms[p.kind] += ms;
      g_timing.count[p.kind] += 1;
    }
    g_timing.pool.push_back(p.e0);
    g_timing.pool.push_back(p.e1);
  }
  g_timing.pending.clear();
}

template <class F>
int launch(int kind, cudaStream_t s, F&& f) {
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  bool timed = false;
  {
    std::lock_guard<std::mutex> g(g_timing.mu);
    if (g_timing.on) {
      e0 = take_event();
      e1 = take_event();
      timed = (e0 && e1);
    }
  }
  if (timed) cudaEventRecord(e0, s);
  f();
  const cudaError_t err = cudaGetLastError();
  g_launches.fetch_add(1);
  if (timed) {
    cudaEventRecord(e1, s);
    std::lock_guard<std::mutex> g(g_timing.mu);
    g_timing.pending.push_back({kind, e0, e1});
  }
  return err == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

// Launches a kernel with programmatic stream serialisation, so that it can
// start its set-up while the previous kernel in the stream drains (every
// kernel of the library waits for its predecessor with griddepcontrol.wait
// before touching global memory).  SA_NO_PDL=1 in the environment launches
// normally instead.
bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("SA_NO_PDL");
    return !(e && e[0] == '1');
  }();
  return on;
}

template <class... P, class... A>
void launch_kernel(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

#ifdef SA_TEST_HOOKS
// Range check of a device tile table (test build): row pointers start at 0,
// never decrease and end at nnz; every entry's tile index lies in
// [0, max_tile); every launch slot names a row and that row's entries.
// Records SA_ERR_LUT in the status word; the kernels launched after it then
// return before touching any table or tensor.
__global__ void sa_check_table_kernel(DevTable t, int max_tile) {
  const int tid = blockIdx.x * blockDim.x + threadIdx.x, nth = gridDim.x * blockDim.x;
  bool bad = false;
  if (tid == 0) bad = t.row_ptr[0] != 0 || t.row_ptr[t.n_rows] != t.nnz;
  for (int i = tid; i < t.n_rows; i += nth) {
    bad |= t.row_ptr[i + 1] < t.row_ptr[i];
    const int o = t.order[i];
    bad |= o < 0 || o >= t.n_rows;
    const int4 sc = *reinterpret_cast<const int4*>(t.sched + 4 * i);
    bad |= sc.x < 0 || sc.x >= t.n_rows || sc.y < 0 || sc.z < 0 || sc.y + sc.z > t.nnz;
  }
  for (int i = tid; i < t.nnz; i += nth) {
    const int tile = t.ent[i] >> 3;
    bad |= tile < 0 || tile >= max_tile || ((t.ent[i] >> 1) & 3) > SRC_S;
  }
  if (bad) atomicExch(&g_status, kStatusLut);
}

int check_tables(const DeviceCopy& dc, int N, cudaStream_t s) {
  const DevTable* ts[4] = {&dc.fwd_main, &dc.fwd_col, &dc.bwd_main, &dc.bwd_sec};
  for (const DevTable* t : ts) {
    if (t->n_rows == 0) continue;
    sa_check_table_kernel<<<8, 256, 0, s>>>(*t, N / 64 + 2);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  }
  return SA_OK;
}
#endif

// ------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool have_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

struct Geo {
  int BH, N, D, l, c, R;
  int boxw;
  CUtensorMapSwizzle swz;
};

// Natural order: {D, N, BH}, box {boxw, rows, 1}.
int map_nat(CUtensorMap* m, const void* base, const Geo& g, int rows) {
  const cuuint64_t dims[3] = {(cuuint64_t)g.D, (cuuint64_t)g.N, (cuuint64_t)g.BH};
  const cuuint64_t strides[2] = {(cuuint64_t)g.D * 2, (cuuint64_t)g.N * g.D * 2};
  const cuuint32_t box[3] = {(cuuint32_t)g.boxw, (cuuint32_t)rows, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                        es, CU_TENSOR_MAP_INTERLEAVE_NONE, g.swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SA_OK : SA_ERR_CUDA;
}

// The sequence as a 2-D array with rows of length l: {D, l, R, BH}.
// Column view box {boxw, 1, min(R, rows), 1}; summary box
// {boxw, cb, gb, 1} from summary_box(c, rows).
int map_grid(CUtensorMap* m, const void* base, const Geo& g, uint32_t b1, uint32_t b2) {
  const cuuint64_t dims[4] = {(cuuint64_t)g.D, (cuuint64_t)g.l, (cuuint64_t)g.R, (cuuint64_t)g.BH};
  const cuuint64_t strides[3] = {(cuuint64_t)g.D * 2, (cuuint64_t)g.l * g.D * 2, (cuuint64_t)g.N * g.D * 2};
  const cuuint32_t box[4] = {(cuuint32_t)g.boxw, b1, b2, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                        es, CU_TENSOR_MAP_INTERLEAVE_NONE, g.swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SA_OK : SA_ERR_CUDA;
}

struct MapSet {
  CUtensorMap nat, col, sum;
};

// fp32 maps over the dQ accumulator [BH, N, D] for TMA bulk reduce-add:
// natural {D, N, BH} box {32, 32, 1}; column-major {D, l, R, BH} box
// {32, 1, min(R, 32), 1}; 128-byte swizzle (32 fp32 per row of a box).
int make_dq_maps(CUtensorMap* nat, CUtensorMap* col, const float* base, const Geo& g, int pattern) {
  std::memset(nat, 0, sizeof(*nat));
  std::memset(col, 0, sizeof(*col));
  if (g.D > 64) return SA_OK;  // not used for D = 128
  const cuuint32_t es[4] = {1, 1, 1, 1};
  {
    const cuuint64_t dims[3] = {(cuuint64_t)g.D, (cuuint64_t)g.N, (cuuint64_t)g.BH};
    const cuuint64_t strides[2] = {(cuuint64_t)g.D * 4, (cuuint64_t)g.N * g.D * 4};
    const cuuint32_t box[3] = {32, 32, 1};
    if (g_encode(nat, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, es,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return SA_ERR_CUDA;
  }
  if ((pattern == SA_STRIDED || pattern == SA_COLUMN) && g.R > 0) {  // R = 0: no whole row, no column view
    const cuuint64_t dims[4] = {(cuuint64_t)g.D, (cuuint64_t)g.l, (cuuint64_t)g.R, (cuuint64_t)g.BH};
    const cuuint64_t strides[3] = {(cuuint64_t)g.D * 4, (cuuint64_t)g.l * g.D * 4, (cuuint64_t)g.N * g.D * 4};
    const cuuint32_t box[4] = {32, 1, (cuuint32_t)gcd_int(g.R, 32), 1};
    if (g_encode(col, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float*>(base), dims, strides, box, es,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return SA_ERR_CUDA;
  }
  return SA_OK;
}

// Maps of the dV/dK epilogue (D <= 64), boxes of 32 key rows:
//   out_k/out_v: bf16 dK/dV [BH, N, D], natural {D, N, BH}, box {D, 32, 1}
//     (column-major {D, l, R, BH}, box {D, 1, min(R, 32), 1}, for a
//     column-view pass that writes final outputs)
//   part_k/part_v: fp32 partials [BH, N, D] in the key view of the pass:
//     natural {D, N, BH} box {32, 32, 1}; column-major {D, l, R, BH} box
//     {32, 1, min(R, 32), 1}; summary {D, l, R, BH} box {32, min(c, 32),
//     max(1, 32 / c), 1}; 128-byte swizzle (32 fp32 per box row).
struct EpiMaps {
  CUtensorMap out_k, out_v, part_k, part_v;
};

int make_epi_maps(EpiMaps* em, const void* dk, const void* dv, const float* dk_part, const float* dv_part,
                  const Geo& g, int key_view) {
  std::memset(em, 0, sizeof(*em));
  if (g.D > 64) return SA_OK;  // D = 128 stores with plain instructions
  const cuuint32_t es[4] = {1, 1, 1, 1};
  {
    const auto swz = g.D == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUtensorMap* outs[2] = {&em->out_k, &em->out_v};
    const void* bases[2] = {dk, dv};
    for (int i = 0; i < 2; ++i) {
      CUresult r;
      if (key_view == SRC_T) {  // column-major rows: {D, l, R, BH}, box {D, 1, min(R, 32), 1}
        const cuuint64_t dims[4] = {(cuuint64_t)g.D, (cuuint64_t)g.l, (cuuint64_t)g.R, (cuuint64_t)g.BH};
        const cuuint64_t strides[3] = {(cuuint64_t)g.D * 2, (cuuint64_t)g.l * g.D * 2, (cuuint64_t)g.N * g.D * 2};
        const cuuint32_t box[4] = {(cuuint32_t)g.D, 1, (cuuint32_t)gcd_int(g.R, 32), 1};
        r = g_encode(outs[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(bases[i]), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      } else {
        const cuuint64_t dims[3] = {(cuuint64_t)g.D, (cuuint64_t)g.N, (cuuint64_t)g.BH};
        const cuuint64_t strides[2] = {(cuuint64_t)g.D * 2, (cuuint64_t)g.N * g.D * 2};
        const cuuint32_t box[3] = {(cuuint32_t)g.D, 32, 1};
        r = g_encode(outs[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(bases[i]), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      }
      if (r != CUDA_SUCCESS) return SA_ERR_CUDA;
    }
  }
  CUtensorMap* parts[2] = {&em->part_k, &em->part_v};
  const float* pbases[2] = {dk_part, dv_part};
  for (int i = 0; i < 2; ++i) {
    CUresult r;
    if (key_view == SRC_N) {
      const cuuint64_t dims[3] = {(cuuint64_t)g.D, (cuuint64_t)g.N, (cuuint64_t)g.BH};
      const cuuint64_t strides[2] = {(cuuint64_t)g.D * 4, (cuuint64_t)g.N * g.D * 4};
      const cuuint32_t box[3] = {32, 32, 1};
      r = g_encode(parts[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(pbases[i]), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
      const cuuint64_t dims[4] = {(cuuint64_t)g.D, (cuuint64_t)g.l, (cuuint64_t)g.R, (cuuint64_t)g.BH};
      const cuuint64_t strides[3] = {(cuuint64_t)g.D * 4, (cuuint64_t)g.l * g.D * 4, (cuuint64_t)g.N * g.D * 4};
      int cb = 1, gb = 1;
      summary_box(g.c, 32, &cb, &gb);
      const cuuint32_t box[4] = {32, key_view == SRC_T ? 1u : (cuuint32_t)cb,
                                 key_view == SRC_T ? (cuuint32_t)gcd_int(g.R, 32) : (cuuint32_t)gb, 1};
      r = g_encode(parts[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float*>(pbases[i]), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    if (r != CUDA_SUCCESS) return SA_ERR_CUDA;
  }
  return SA_OK;
}

int make_maps(MapSet* ms, const void* base, const Geo& g, int pattern, int rows) {
  std::memset(ms, 0, sizeof(*ms));
  int st = map_nat(&ms->nat, base, g, rows);
  if (st) return st;
  if ((pattern == SA_STRIDED || pattern == SA_COLUMN) && g.R > 0) {  // R = 0: no whole row, no column view
    st = map_grid(&ms->col, base, g, 1, (uint32_t)gcd_int(g.R, rows));
    if (st) return st;
  }
  if (pattern == SA_FIXED && g.R > 0) {  // R = 0: no whole block, no summary view
    int cb = 1, gb = 1;
    summary_box(g.c, rows, &cb, &gb);
    st = map_grid(&ms->sum, base, g, (uint32_t)cb, (uint32_t)gb);
    if (st) return st;
  }
  return SA_OK;
}

// ------------------------------------------------------------ device tables
int to_device(const sa_layout* L, DeviceCopy* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
  std::lock_guard<std::mutex> g(L->mu);
  for (auto& d : L->dev)
    if (d.device == dev) {
      *out = d;
      return SA_OK;
    }
  constexpr int NT = 4;
  const TileTable* tabs[NT] = {&L->fwd_main, &L->fwd_col, &L->bwd_main, &L->bwd_sec};
  std::vector<int32_t> blob;
  size_t offs[NT][5];
  for (int t = 0; t < NT; ++t) {
    const TileTable& tt = *tabs[t];
    offs[t][3] = blob.size();  // 16-byte aligned: every section is padded to 4 ints
    blob.insert(blob.end(), tt.sched.begin(), tt.sched.end());
    offs[t][0] = blob.size();
    blob.insert(blob.end(), tt.row_ptr.begin(), tt.row_ptr.end());
    while (blob.size() % 4) blob.push_back(0);
    offs[t][1] = blob.size();
    blob.insert(blob.end(), tt.ent.begin(), tt.ent.end());
    while (blob.size() % 4) blob.push_back(0);
    offs[t][2] = blob.size();
    blob.insert(blob.end(), tt.order.begin(), tt.order.end());
    while (blob.size() % 4) blob.push_back(0);
    offs[t][4] = blob.size();
    blob.insert(blob.end(), tt.bits.begin(), tt.bits.end());
    while (blob.size() % 4) blob.push_back(0);
  }
  if (blob.empty()) blob.push_back(0);
  void* dptr = nullptr;
  if (cudaMalloc(&dptr, blob.size() * sizeof(int32_t)) != cudaSuccess) return SA_ERR_CUDA;
  if (cudaMemcpy(dptr, blob.data(), blob.size() * sizeof(int32_t), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaFree(dptr);
    return SA_ERR_CUDA;
  }
  DeviceCopy d;
  d.device = dev;
  d.blob = dptr;
  DevTable* dts[NT] = {&d.fwd_main, &d.fwd_col, &d.bwd_main, &d.bwd_sec};
  const int32_t* base = static_cast<const int32_t*>(dptr);
  for (int t = 0; t < NT; ++t) {
    dts[t]->row_ptr = base + offs[t][0];
    dts[t]->ent = base + offs[t][1];
    dts[t]->order = base + offs[t][2];
    dts[t]->sched = base + offs[t][3];
    dts[t]->bits = tabs[t]->bits.empty() ? nullptr : reinterpret_cast<const uint32_t*>(base + offs[t][4]);
    dts[t]->n_rows = tabs[t]->n_rows;
    dts[t]->nnz = static_cast<int>(tabs[t]->ent.size());
  }
  L->dev.push_back(d);
  *out = d;
  return SA_OK;
}

// ------------------------------------------------------------ checks
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_call(int B, int H, int N, int D, const sa_layout* L) {
  if (!L || B < 1 || H < 1 || N < 1) return SA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 0x7fffffffLL) return SA_ERR_INVALID_ARG;
  if (L->N != N) return SA_ERR_LUT;
  if (D != 32 && D != 64 && D != 128) return SA_ERR_UNSUPPORTED;
  if (D == 32) {
    // Rows of 64 bytes: a TMA box must start on a 128-byte boundary of shared
    // memory, so the column and summary views cannot be moved in runs of an
    // odd number of rows (odd R; odd c above 1).
    if ((L->pattern == SA_STRIDED || L->pattern == SA_COLUMN) && (L->R & 1)) return SA_ERR_UNSUPPORTED;
    if (L->pattern == SA_FIXED && L->c > 1 && (L->c & 1)) return SA_ERR_UNSUPPORTED;
  }
  if (!have_encode()) return SA_ERR_CUDA;
  return SA_OK;
}

Geo make_geo(int B, int H, int N, int D, const sa_layout* L) {
  Geo g;
  g.BH = B * H;
  g.N = N;
  g.D = D;
  g.l = (L->pattern == SA_ALL) ? 1 : L->l;
  g.c = L->c > 0 ? L->c : 1;
  g.R = (L->pattern == SA_STRIDED || L->pattern == SA_FIXED || L->pattern == SA_COLUMN) ? L->R : 1;
  g.boxw = D >= 64 ? 64 : D;
  g.swz = D >= 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return g;
}

template <class K>
int set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess
             ? SA_OK
             : SA_ERR_CUDA;
}

// The pattern whose interval rules the kernels apply: SA_BLOCK has the
// natural view of SA_FIXED (no summary view); SA_BLOCKS is causal inside
// the listed blocks, the rule of SA_ALL (its tables hold only listed blocks,
// and every kernel tile lies inside one block).
int kernel_pattern(int pattern) {
  if (pattern == SA_BLOCK) return SA_FIXED;
  if (pattern == SA_BLOCKS) return SA_ALL;
  return pattern;
}

int sm_count();

// Persistent forward grid: every resident CTA slot (two per SM for D <= 64),
// at most one CTA per item.
unsigned fwd_grid(int n_rows, int BH, int D) {
  const long long items = static_cast<long long>(n_rows) * BH;
  const long long slots = static_cast<long long>(sm_count()) * (D <= 64 ? 2 : 1);
  return static_cast<unsigned>(std::max(1LL, std::min(items, slots)));
}

template <int D>
int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
             float scale, const sa_layout* L, cudaStream_t s) {
  const Geo g = make_geo(B, H, N, D, L);
  MapSet mq, mk, mv;
  int st;
  if ((st = make_maps(&mq, q, g, L->pattern, FwdCfg<D>::TQ))) return st;
  if ((st = make_maps(&mk, k, g, L->pattern, FwdCfg<D>::TK))) return st;
  if ((st = make_maps(&mv, v, g, L->pattern, FwdCfg<D>::TK))) return st;
  // Output maps of the epilogue: 32-row boxes, natural and column-major.
  CUtensorMap mo_nat, mo_col;
  std::memset(&mo_col, 0, sizeof(mo_col));
  if ((st = map_nat(&mo_nat, o, g, 32))) return st;
  if ((L->pattern == SA_STRIDED || L->pattern == SA_COLUMN) && g.R > 0 &&
      (st = map_grid(&mo_col, o, g, 1, static_cast<uint32_t>(gcd_int(g.R, 32)))))
    return st;
  DeviceCopy dc;
  if ((st = to_device(L, &dc))) return st;
#ifdef SA_TEST_HOOKS
  if ((st = check_tables(dc, N, s))) return st;
#endif
  // a caller block mask with blocks below a tile: the variant that applies sub-block bits
  const bool blk = L->pattern == SA_BLOCKS && L->block < kFwdTQ;
  auto kern = blk ? sa_fwd_kernel<D, true> : sa_fwd_kernel<D, false>;
  if ((st = set_smem(kern, FwdCfg<D>::SMEM))) return st;
  FwdArgs a;
  a.bits = blk ? dc.fwd_main.bits : nullptr;
  a.blk = blk ? L->block : 0;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.N = N;
  a.l = g.l;
  a.c = g.c;
  a.R = g.R;
  a.pattern = kernel_pattern(L->pattern);
  a.t_open = (L->pattern == SA_COLUMN) ? 0 : 1;
  a.BH = g.BH;
  a.box = make_boxes(g.R, g.c);
  a.scale_log2 = static_cast<float>(1.4426950408889634 * static_cast<double>(scale));
  // Column view first (SA_STRIDED, SA_COLUMN); the natural view then merges
  // into its result (SA_STRIDED) or runs alone (the other patterns).
  const bool col_pass = dc.fwd_col.n_rows > 0;
  if (col_pass) {
    a.row_ptr = dc.fwd_col.row_ptr;
    a.ent = dc.fwd_col.ent;
    a.order = dc.fwd_col.order;
    a.q_col = 1;
    a.merge = 0;
    a.n_rows = dc.fwd_col.n_rows;
    dim3 grid(fwd_grid(a.n_rows, g.BH, D));
    st = launch(K_FWD_COL * K_PATTERNS + L->pattern, s, [&] {
      launch_kernel(kern, grid, FwdCfg<D>::THREADS, FwdCfg<D>::SMEM, s, mq.nat, mq.col, mk.nat, mk.col, mk.sum, mv.nat,
                    mv.col, mv.sum, mo_nat, mo_col, a);
    });
    if (st) return st;
  }
  // The partial last row of a strided pattern (N not a multiple of l): its
  // column part on CUDA cores, merged below like the column view's.
  const int r_tail = (L->pattern == SA_STRIDED && L->R > 0) ? N - L->R * L->l : 0;
  if (r_tail > 0) {
    const long long warps = static_cast<long long>(g.BH) * r_tail;
    st = launch(K_FWD_TAIL * K_PATTERNS + L->pattern, s, [&] {
      launch_kernel(sa_tail_fwd_kernel<D>, static_cast<unsigned>((warps + 3) / 4), 128, 0, s,
                    static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                    static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(o), lse, g.BH, N, L->l, L->R,
                    a.scale_log2);
    });
    if (st) return st;
  }
  a.row_ptr = dc.fwd_main.row_ptr;
  a.ent = dc.fwd_main.ent;
  a.order = dc.fwd_main.order;
  a.q_col = 0;
  a.merge = (col_pass || r_tail > 0) ? 1 : 0;
  if (dc.fwd_main.n_rows == 0) return SA_OK;  // SA_COLUMN: no natural view
  a.n_rows = dc.fwd_main.n_rows;
  dim3 grid(fwd_grid(a.n_rows, g.BH, D));
  return launch(K_FWD_MAIN * K_PATTERNS + L->pattern, s, [&] {
    launch_kernel(kern, grid, FwdCfg<D>::THREADS, FwdCfg<D>::SMEM, s, mq.nat, mq.col, mk.nat, mk.col, mk.sum, mv.nat,
                  mv.col, mv.sum, mo_nat, mo_col, a);
  });
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }


// The default softmax scale 1/sqrt(D).
float default_scale(int D) { return static_cast<float>(1.0 / std::sqrt(static_cast<double>(D > 0 ? D : 1))); }

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

struct WsLayout {
  size_t ld_nat, ld_col, dq, dk, dv, total;
  int n_pad;
};

// Backward workspace: packed (lse * log2 e, Delta) per query in natural order
// (and column-major order for strided), the fp32 dQ accumulator, and for
// strided / fixed the fp32 dK, dV partials of the secondary view.
WsLayout ws_layout(int B, int H, int N, int D, const sa_layout* L) {
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t rows = BH * N;
  WsLayout w;
  w.n_pad = (N + BwdCfg<64>::TQ - 1) / BwdCfg<64>::TQ * BwdCfg<64>::TQ;
  const size_t ld_bytes = align256(BH * w.n_pad * 8);  // two floats per query position
  w.ld_nat = 0;
  w.ld_col = ld_bytes;
  const bool col = L->pattern == SA_STRIDED || L->pattern == SA_COLUMN;
  w.dq = w.ld_col + (col ? ld_bytes : 0);
  w.dk = w.dq + align256(rows * D * 4);
  const bool sec = L->pattern == SA_STRIDED || L->pattern == SA_FIXED;
  w.dv = w.dk + (sec ? align256(rows * D * 4) : 0);
  w.total = w.dv + (sec ? align256(rows * D * 4) : 0);
  return w;
}

int grid_for(long long work_items, int per_block) {
  long long b = (work_items + per_block - 1) / per_block;
  if (b < 1) b = 1;
  if (b > 148 * 16) b = 148 * 16;
  return static_cast<int>(b);
}

// Every instantiation of the backward kernel that a launch below may pick:
// (FINAL_T, BLK, DqMode) = the column view of SA_COLUMN (reduce or store),
// a secondary or natural pass (reduce, store or final), a natural pass of a
// caller mask with small blocks (reduce or final).
template <int D, bool LONG>
int set_bwd_smem() {
  constexpr int sm = BwdCfg<D, LONG>::SMEM;
  int st;
  if ((st = set_smem(sa_bwd_kernel<D, LONG, false, false, kDqReduce>, sm))) return st;
  if ((st = set_smem(sa_bwd_kernel<D, LONG, false, false, kDqStore>, sm))) return st;
  if ((st = set_smem(sa_bwd_kernel<D, LONG, false, false, kDqFinal>, sm))) return st;
  if ((st = set_smem(sa_bwd_kernel<D, LONG, true, false, kDqReduce>, sm))) return st;
  if ((st = set_smem(sa_bwd_kernel<D, LONG, true, false, kDqStore>, sm))) return st;
  if ((st = set_smem(sa_bwd_kernel<D, LONG, false, true, kDqReduce>, sm))) return st;
  return set_smem(sa_bwd_kernel<D, LONG, false, true, kDqFinal>, sm);
}

template <int D>
int bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
             void* dq, void* dk, void* dv, int B, int H, int N, float scale, const sa_layout* L, void* ws, cudaStream_t s) {
  const Geo g = make_geo(B, H, N, D, L);
  MapSet mq, mdo, mk, mv;
  int st;
  if ((st = make_maps(&mq, q, g, L->pattern, BwdCfg<D>::TQ))) return st;
  if ((st = make_maps(&mdo, dO, g, L->pattern, BwdCfg<D>::TQ))) return st;
  if ((st = make_maps(&mk, k, g, L->pattern, BwdCfg<D>::TK))) return st;
  if ((st = make_maps(&mv, v, g, L->pattern, BwdCfg<D>::TK))) return st;
  DeviceCopy dc;
  if ((st = to_device(L, &dc))) return st;
#ifdef SA_TEST_HOOKS
  if ((st = check_tables(dc, N, s))) return st;
#endif
  if ((st = set_bwd_smem<D, false>())) return st;
  if constexpr (D <= 64) {
    if ((st = set_bwd_smem<D, true>())) return st;
    // the fixed pattern's natural pass with the summary keys' rows reduced into the partials
    if ((st = set_smem(sa_bwd_kernel<D, false, false, false, kDqReduce, true>, BwdCfg<D, false>::SMEM))) return st;
    if ((st = set_smem(sa_bwd_kernel<D, false, false, false, kDqFinal, true>, BwdCfg<D, false>::SMEM))) return st;
  }
  const WsLayout w = ws_layout(B, H, N, D, L);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* ld_nat = reinterpret_cast<float*>(wsb + w.ld_nat);
  float* ld_col = (L->pattern == SA_STRIDED || L->pattern == SA_COLUMN) ? reinterpret_cast<float*>(wsb + w.ld_col)
                                                                        : nullptr;
  float* dq_acc = reinterpret_cast<float*>(wsb + w.dq);
  float* dk_part = reinterpret_cast<float*>(wsb + w.dk);
  float* dv_part = reinterpret_cast<float*>(wsb + w.dv);
  const long long rows = static_cast<long long>(g.BH) * N;
  CUtensorMap mdq_nat, mdq_col;
  if ((st = make_dq_maps(&mdq_nat, &mdq_col, dq_acc, g, L->pattern))) return st;

  const bool sec = dc.bwd_sec.n_rows > 0 && g.R > 0;  // SA_STRIDED, SA_FIXED, SA_COLUMN with a whole row
  const int r_tail = (L->pattern == SA_STRIDED && L->R > 0) ? N - L->R * L->l : 0;
  // The natural pass writes the final dQ itself when each query step meets one
  // of its key tiles; the fp32 accumulator then only carries the earlier
  // passes' sum (and is neither zeroed nor read when there are none).
  const bool dq_fin = L->dq_single && dc.bwd_main.n_rows > 0;
  const bool dq_in = sec || r_tail > 0;
  // ... and the secondary pass stores its rows instead of adding them when it
  // meets each one once and no partial row adds to them first.
  const bool dq_store = sec && L->dq_sec_single && r_tail == 0;
  const bool zero_dq = !(dq_fin && !dq_in) && !dq_store;
  st = launch(K_BWD_PRE * K_PATTERNS + L->pattern, s, [&] {
    launch_kernel(sa_bwd_pre_kernel<D>, grid_for(rows * (D / 8), 256), 256, 0, s,
                  static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, ld_nat, ld_col,
                  zero_dq ? dq_acc : nullptr, g.BH, N, w.n_pad, g.l, g.R);
  });
  if (st) return st;

  BwdArgs a;
  a.ld_nat = ld_nat;
  a.ld_col = ld_col ? ld_col : ld_nat;
  a.n_pad = w.n_pad;
  a.dq_acc = dq_acc;
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.dk_part = dk_part;
  a.dv_part = dv_part;
  a.N = N;
  a.l = g.l;
  a.c = g.c;
  a.R = g.R;
  a.pattern = kernel_pattern(L->pattern);
  a.scale = scale;
  a.scale_log2 = static_cast<float>(1.4426950408889634 * static_cast<double>(scale));
  a.box = make_boxes(g.R, g.c);
  a.bits = nullptr;
  a.blk = 0;
  a.dq_out = static_cast<__nv_bfloat16*>(dq);
  a.dq_in = dq_in ? 1 : 0;
  // SA_COLUMN has no natural view: its column-view pass writes the final dK/dV.
  const bool sec_final = L->pattern == SA_COLUMN;
  a.BH = g.BH;
  const int n_sm = sm_count();
  // Tables whose items average many steps take the LONG shape of the kernel.
  bool summary_reduced = false;  // the natural pass reduced the summary keys' rows into the partials
  auto run = [&](int kind, const DevTable& t, int dqm) -> int {
    EpiMaps em;
    const int mst = make_epi_maps(&em, dk, dv, dk_part, dv_part, g, a.key_view);
    if (mst) return mst;
    const long long items = static_cast<long long>(t.n_rows) * g.BH;
    dim3 grid(static_cast<unsigned>(std::min<long long>(items, n_sm)));
    const bool long_items = D <= 64 && t.nnz >= kBwdLongSteps * static_cast<long long>(t.n_rows);
    const bool final_t = sec_final && a.key_view == SRC_T;
    const bool blk = a.blk > 0;  // caller block mask with blocks below a tile (natural view only)
    const bool sum_red = D <= 64 && !long_items && a.add_part == 2 && !blk && dqm != kDqStore;
    auto go = [&](auto kernel, int threads, int smem) {
      launch_kernel(kernel, grid, threads, smem, s, mq.nat, mq.col, mdo.nat, mdo.col, mk.nat, mk.col, mk.sum, mv.nat,
                    mv.col, mv.sum, mdq_nat, mdq_col, em.out_k, em.out_v, em.part_k, em.part_v, a);
    };
    // the kernel variant of a shape: (FINAL_T, BLK) x DqMode
    auto pick = [&](auto shape) {
      constexpr bool L = decltype(shape)::value;
      using CF = BwdCfg<D, L>;
      if (final_t) {
        if (dqm == kDqStore) go(sa_bwd_kernel<D, L, true, false, kDqStore>, CF::THREADS, CF::SMEM);
        else go(sa_bwd_kernel<D, L, true, false, kDqReduce>, CF::THREADS, CF::SMEM);
      } else if (blk) {
        if (dqm == kDqFinal) go(sa_bwd_kernel<D, L, false, true, kDqFinal>, CF::THREADS, CF::SMEM);
        else go(sa_bwd_kernel<D, L, false, true, kDqReduce>, CF::THREADS, CF::SMEM);
      } else if (dqm == kDqFinal) {
        go(sa_bwd_kernel<D, L, false, false, kDqFinal>, CF::THREADS, CF::SMEM);
      } else if (dqm == kDqStore) {
        go(sa_bwd_kernel<D, L, false, false, kDqStore>, CF::THREADS, CF::SMEM);
      } else {
        go(sa_bwd_kernel<D, L, false, false, kDqReduce>, CF::THREADS, CF::SMEM);
      }
    };
    if (sum_red) summary_reduced = true;
    return launch(kind, s, [&] {
      if constexpr (D <= 64) {
        if (sum_red) {
          using CS = BwdCfg<D, false>;
          if (dqm == kDqFinal) go(sa_bwd_kernel<D, false, false, false, kDqFinal, true>, CS::THREADS, CS::SMEM);
          else go(sa_bwd_kernel<D, false, false, false, kDqReduce, true>, CS::THREADS, CS::SMEM);
          return;
        }
        if (long_items) {
          pick(std::true_type{});
          return;
        }
      }
      pick(std::false_type{});
    });
  };
  if (sec) {
    a.sched = dc.bwd_sec.sched;
    a.ent = dc.bwd_sec.ent;
    a.n_slots = dc.bwd_sec.n_rows;
    a.key_view = (L->pattern == SA_FIXED) ? SRC_S : SRC_T;
    a.add_part = 0;
    if ((st = run(K_BWD_SEC * K_PATTERNS + L->pattern, dc.bwd_sec, dq_store ? kDqStore : kDqReduce))) return st;
  }
  if (r_tail > 0) {  // the partial last row's column part (after the column view's pass)
    const long long warps = static_cast<long long>(g.BH) * r_tail;
    st = launch(K_BWD_TAIL * K_PATTERNS + L->pattern, s, [&] {
      launch_kernel(sa_tail_bwd_kernel<D>, static_cast<unsigned>((warps + 3) / 4), 128, 0, s,
                    static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                    static_cast<const __nv_bfloat16*>(v), static_cast<const __nv_bfloat16*>(dO),
                    static_cast<const float*>(ld_nat), dq_acc, dk_part, dv_part, g.BH, N, L->l, L->R, w.n_pad, scale,
                    a.scale_log2);
    });
    if (st) return st;
  }
  if (dc.bwd_main.n_rows > 0) {
    a.bits = dc.bwd_main.bits;
    a.blk = (L->pattern == SA_BLOCKS && L->block < kBwdTK) ? L->block : 0;
    a.sched = dc.bwd_main.sched;
    a.ent = dc.bwd_main.ent;
    a.n_slots = dc.bwd_main.n_rows;
    a.key_view = SRC_N;
    a.add_part = (sec && !sec_final) ? (L->pattern == SA_STRIDED ? 1 : 2) : 0;
    if ((st = run(K_BWD_MAIN * K_PATTERNS + L->pattern, dc.bwd_main, dq_fin ? kDqFinal : kDqReduce))) return st;
  }
  if (summary_reduced && g.R > 0) {  // the summary keys' dK, dV: their fp32 sums rounded to bf16
    const long long n = static_cast<long long>(g.BH) * g.R * g.c * (D / 8);
    st = launch(K_BWD_SUMFIN * K_PATTERNS + L->pattern, s, [&] {
      launch_kernel(sa_bwd_summary_final_kernel<D>, grid_for(n, 256), 256, 0, s, static_cast<const float*>(dk_part),
                    static_cast<const float*>(dv_part), static_cast<__nv_bfloat16*>(dk),
                    static_cast<__nv_bfloat16*>(dv), g.BH, N, g.l, g.c, g.R);
    });
    if (st) return st;
  }
  if (dq_fin) return SA_OK;
  const long long n8 = rows * D / 8;
  return launch(K_BWD_FINAL * K_PATTERNS + L->pattern, s, [&] {
    launch_kernel(sa_bwd_final_kernel, grid_for(n8, 256), 256, 0, s, static_cast<const float*>(dq_acc),
                  static_cast<__nv_bfloat16*>(dq), n8);
  });
}

}  // namespace
}  // namespace sa

// ==================================================================== C ABI
using namespace sa;

extern "C" {

int sparse_attn_layout_blocks(int N, int block, const int32_t* row_ptr, const int32_t* col_idx, sa_layout** out) {
  if (!out) return SA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!row_ptr || !col_idx || N < 1 || block < 1) return SA_ERR_INVALID_ARG;
  // blocks of a multiple of 128 (every kernel tile inside one block), or of
  // 16, 32 or 64 positions (tiles carry which of their blocks are listed)
  const bool whole = block % kFwdTQ == 0 && block % kBwdTK == 0;
  if (!(whole || block == 16 || block == 32 || block == 64) || N % block != 0) return SA_ERR_UNSUPPORTED;
  sa_layout* L = new (std::nothrow) sa_layout();
  if (!L) return SA_ERR_INVALID_ARG;
  L->pattern = SA_BLOCKS;
  L->N = N;
  L->l = 1;
  L->c = 0;
  L->block = block;
  L->R = 1;
  const int st = build_layout_blocks(L, row_ptr, col_idx);
  if (st != SA_OK) {
    delete L;
    return st;
  }
  *out = L;
  return SA_OK;
}

int sparse_attn_layout(int pattern, int N, int l, int c, int block, sa_layout** out) {
  if (!out) return SA_ERR_INVALID_ARG;
  *out = nullptr;
  if (pattern < SA_ALL || pattern > SA_BLOCK || N < 1 || block < 1) return SA_ERR_INVALID_ARG;
  if (pattern != SA_ALL && l < 1) return SA_ERR_INVALID_ARG;
  if (pattern == SA_FIXED && (c < 1 || c > l)) return SA_ERR_INVALID_ARG;
  if (N % block != 0) return SA_ERR_UNSUPPORTED;
  // R = N / l whole rows of the 2-D view.  With N not a multiple of l, the
  // fixed pattern's summary view keeps the whole blocks (the keys of a
  // partial last block are seen by no later block), and the strided
  // pattern's column view covers the whole rows while the partial row's
  // column part runs in its own kernels.  The single column head (SA_COLUMN)
  // needs whole rows.
  const bool grid2d = pattern == SA_STRIDED || pattern == SA_FIXED || pattern == SA_COLUMN;
  if (pattern == SA_COLUMN && N % l != 0) return SA_ERR_UNSUPPORTED;
  sa_layout* L = new (std::nothrow) sa_layout();
  if (!L) return SA_ERR_INVALID_ARG;
  L->pattern = pattern;
  L->N = N;
  L->l = (pattern == SA_ALL) ? 1 : l;
  L->c = (pattern == SA_FIXED) ? c : 0;
  L->block = block;
  L->R = grid2d ? N / l : 1;
  const int st = build_layout(L);
  if (st != SA_OK) {
    delete L;
    return st;
  }
  *out = L;
  return SA_OK;
}

int sparse_attn_layout_export(const sa_layout* L, int view, int32_t* row_ptr, int32_t* col_idx, uint8_t* kind,
                              int* n_rows, int* nnzb) {
  if (!L || !n_rows || !nnzb) return SA_ERR_INVALID_ARG;
  const int v = view & 3;
  const bool tr = (view & SA_VIEW_TRANSPOSED) != 0;
  if (v > SA_VIEW_SUMMARY || (view & ~(3 | SA_VIEW_TRANSPOSED))) return SA_ERR_INVALID_ARG;
  if (!L->has[v]) {
    *n_rows = 0;
    *nnzb = 0;
    if (row_ptr) row_ptr[0] = 0;
    return SA_OK;
  }
  const Csr& t = tr ? L->viewT[v] : L->view[v];
  *n_rows = t.n_rows;
  *nnzb = static_cast<int>(t.col_idx.size());
  if (row_ptr) std::memcpy(row_ptr, t.row_ptr.data(), t.row_ptr.size() * sizeof(int32_t));
  if (col_idx && !t.col_idx.empty()) std::memcpy(col_idx, t.col_idx.data(), t.col_idx.size() * sizeof(int32_t));
  if (kind && !t.kind.empty()) std::memcpy(kind, t.kind.data(), t.kind.size());
  return SA_OK;
}

int sparse_attn_layout_info(const sa_layout* L, int* pattern, int* N, int* l, int* c, int* block) {
  if (!L) return SA_ERR_INVALID_ARG;
  if (pattern) *pattern = L->pattern;
  if (N) *N = L->N;
  if (l) *l = L->l;
  if (c) *c = L->c;
  if (block) *block = L->block;
  return SA_OK;
}

int sparse_attn_layout_upload(const sa_layout* L, void* stream) {
  (void)stream;
  if (!L) return SA_ERR_INVALID_ARG;
  DeviceCopy dc;
  return to_device(L, &dc);
}

void sparse_attn_layout_free(sa_layout* L) {
  if (!L) return;
  int cur = -1;
  const bool have = cudaGetDevice(&cur) == cudaSuccess;
  for (auto& d : L->dev) {
    if (cudaSetDevice(d.device) == cudaSuccess) {
      cudaDeviceSynchronize();
      cudaFree(d.blob);
    }
  }
  if (have && !L->dev.empty()) cudaSetDevice(cur);
  delete L;
}

int sparse_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int D,
                    const sa_layout* L, void* stream) {
  return sparse_attn_fwd_ex(q, k, v, o, lse, B, H, N, D, default_scale(D), L, stream);
}

int sparse_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int D,
                       float scale, const sa_layout* L, void* stream) {
  if (!q || !k || !v || !o || !lse) return SA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return SA_ERR_INVALID_ARG;
  int st = check_call(B, H, N, D, L);
  if (st) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (D) {
    case 32: return fwd_impl<32>(q, k, v, o, lse, B, H, N, scale, L, s);
    case 64: return fwd_impl<64>(q, k, v, o, lse, B, H, N, scale, L, s);
    default: return fwd_impl<128>(q, k, v, o, lse, B, H, N, scale, L, s);
  }
}

size_t sparse_attn_bwd_workspace_size(int B, int H, int N, int D, const sa_layout* L) {
  if (!L || B < 1 || H < 1 || N < 1 || D < 1) return 0;
  return ws_layout(B, H, N, D, L).total;
}

int sparse_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                    void* dq, void* dk, void* dv, int B, int H, int N, int D, const sa_layout* L, void* workspace,
                    size_t ws_bytes, void* stream) {
  return sparse_attn_bwd_ex(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, D, default_scale(D), L, workspace, ws_bytes,
                            stream);
}

int sparse_attn_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                       void* dq, void* dk, void* dv, int B, int H, int N, int D, float scale, const sa_layout* L,
                       void* workspace, size_t ws_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return SA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return SA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, lse, dO, dq, dk, dv};
  for (const void* p : ptrs)
    if (!aligned16(p)) return SA_ERR_INVALID_ARG;
  int st = check_call(B, H, N, D, L);
  if (st) return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) ||
      ws_bytes < sparse_attn_bwd_workspace_size(B, H, N, D, L))
    return SA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (D) {
    case 32: return bwd_impl<32>(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, scale, L, workspace, s);
    case 64: return bwd_impl<64>(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, scale, L, workspace, s);
    default: return bwd_impl<128>(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, scale, L, workspace, s);
  }
}

int sparse_attn_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return SA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return SA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
    return v;
  }
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

const char* sparse_attn_strerror(int status) {
  switch (status) {
    case SA_OK: return "ok";
    case SA_ERR_INVALID_ARG: return "invalid argument";
    case SA_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case SA_ERR_CUDA: return "CUDA error";
    case SA_ERR_LUT: return "layout does not match the call";
    case SA_ERR_TIMEOUT: return "device-side wait timed out";
    case SA_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int sparse_attn_kernel_kinds(void) { return K_NUM; }

int sparse_attn_timing_enable(int on) {
  std::lock_guard<std::mutex> g(g_timing.mu);
  g_timing.on = (on != 0);
  return SA_OK;
}

int sparse_attn_timing_reset(void) {
  std::lock_guard<std::mutex> g(g_timing.mu);
  drain_timing_locked();
  for (int i = 0; i < K_NUM; ++i) {
    g_timing.total_ms[i] = 0;
    g_timing.count[i] = 0;
  }
  return SA_OK;
}

int sparse_attn_timing_read(int kind, const char** name, double* total_ms, long long* launches) {
  if (kind < 0 || kind >= K_NUM) return SA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(g_timing.mu);
  drain_timing_locked();
  if (name) *name = kind_name(kind);
  if (total_ms) *total_ms = g_timing.total_ms[kind];
  if (launches) *launches = g_timing.count[kind];
  return SA_OK;
}

long long sparse_attn_launch_count(void) { return g_launches.load(); }

}  // extern "C"

// ==================================================================== no-alloc backward
// Scratch for sparse_attn_bwd_noalloc: a file-scope device array, so callers
// that cannot allocate device memory can still run the backward pass.  Host
// code must not use the symbol itself as a device address; the address is
// looked up per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_sa_noalloc_scratch[SA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 128;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_sa_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return SA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return SA_OK;
}

// True when the layout's tables are already on the current device.
bool layout_on_device(const sa_layout* L) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> g(L->mu);
  for (const auto& d : L->dev)
    if (d.device == dev) return true;
  return false;
}
}  // namespace

extern "C" int sparse_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                       const float* lse, const void* dO, void* dq, void* dk, void* dv, int B,
                                       int H, int N, int D, const sa_layout* L, void* stream) {
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return SA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, lse, dO, dq, dk, dv};
  for (const void* p : ptrs)
    if (!aligned16(p)) return SA_ERR_INVALID_ARG;
  int st = check_call(B, H, N, D, L);
  if (st) return st;
  const size_t need = sparse_attn_bwd_workspace_size(B, H, N, D, L);
  if (need == 0 || need > SA_NOALLOC_SCRATCH_BYTES) return SA_ERR_WORKSPACE;
  if (!layout_on_device(L)) return SA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch))) return st;
  return sparse_attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, D, L, scratch, SA_NOALLOC_SCRATCH_BYTES,
                         stream);
}

#ifdef SA_TEST_HOOKS
// ==================================================================== test build only
// Not part of the ABI (the header does not declare them): hooks of the
// failure-detection tests, exported by libsparse_attn_test.so alone.
extern "C" int sparse_attn_test_withhold(int on) {
  return cudaMemcpyToSymbol(g_test_withhold, &on, sizeof(int)) == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

// Overwrites entry `index` of the forward natural-view tile table of the
// layout's copy on the current device with `value` (a corrupted table).
extern "C" int sparse_attn_test_corrupt_entry(const sa_layout* L, int index, int value) {
  DeviceCopy dc;
  const int st = to_device(L, &dc);
  if (st) return st;
  if (index < 0 || index >= dc.fwd_main.nnz) return SA_ERR_INVALID_ARG;
  return cudaMemcpy(const_cast<int32_t*>(dc.fwd_main.ent) + index, &value, sizeof(int), cudaMemcpyHostToDevice) ==
                 cudaSuccess
             ? SA_OK
             : SA_ERR_CUDA;
}
#endif
