// Internal declarations shared by the layout builder, the C ABI and the
// kernels.  Not part of the public interface (include/sparse_attn.h is).
#pragma once

#include <cstdint>
#include <mutex>
#include <vector>

#include "sparse_attn.h"

namespace sa {

// Kernel tile sizes.  The public block tables are at the caller's `block`
// granularity; the kernels run on coarser tiles whose tables are derived
// from them (a tile is present when any block overlapping it is, FULL when
// every overlapping block is FULL and the tile lies inside the view).
constexpr int kFwdTQ = 128;  // forward: query rows per CTA (tcgen05 M)
constexpr int kFwdTK = 64;   // forward: keys per step (tcgen05 N of Q K^T)
constexpr int kBwdTK = 128;  // backward: keys per CTA (tcgen05 M of K Q^T)
constexpr int kBwdTQ = 64;   // backward: queries per step
// Backward tables whose items average at least this many steps run the
// kernel shape with the deeper Q/dO ring (P^T in TMEM).
constexpr int kBwdLongSteps = 4;

enum Src : int { SRC_N = 0, SRC_T = 1, SRC_S = 2 };

// Entry of a kernel tile table: (tile << 3) | (src << 1) | partial.
inline int32_t pack_entry(int tile, int src, int partial) {
  return (tile << 3) | (src << 1) | (partial & 1);
}

struct Csr {
  std::vector<int32_t> row_ptr, col_idx;
  std::vector<uint8_t> kind;
  int n_rows = 0, n_cols = 0;
};

struct TileTable {
  std::vector<int32_t> row_ptr;  // n_rows + 1
  std::vector<int32_t> ent;      // packed entries, ascending tile per source
  std::vector<int32_t> order;    // rows by descending entry count (launch order)
  std::vector<int32_t> sched;    // per launch slot s: {row order[s], its first entry, its count, 0}
  // Caller block masks with blocks smaller than the kernel tiles: per entry,
  // which (row block, column block) pairs of the tile are listed (see
  // sub_block_bits in the layout builder); empty otherwise.
  std::vector<int32_t> bits;
  int n_rows = 0;
};

struct DevTable {
  const int32_t* row_ptr = nullptr;
  const int32_t* ent = nullptr;
  const int32_t* order = nullptr;
  const int32_t* sched = nullptr;  // 16-byte aligned, 4 ints per slot
  const uint32_t* bits = nullptr;  // per entry (caller block masks with blocks below a tile), or null
  int n_rows = 0;
  int nnz = 0;
};

struct DeviceCopy {
  int device = -1;
  void* blob = nullptr;
  DevTable fwd_main, fwd_col, bwd_main, bwd_sec;
};

}  // namespace sa

struct sa_layout {
  int pattern = 0, N = 0, l = 1, c = 0, block = 1, R = 1;
  bool has[3] = {false, false, false};
  sa::Csr view[3];   // public tables, query-block major
  sa::Csr viewT[3];  // public tables, key-block major
  // Kernel tables.
  sa::TileTable fwd_main;  // natural query tiles: N-view keys (+ S-view keys for fixed)
  sa::TileTable fwd_col;   // column-order query tiles: T-view keys (strided)
  sa::TileTable bwd_main;  // natural key tiles: N-view query tiles
  sa::TileTable bwd_sec;   // T-order (strided) or summary-order (fixed) key tiles
  // Every 64-query step of the natural view meets exactly one key tile, so
  // the backward's natural pass completes each dQ row with one product.
  bool dq_single = false;
  // The same for the secondary view's key tiles over the query steps of its
  // whole rows (the column view with R dividing 64).
  bool dq_sec_single = false;
  mutable std::mutex mu;
  mutable std::vector<sa::DeviceCopy> dev;
};

namespace sa {
// Builds every table of a layout (host only).  Returns an sa_status.
int build_layout(sa_layout* L);
// Builds the tables of a caller's block mask (SA_BLOCKS; L->N, L->block set,
// N % block == 0); row_ptr has N / block + 1 entries.  Returns an sa_status.
int build_layout_blocks(sa_layout* L, const int32_t* row_ptr, const int32_t* col_idx);
// Number of key positions of a view (summary view: R * c).
int view_keys(const sa_layout* L, int view);
// Per-entry sub-block bits of a caller block mask with blocks below a tile.
void sub_block_bits(sa_layout* L);
}  // namespace sa
