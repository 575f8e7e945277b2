// Layout builder: block look-up tables of the factorized patterns.
//
// The block-sparse kernels of the Sparse Transformer slice queries and keys
// into blocks and visit only the blocks that hold part of the mask ("OpenAI
// Sparse Transformer", "Implementation and Limitations"; pcnews translation,
// "Релиз кода").  A factorized pattern is block-dense only after the column
// step is relabelled: attention along a column of the 2-D array is attention
// along a row of the transposed array (pcnews translation, "Разреженное
// внимание").  So each pattern is split into views that are dense in their
// own order (natural; column-major for the strided column part; consecutive
// summary keys for the fixed pattern's summary part).
//
// In every view the keys a query position x may see form one interval
// [lo(x), hi(x)] of view key positions (possibly empty), with lo and hi
// non-decreasing in x.  The builder classifies each (query block, key block)
// pair from these intervals, row by row; it never forms the element mask.
#include <algorithm>
#include <cstring>
#include <numeric>

#include "sa_internal.h"

namespace sa {

namespace {

struct Interval {
  long long lo, hi;  // inclusive; empty when lo > hi
};

// Key interval of view position x.
Interval key_interval(const sa_layout* L, int view, long long x) {
  const long long l = L->l, c = L->c, R = L->R;
  if (view == SA_VIEW_NATURAL) {
    switch (L->pattern) {
      case SA_ALL:
        return {0, x};
      case SA_LOCAL:
      case SA_STRIDED:
        return {std::max(0LL, x - l + 1), x};
      default:  // SA_FIXED, SA_BLOCK: own l-block, causal
        return {(x / l) * l, x};
    }
  }
  if (view == SA_VIEW_COLUMN) {
    // Inside the run of x's column, strict unless the view stands alone.
    // Column-major order: columns 0 .. r-1 hold R + 1 positions when N is not
    // a multiple of l (r = N - R l, the length of the partial last row), the
    // others R.
    const long long r = L->N - R * l;
    long long start;
    if (x < r * (R + 1)) {
      start = (x / (R + 1)) * (R + 1);
    } else {
      const long long c = r + (x - r * (R + 1)) / R;
      start = r * (R + 1) + (c - r) * R;
    }
    return {start, L->pattern == SA_COLUMN ? x : x - 1};
  }
  // SA_VIEW_SUMMARY: summary keys of strictly earlier blocks
  return {0, (x / l) * c - 1};
}

Csr build_public(const sa_layout* L, int view) {
  Csr t;
  const int b = L->block;
  const long long nq = L->N;
  const long long nk = view_keys(L, view);
  t.n_rows = static_cast<int>((nq + b - 1) / b);
  t.n_cols = static_cast<int>((nk + b - 1) / b);
  t.row_ptr.assign(1, 0);
  std::vector<Interval> iv(b);
  for (int r = 0; r < t.n_rows; ++r) {
    long long lo_min = nk, hi_max = -1;
    for (int u = 0; u < b; ++u) {
      iv[u] = key_interval(L, view, static_cast<long long>(r) * b + u);
      if (iv[u].lo <= iv[u].hi) {
        lo_min = std::min(lo_min, iv[u].lo);
        hi_max = std::max(hi_max, iv[u].hi);
      }
    }
    if (hi_max >= 0) {
      for (long long cb = lo_min / b; cb <= hi_max / b && cb < t.n_cols; ++cb) {
        const long long y0 = cb * b, y1 = cb * b + b - 1;
        bool any = false, all = (y1 < nk);
        for (int u = 0; u < b; ++u) {
          const long long lo = iv[u].lo, hi = iv[u].hi;
          if (std::max(lo, y0) <= std::min(hi, y1)) any = true;
          if (!(lo <= y0 && hi >= y1)) all = false;
        }
        if (any) {
          t.col_idx.push_back(static_cast<int32_t>(cb));
          t.kind.push_back(all ? SA_BLOCK_FULL : SA_BLOCK_PARTIAL);
        }
      }
    }
    t.row_ptr.push_back(static_cast<int32_t>(t.col_idx.size()));
  }
  return t;
}

Csr transpose(const Csr& a) {
  Csr t;
  t.n_rows = a.n_cols;
  t.n_cols = a.n_rows;
  std::vector<int32_t> cnt(a.n_cols + 1, 0);
  for (int32_t cidx : a.col_idx) cnt[cidx + 1]++;
  for (int i = 0; i < a.n_cols; ++i) cnt[i + 1] += cnt[i];
  t.row_ptr = cnt;
  t.col_idx.resize(a.col_idx.size());
  t.kind.resize(a.kind.size());
  std::vector<int32_t> fill(cnt.begin(), cnt.end() - 1);
  for (int r = 0; r < a.n_rows; ++r) {  // ascending r keeps each output row sorted
    for (int e = a.row_ptr[r]; e < a.row_ptr[r + 1]; ++e) {
      const int32_t dst = fill[a.col_idx[e]]++;
      t.col_idx[dst] = r;
      t.kind[dst] = a.kind[e];
    }
  }
  return t;
}

// Coarsens a public table (rows = major blocks, cols = minor blocks, both of
// `b` positions) to tiles of TM major x Tm minor positions.  n_major and
// n_minor are the view's extents in positions.  Appends entries to `out`.
struct CoarseRow {
  std::vector<std::pair<int, int>> ent;  // (minor tile, partial)
};

std::vector<CoarseRow> coarsen(const Csr& a, int b, int TM, int Tm, long long n_major,
                               long long n_minor) {
  const int n_tiles = static_cast<int>((n_major + TM - 1) / TM);
  std::vector<CoarseRow> rows(n_tiles);
  std::vector<int> full_cnt, touched;
  const int n_minor_tiles = static_cast<int>((n_minor + Tm - 1) / Tm);
  full_cnt.assign(n_minor_tiles, 0);
  std::vector<char> present(n_minor_tiles, 0);
  for (int r = 0; r < n_tiles; ++r) {
    const long long p0 = static_cast<long long>(r) * TM;
    const long long p1 = std::min(p0 + TM, n_major) - 1;
    const int rb0 = static_cast<int>(p0 / b), rb1 = static_cast<int>(p1 / b);
    const int n_rb = rb1 - rb0 + 1;
    touched.clear();
    for (int rb = rb0; rb <= rb1 && rb < a.n_rows; ++rb) {
      for (int e = a.row_ptr[rb]; e < a.row_ptr[rb + 1]; ++e) {
        const long long y0 = static_cast<long long>(a.col_idx[e]) * b;
        const long long y1 = std::min(y0 + b, n_minor) - 1;
        for (long long t = y0 / Tm; t <= y1 / Tm; ++t) {
          if (!present[t]) {
            present[t] = 1;
            touched.push_back(static_cast<int>(t));
          }
          if (a.kind[e] == SA_BLOCK_FULL) full_cnt[t]++;
        }
      }
    }
    std::sort(touched.begin(), touched.end());
    const bool major_whole = (p0 + TM <= n_major) && (p1 == p0 + TM - 1);
    for (int t : touched) {
      const long long q0 = static_cast<long long>(t) * Tm;
      const long long q1 = q0 + Tm - 1;
      const int cb0 = static_cast<int>(q0 / b);
      const int cb1 = static_cast<int>(std::min(q1, n_minor - 1) / b);
      const int need = n_rb * (cb1 - cb0 + 1);
      const bool full = major_whole && (q1 < n_minor) && full_cnt[t] == need;
      rows[r].ent.push_back({t, full ? 0 : 1});
      present[t] = 0;
      full_cnt[t] = 0;
    }
  }
  return rows;
}

void finish_table(TileTable& tt, const std::vector<std::vector<int32_t>>& rows) {
  tt.n_rows = static_cast<int>(rows.size());
  tt.row_ptr.assign(1, 0);
  tt.ent.clear();
  for (const auto& r : rows) {
    tt.ent.insert(tt.ent.end(), r.begin(), r.end());
    tt.row_ptr.push_back(static_cast<int32_t>(tt.ent.size()));
  }
  tt.order.resize(tt.n_rows);
  std::iota(tt.order.begin(), tt.order.end(), 0);
  // Longest rows first; among equals, later rows first.
  std::stable_sort(tt.order.begin(), tt.order.end(), [&](int x, int y) {
    const int lx = tt.row_ptr[x + 1] - tt.row_ptr[x], ly = tt.row_ptr[y + 1] - tt.row_ptr[y];
    if (lx != ly) return lx > ly;
    return x > y;
  });
  tt.sched.assign(4 * static_cast<size_t>(tt.n_rows), 0);
  for (int s = 0; s < tt.n_rows; ++s) {
    const int r = tt.order[s];
    tt.sched[4 * s + 0] = r;
    tt.sched[4 * s + 1] = tt.row_ptr[r];
    tt.sched[4 * s + 2] = tt.row_ptr[r + 1] - tt.row_ptr[r];
  }
}

}  // namespace

int view_keys(const sa_layout* L, int view) {
  if (view == SA_VIEW_SUMMARY) {
    // the last c offsets of every block, the last (partial) block included
    const int tail = L->N - L->R * L->l;
    return L->R * L->c + std::max(0, tail - (L->l - L->c));
  }
  return L->N;
}

namespace {

// Whether every 64-query step of [0, N) is the entry of exactly one key tile
// of a backward table (the fixed pattern's own-block view with l = 128, the
// block-diagonal views, the column view when R divides 64): the pass over
// that table then meets each dQ row once.
bool one_key_tile_per_step(const TileTable& t, int N) {
  const int steps = (N + kBwdTQ - 1) / kBwdTQ;
  if (t.n_rows == 0 || static_cast<long long>(t.ent.size()) != steps) return false;
  std::vector<uint8_t> seen(steps, 0);
  for (const int32_t e : t.ent) {
    const int x = e >> 3;
    if (x < 0 || x >= steps || seen[x]) return false;
    seen[x] = 1;
  }
  return true;
}

// Kernel tile tables from the public tables in L->view / L->viewT.
void build_kernel_tables(sa_layout* L) {
  const long long N = L->N;
  const int b = L->block;

  // Forward, natural query tiles: summary entries first (fixed), then natural.
  if (L->has[SA_VIEW_NATURAL]) {
    auto nat = coarsen(L->view[SA_VIEW_NATURAL], b, kFwdTQ, kFwdTK, N, N);
    std::vector<CoarseRow> sum;
    if (L->has[SA_VIEW_SUMMARY])
      sum = coarsen(L->view[SA_VIEW_SUMMARY], b, kFwdTQ, kFwdTK, N, view_keys(L, SA_VIEW_SUMMARY));
    std::vector<std::vector<int32_t>> rows(nat.size());
    for (size_t r = 0; r < nat.size(); ++r) {
      if (!sum.empty())
        for (auto& e : sum[r].ent) rows[r].push_back(pack_entry(e.first, SRC_S, e.second));
      for (auto& e : nat[r].ent) rows[r].push_back(pack_entry(e.first, SRC_N, e.second));
    }
    finish_table(L->fwd_main, rows);
  } else {
    finish_table(L->fwd_main, {});
  }
  // The column view's kernel passes cover the whole rows of the 2-D view
  // (Ng = R l positions in column-major order); the positions of a partial
  // last row, if any, get their column part from the tail kernels.  With
  // whole rows only this is the public column table itself.
  const long long Ng = static_cast<long long>(L->R) * L->l;
  Csr colg, colgT;
  int bg = b;
  if (L->has[SA_VIEW_COLUMN]) {
    if (Ng == N) {
      colg = L->view[SA_VIEW_COLUMN];
      colgT = L->viewT[SA_VIEW_COLUMN];
    } else {
      sa_layout G;
      G.pattern = L->pattern;
      G.N = static_cast<int>(Ng);
      G.l = L->l;
      G.c = L->c;
      G.R = L->R;
      G.block = bg = kBwdTQ;  // a granularity of every kernel tile
      colg = build_public(&G, SA_VIEW_COLUMN);
      colgT = transpose(colg);
    }
  }
  // Forward, column-order query tiles (strided).
  if (L->has[SA_VIEW_COLUMN]) {
    auto col = coarsen(colg, bg, kFwdTQ, kFwdTK, Ng, Ng);
    std::vector<std::vector<int32_t>> rows(col.size());
    for (size_t r = 0; r < col.size(); ++r)
      for (auto& e : col[r].ent) rows[r].push_back(pack_entry(e.first, SRC_T, e.second));
    finish_table(L->fwd_col, rows);
  } else {
    finish_table(L->fwd_col, {});
  }
  // Backward, natural key tiles -> natural query tiles.
  if (L->has[SA_VIEW_NATURAL]) {
    auto kt = coarsen(L->viewT[SA_VIEW_NATURAL], b, kBwdTK, kBwdTQ, N, N);
    std::vector<std::vector<int32_t>> rows(kt.size());
    for (size_t r = 0; r < kt.size(); ++r)
      for (auto& e : kt[r].ent) rows[r].push_back(pack_entry(e.first, SRC_N, e.second));
    finish_table(L->bwd_main, rows);
  } else {
    finish_table(L->bwd_main, {});
  }
  L->dq_single = one_key_tile_per_step(L->bwd_main, L->N);
  // Backward, secondary view key tiles (T order or summary order).
  if (L->has[SA_VIEW_COLUMN] || L->has[SA_VIEW_SUMMARY]) {
    const int v = L->has[SA_VIEW_COLUMN] ? SA_VIEW_COLUMN : SA_VIEW_SUMMARY;
    const int src = (v == SA_VIEW_COLUMN) ? SRC_T : SRC_S;
    auto kt = (v == SA_VIEW_COLUMN) ? coarsen(colgT, bg, kBwdTK, kBwdTQ, Ng, Ng)
                                    : coarsen(L->viewT[v], b, kBwdTK, kBwdTQ, view_keys(L, v), N);
    std::vector<std::vector<int32_t>> rows(kt.size());
    for (size_t r = 0; r < kt.size(); ++r)
      for (auto& e : kt[r].ent) rows[r].push_back(pack_entry(e.first, src, e.second));
    finish_table(L->bwd_sec, rows);
    L->dq_sec_single = one_key_tile_per_step(L->bwd_sec, static_cast<int>(v == SA_VIEW_COLUMN ? Ng : N));
  } else {
    finish_table(L->bwd_sec, {});
  }
}

}  // namespace

int build_layout(sa_layout* L) {
  const int p = L->pattern;
  L->has[SA_VIEW_NATURAL] = (p != SA_COLUMN);
  L->has[SA_VIEW_COLUMN] = (p == SA_STRIDED || p == SA_COLUMN);
  L->has[SA_VIEW_SUMMARY] = (p == SA_FIXED);
  for (int v = 0; v < 3; ++v) {
    if (!L->has[v]) continue;
    L->view[v] = build_public(L, v);
    L->viewT[v] = transpose(L->view[v]);
  }
  build_kernel_tables(L);
  return SA_OK;
}

namespace {

// Blocks smaller than the kernel tiles (16, 32 or 64 positions): a tile holds
// several blocks, some of which may be unlisted.  Per entry, bit
// (i * nj + j) says whether the i-th block along the tile's rows and the j-th
// along its columns is listed: forward tiles are 128 queries x 64 keys
// (i: query block, j: key block), backward tiles 128 keys x 64 queries
// (i: key block, j: query block).
bool listed(const Csr& t, int qb, int kb) {
  if (qb < 0 || qb >= t.n_rows) return false;
  const auto b = t.col_idx.begin() + t.row_ptr[qb], e = t.col_idx.begin() + t.row_ptr[qb + 1];
  return std::binary_search(b, e, kb);
}

void table_bits(TileTable& tt, const Csr& mask, int b, int tm, int tn, bool key_major) {
  const int ni = tm / b, nj = tn / b;
  tt.bits.assign(tt.ent.size(), 0);
  for (int r = 0; r < tt.n_rows; ++r) {
    for (int e = tt.row_ptr[r]; e < tt.row_ptr[r + 1]; ++e) {
      const int tile = tt.ent[e] >> 3;
      uint32_t m = 0;
      for (int i = 0; i < ni; ++i)
        for (int j = 0; j < nj; ++j) {
          const int rb = r * ni + i, cb = tile * nj + j;  // blocks along the tile's rows / columns
          if (key_major ? listed(mask, cb, rb) : listed(mask, rb, cb)) m |= 1u << (i * nj + j);
        }
      tt.bits[e] = static_cast<int32_t>(m);
    }
  }
}

}  // namespace

void sub_block_bits(sa_layout* L) {
  const Csr& m = L->view[SA_VIEW_NATURAL];
  table_bits(L->fwd_main, m, L->block, kFwdTQ, kFwdTK, false);
  table_bits(L->bwd_main, m, L->block, kBwdTK, kBwdTQ, true);
}

int build_layout_blocks(sa_layout* L, const int32_t* row_ptr, const int32_t* col_idx) {
  // The caller's table is the natural view: per query block, ascending key
  // blocks at or below the diagonal, the diagonal block last.  Diagonal
  // blocks hold the causal triangle (PARTIAL); the others are FULL.
  const int nb = L->N / L->block;
  if (row_ptr[0] != 0) return SA_ERR_INVALID_ARG;
  Csr t;
  t.n_rows = t.n_cols = nb;
  t.row_ptr.assign(1, 0);
  for (int r = 0; r < nb; ++r) {
    const int32_t e0 = row_ptr[r], e1 = row_ptr[r + 1];
    if (e1 <= e0 || col_idx[e1 - 1] != r) return SA_ERR_INVALID_ARG;  // empty, or no diagonal block
    for (int32_t e = e0; e < e1; ++e) {
      const int32_t cb = col_idx[e];
      if (cb < 0 || (e > e0 && cb <= col_idx[e - 1])) return SA_ERR_INVALID_ARG;
      t.col_idx.push_back(cb);
      t.kind.push_back(cb == r ? SA_BLOCK_PARTIAL : SA_BLOCK_FULL);
    }
    t.row_ptr.push_back(static_cast<int32_t>(t.col_idx.size()));
  }
  L->has[SA_VIEW_NATURAL] = true;
  L->view[SA_VIEW_NATURAL] = t;
  L->viewT[SA_VIEW_NATURAL] = transpose(t);
  build_kernel_tables(L);
  if (L->block < kFwdTQ) sub_block_bits(L);
  return SA_OK;
}

}  // namespace sa
