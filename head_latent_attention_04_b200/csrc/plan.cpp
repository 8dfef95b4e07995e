// Host split-KV planner for the persistent decode kernel.
//
// Work unit: one page (64 keys) of one query row.  Each query position i of
// the s_q new tokens is its own row group (the s_q groups run side by side on
// disjoint sets of clusters and walk the same pages at about the same time,
// so the repeated reads of a page tend to hit L2).  Within a
// group the rows are laid end to end in sequence order, each preceded by
// kItemCostPages virtual pages that stand for the fixed cost of starting a
// work item (loading the row's query, writing its output), and this line of
// P' units is cut into `clusters_per_group` contiguous ranges of equal size
// (floor(c * P' / G)).  The intersection of a range with a row's real pages
// is one work item, so a cluster that crosses a row boundary takes fewer
// pages.  A row that falls inside a single range is written directly; a row
// cut by range boundaries gets one partial slot per piece, numbered
// consecutively in row order.
#include "plan_format.h"
#include "mla_internal.h"

#include <algorithm>
#include <vector>

namespace mla {

static inline int32_t kv_len_of(const mla_dims_t& d, int32_t T, int32_t qi) {
  return d.causal ? T - d.s_q + 1 + qi : T;
}

mla_status_t build_plan(const mla_dims_t& d, const int32_t* seq_lens, int32_t num_clusters,
                        int32_t* plan, int64_t plan_words, int32_t* num_slots_out) {
  const int32_t B = d.B, S = d.s_q, N = B * S;
  const int32_t page = d.page_size;
  if (plan_words < plan_words_upper_bound(num_clusters, N))
    return set_error(MLA_ERR_WORKSPACE_TOO_SMALL, "plan buffer smaller than mla_plan_size");

  // rows in order n = b * s_q + qi
  std::vector<int32_t> kv_len(N), pages(N);
  for (int32_t b = 0; b < B; ++b) {
    const int32_t T = seq_lens[b];
    if (T < S || (int64_t)T > (int64_t)d.max_blocks_per_seq * page)
      return set_error(MLA_ERR_INVALID_ARG, "seq_lens[%d] = %d outside [s_q, max_blocks*page]", b, T);
    for (int32_t qi = 0; qi < S; ++qi) {
      kv_len[b * S + qi] = kv_len_of(d, T, qi);
      pages[b * S + qi] = (kv_len[b * S + qi] + page - 1) / page;
    }
  }

  const int32_t groups = (num_clusters >= S) ? S : 1;
  const int32_t per_group = num_clusters / groups;

  // group g holds rows with qi == g (or all rows when groups == 1), in row order
  std::vector<std::vector<int32_t>> group_rows(groups);
  for (int32_t n = 0; n < N; ++n) group_rows[groups == 1 ? 0 : n % S].push_back(n);

  struct Piece { int32_t cluster, row, p0, p1; };
  std::vector<Piece> pieces;                 // in (group, row) order
  std::vector<int32_t> row_pieces(N, 0);
  for (int32_t g = 0; g < groups; ++g) {
    int64_t P = 0;
    for (int32_t n : group_rows[g]) P += kItemCostPages + pages[n];
    int64_t off = 0;
    for (int32_t n : group_rows[g]) {
      const int64_t r0 = off + kItemCostPages, r1 = r0 + pages[n];
      off = r1;
      for (int32_t c = 0; c < per_group; ++c) {
        const int64_t lo = (int64_t)c * P / per_group, hi = (int64_t)(c + 1) * P / per_group;
        const int64_t a = std::max(lo, r0), e = std::min(hi, r1);
        if (a < e) {
          pieces.push_back({g * per_group + c, n, (int32_t)(a - r0), (int32_t)(e - r0)});
          row_pieces[n]++;
        }
      }
    }
  }

  // slots: rows with more than one piece, consecutive per row, in row order
  std::vector<int32_t> row_slot_begin(N + 1, 0);
  for (int32_t n = 0; n < N; ++n)
    row_slot_begin[n + 1] = row_slot_begin[n] + (row_pieces[n] > 1 ? row_pieces[n] : 0);
  const int32_t num_slots = row_slot_begin[N];

  // items grouped by cluster (stable: within a cluster, row order)
  std::vector<int32_t> piece_idx_in_row(pieces.size());
  {
    std::vector<int32_t> seen(N, 0);
    for (size_t i = 0; i < pieces.size(); ++i) piece_idx_in_row[i] = seen[pieces[i].row]++;
  }
  std::vector<size_t> order(pieces.size());
  for (size_t i = 0; i < order.size(); ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(),
                   [&](size_t x, size_t y) { return pieces[x].cluster < pieces[y].cluster; });

  const int32_t I = (int32_t)pieces.size();
  const int32_t off_cluster = kPlanHeaderWords;
  const int32_t off_items = off_cluster + num_clusters + 1;
  const int32_t off_rows = off_items + I * kItemWords;
  const int32_t total = off_rows + N + 1;

  std::fill(plan, plan + plan_words, 0);
  plan[kHdrMagic] = kPlanMagic;
  plan[kHdrNumClusters] = num_clusters;
  plan[kHdrNumItems] = I;
  plan[kHdrNumSlots] = num_slots;
  plan[kHdrNumRows] = N;
  plan[kHdrHeads] = d.n_heads;
  plan[kHdrSq] = S;
  plan[kHdrB] = B;
  plan[kHdrOffCluster] = off_cluster;
  plan[kHdrOffItems] = off_items;
  plan[kHdrOffRows] = off_rows;
  plan[kHdrTotalWords] = total;
  plan[kHdrMaxBlocks] = d.max_blocks_per_seq;
  plan[kHdrCausal] = d.causal ? 1 : 0;

  int32_t* cl = plan + off_cluster;
  for (int32_t c = 0; c <= num_clusters; ++c) cl[c] = 0;
  for (const Piece& p : pieces) cl[p.cluster + 1]++;
  for (int32_t c = 0; c < num_clusters; ++c) cl[c + 1] += cl[c];

  int32_t* it = plan + off_items;
  for (int32_t k = 0; k < I; ++k) {
    const Piece& p = pieces[order[k]];
    int32_t* w = it + k * kItemWords;
    w[kItB] = p.row / S;
    w[kItQi] = p.row % S;
    w[kItPageBegin] = p.p0;
    w[kItPageEnd] = p.p1;
    w[kItKvLen] = kv_len[p.row];
    w[kItSlot] = row_pieces[p.row] > 1 ? row_slot_begin[p.row] + piece_idx_in_row[order[k]] : -1;
    w[kItRow] = p.row;
  }
  int32_t* rs = plan + off_rows;
  for (int32_t n = 0; n <= N; ++n) rs[n] = row_slot_begin[n];

  if (num_slots_out) *num_slots_out = num_slots;
  return MLA_OK;
}

}  // namespace mla
