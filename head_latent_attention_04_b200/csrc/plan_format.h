// Layout of the split-KV plan shared by the host planner and the kernels.
// All entries are int32 words.  The plan is position independent: the
// kernels read it from device memory through the offsets in the header.
#pragma once
#include <stdint.h>

namespace mla {

constexpr int32_t kPlanMagic = 0x314C414D;  // "MLA1" little-endian
constexpr int kPlanHeaderWords = 16;
constexpr int kItemWords = 8;
// Planner cost of starting a work item, in pages: loading the row's query
// into TMEM, refilling the pipeline and writing the output take about as long
// as five pages of the attention pipeline (measured per-cluster finish times:
// 4.5 to 5.6 pages per extra item across the benchmark workloads).
constexpr int32_t kItemCostPages = 5;

enum PlanHeader : int {
  kHdrMagic = 0,
  kHdrNumClusters = 1,
  kHdrNumItems = 2,
  kHdrNumSlots = 3,
  kHdrNumRows = 4,      // N = B * s_q
  kHdrHeads = 5,
  kHdrSq = 6,
  kHdrB = 7,
  kHdrOffCluster = 8,   // cluster_item_begin[num_clusters + 1]
  kHdrOffItems = 9,     // items[num_items][kItemWords]
  kHdrOffRows = 10,     // row_slot_begin[num_rows + 1]
  kHdrTotalWords = 11,
  kHdrMaxBlocks = 12,   // columns of block_table the plan was made for
  kHdrCausal = 13,      // the dims' causal flag the plan was made with
};

// One work item: a contiguous page range of one query row's key sequence.
enum ItemField : int {
  kItB = 0,          // sequence
  kItQi = 1,         // query position within the sequence (0 .. s_q-1)
  kItPageBegin = 2,  // first page (index into the sequence's block_table row)
  kItPageEnd = 3,    // one past the last page
  kItKvLen = 4,      // keys this query attends: tokens [0, kv_len)
  kItSlot = 5,       // partial-output slot, or -1 when the item covers the whole row
  kItRow = 6,        // n = b * s_q + qi
};

inline int64_t plan_words_upper_bound(int32_t num_clusters, int32_t n_rows) {
  const int64_t items = (int64_t)num_clusters + n_rows;
  return kPlanHeaderWords + (num_clusters + 1) + items * kItemWords + (n_rows + 1);
}

inline int64_t plan_slots_upper_bound(int32_t num_clusters, int32_t n_rows) {
  return (int64_t)num_clusters + n_rows;
}

}  // namespace mla
