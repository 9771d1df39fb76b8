// kernels.cuh -- parameter blocks and launch helpers shared by the kernels
// and the C-ABI layer.  Host and device.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace fp8idx {

constexpr int kHeads = 32;         // index heads
constexpr int kDim = 128;          // index head dim (bytes per fp8 row)
constexpr int kBlockKeys = 128;    // keys per tile = MMA M = TMEM lanes
constexpr int kPageSize = 64;      // tokens per key page (paged form)
constexpr int kMaxTopK = 2048;
constexpr int kPrefillRows = 8;    // query rows per prefill unit (row block)
constexpr int kMaxEpiWarps = 12;   // epilogue warps per CTA at most (workspace scratch is sized for it)
constexpr int kStatusBytes = 256;  // device status block at the head of every workspace
// Tiles between two votes of an epilogue warp, after t tiles of the unit:
// short early, where the running threshold still moves fast, and growing with
// the tiles already streamed (clamp(t, min, max): the votes fall at about
// t = 4, 8, 16, 32, then every 32 tiles), since the threshold's relative
// movement per tile falls like 1 / t.
constexpr int kMinVoteTiles = 4;
constexpr int kMaxVoteTiles = 32;
__host__ __device__ constexpr int vote_interval(int t) {
  return t < kMinVoteTiles ? kMinVoteTiles : (t > kMaxVoteTiles ? kMaxVoteTiles : t);
}

// device status bits (workspace word 0)
constexpr int kStatusWaitTimeout = 1;
constexpr int kStatusBadPage = 2;
constexpr int kStatusSeqLenTooLong = 4;
constexpr int kStatusCandOverflow = 8;
// device statistics (workspace words 1..) of the fused top-k
constexpr int kStatCompactions = 1;     // in-stream exact compactions of a full candidate buffer
constexpr int kStatGeneralSelects = 2;  // final selects that needed the general radix path
constexpr int kStatCandidates = 3;      // candidates appended, summed over rows
constexpr int kStatMaxBoundary = 4;     // largest boundary-bin population seen
constexpr int kStatRepairs = 5;         // rows whose estimated threshold proved too high (recomputed exactly)
constexpr int kSchedWord = 16;          // status-block word: next unit for dynamic scheduling
constexpr int kRepairCount = 18;        // status-block word: row blocks / requests listed for recomputation
constexpr int kRepairSched = 19;        // status-block word: next listed group for the repair launch
constexpr int kRepairMaxGrid = 32;      // CTAs of a repair launch at most

enum Mode : int { kModeLogits = 0, kModeTopK = 1 };

struct IndexerParams {
  CUtensorMap tmap_q;  // q viewed as [rows * 32, 128] bytes, box {128, R * 32}
  CUtensorMap tmap_k;  // keys [n, 128] (box {128, 128}) or pages [P * 64, 128] (box {128, 64})
  const float* s;      // key scales [n] or [P * 64]
  const float* w;      // head weights [m, 32]
  const int32_t* ks;   // prefill ranges
  const int32_t* ke;
  const int32_t* block_table;  // paged: [B, max_blocks]
  const int32_t* seq_lens;     // paged: [B]
  int64_t n;                   // prefill: number of keys
  int m;                       // query rows (prefill m, paged B * R)
  int max_blocks;
  int num_pages;
  int topk;
  int rows_per_unit;  // query rows of a row block / request (at most the kernel's row capacity)
  int n_chunks;     // key chunks per row block / request
  int chunk_keys;   // keys per chunk (multiple of 128)
  int tail_chunks;  // the last tail_chunks chunks hold tail_keys keys each (multiple of 128), the others chunk_keys
  int tail_keys;
  int num_units;    // row blocks (or requests) x n_chunks
  // logits mode
  float* logits;
  int64_t ld_logits;
  // top-k outputs (direct mode: n_chunks == 1)
  int32_t* out_idx;
  float* out_vals;
  // workspace
  int* status;
  uint2* cand;      // [gridDim.x][2 slots][R][cand_cap] (order key, index); cand_cap % 128 == 0
  int cand_cap;     // per row; split into 4 equal segments, one per key quadrant
  uint2* scratch;   // [gridDim.x][kMaxEpiWarps][topk]: staging of a rare in-kernel compaction
  uint2* part;      // split mode: [num_units][R][topk]
  int* part_cnt;    // split mode: [num_units][R]
  uint32_t* row_theta;  // split mode: [m] best lower bound on each row's k-th order key, zeroed per call
  unsigned long long wait_limit_ns;
  int debug_withhold_first_tile;  // tests only: never issue the first key tile's load (its wait runs out)
  // estimated thresholds: a row's threshold may be raised to an estimate of
  // its k-th value from the keys seen so far; the select (or the merge) checks
  // the estimate against the result and lists the group for recomputation
  int speculate;
  uint32_t* row_spec;   // split mode: [m] largest estimated threshold applied to each row
  int* repair_flag;     // [row blocks / requests]: listed for recomputation (zeroed per call)
  int* repair_list;     // [row blocks / requests]
  int repair_mode;      // this launch recomputes the listed groups, whole rows, exact thresholds
  int out_slots;        // paged: write physical KV slots (block_table[b][j / 64] * 64 + j % 64), not positions j
};

struct MergeParams {
  const uint2* part;
  const int* part_cnt;
  int rows;          // total query rows
  int R;             // query rows per row block / request
  int R_part;        // row stride of the partial lists (the kernel's row capacity)
  int n_chunks;
  int topk;
  int32_t* out_idx;
  float* out_vals;
  const uint32_t* row_spec;  // [rows] largest estimated threshold applied (0: none; NULL: no estimates)
  int* status;               // the call's status block (repair count and stats)
  int* repair_flag;
  int* repair_list;
  const int32_t* block_table;  // non-null: write physical KV slots through this [requests, max_blocks] table
  int max_blocks;
  int num_pages;
};

// Physical KV slot of logical key position j of request b through a block
// table of 64-token pages: -1 for j < 0 or a page entry outside the pool.
__device__ __forceinline__ int32_t slot_of(const int32_t* block_table, int max_blocks, int num_pages, int b,
                                           int32_t j) {
  if (j < 0) return -1;
  const int32_t pg = __ldg(block_table + static_cast<int64_t>(b) * max_blocks + j / kPageSize);
  return pg >= 0 && pg < num_pages ? pg * kPageSize + j % kPageSize : -1;
}

struct TopkRowsParams {
  const float* logits;
  int64_t ld;
  const int32_t* ks;
  const int32_t* ke;
  int64_t n;
  int m;
  int topk;
  int32_t* out_idx;
};

// Launchers (kernels.cu).  They only enqueue work; validation is the caller's.
cudaError_t launch_indexer_prefill_logits(const IndexerParams& p, int H, int grid, cudaStream_t st);
cudaError_t launch_indexer_prefill_topk(const IndexerParams& p, int H, int grid, cudaStream_t st);
cudaError_t launch_indexer_paged_topk(const IndexerParams& p, int R, int H, int grid, cudaStream_t st);
cudaError_t launch_merge(const MergeParams& p, cudaStream_t st);
cudaError_t launch_topk_rows(const TopkRowsParams& p, cudaStream_t st);
cudaError_t launch_fill_empty(int32_t* out_idx, float* out_vals, int rows, int topk,
                              cudaStream_t st);

}  // namespace fp8idx
