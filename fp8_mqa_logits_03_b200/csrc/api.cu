// api.cu -- the C ABI (include/fp8idx.h): argument checks, workspace plans,
// TMA descriptor encoding and kernel launches.  Host code only.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/fp8idx.h"
#include "kernels.cuh"

namespace fp8idx {
__device__ int g_logits_status[kStatusBytes / 4];  // status block of the last fp8idx_mqa_logits call

// Fixed scratch of fp8idx_mqa_logits_topk_noalloc: a module-scope device
// array, so it is created when the library's device code is loaded on a GPU
// and lives until the process exits (64 MiB on every GPU that loads it).
// On the host this name is only a stand-in for the device symbol; its device
// address comes from cudaGetSymbolAddress.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

cudaError_t launch_act_quant_store(const uint16_t* x, int64_t T, const int64_t* slot, int64_t num_slots,
                                   uint8_t* k_pool, float* s_pool, cudaStream_t st);
constexpr int kMaxPrepBatch = 8192;
cudaError_t launch_prepare_ragged(const int32_t* seq_len, const int32_t* q_len, const int32_t* req_idx, int B,
                                  const int32_t* table, int64_t table_rows, int64_t ld, int32_t* ks, int32_t* ke,
                                  int32_t* row_table, int64_t q_cap, int32_t* ragged, int64_t ragged_cap,
                                  int sms, cudaStream_t st);
cudaError_t launch_topk_transform(const int32_t* idx, int64_t rows, int topk, const int32_t* row_base,
                                  const int32_t* row_table, int rows_per_table_row, const int32_t* table,
                                  int64_t table_rows, int64_t ld, int page_size, int32_t* out, int sms,
                                  cudaStream_t st);
}

namespace {

using namespace fp8idx;

thread_local std::string t_last_error;
unsigned long long g_wait_limit_ns = 2000000000ull;
int g_debug_withhold = 0;

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return code;
}

int ok() {
  t_last_error.clear();
  return FP8IDX_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(FP8IDX_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms;
}

// ---------------------------------------------------------------- TMA descriptors

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// A [rows, 128]-byte matrix read in boxes of [box_rows, 128] with the
// 128-byte swizzle the MMA descriptors expect.  Rows past the end read as 0.
int make_rows128_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(FP8IDX_ECUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDim), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDim)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kDim), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FP8IDX_ECUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return FP8IDX_OK;
}

// ---------------------------------------------------------------- plans

struct Plan {
  int R = 8;           // the kernel's row capacity per unit (its MMA rows)
  int rows_per_unit = 8;  // query rows of a row block / request (<= R)
  int H = 32;
  int n_chunks = 1;
  int chunk_keys = 0;
  int tail_chunks = 0;  // the last tail_chunks chunks hold tail_keys keys each
  int tail_keys = 0;
  int num_units = 0;
  int groups = 0;      // row blocks (prefill) or requests (paged)
  int64_t axis = 0;    // the whole key axis
  int grid = 0;
  int cap = 0;
  int rgrid = 0;       // CTAs of the repair launch
  int rcap = 0;        // its candidate capacity per row (whole rows)
  size_t off_cand = 0, off_scratch = 0, off_part = 0, off_cnt = 0, off_theta = 0, off_spec = 0,
         off_repair = 0, off_rcand = 0, total = 0;
};

// Room for the candidates a row collects over `keys` keys (four equal
// segments, one per epilogue warp of the row).  With a running threshold at
// the k-th value seen so far, a key enters with probability about
// min(1, k / position), so about k * (1 + ln(keys / k)) keys enter in all;
// half again of that covers the histogram's bin slack.  A segment that fills
// up is compacted to its exact top-k in the kernel, so it must hold k plus
// the 32 keys per tile its warp may append before the next vote; a segment
// never needs more than its whole share of the keys (32 per tile).
int candidate_capacity(int topk, int64_t keys) {
  const double ratio = std::max(1.0, static_cast<double>(keys) / topk);
  const double expect = topk * (1.0 + std::log(ratio));
  const int64_t cap = static_cast<int64_t>(1.5 * expect) + 2 * kBlockKeys;
  const int64_t floor_cap = 4 * (static_cast<int64_t>(topk) + kMaxVoteTiles * 32);
  const int64_t all_keys = round_up(std::max<int64_t>(keys, 1), kBlockKeys);
  return static_cast<int>(round_up(std::min(all_keys, std::max<int64_t>(cap, floor_cap)), kBlockKeys));
}

void finish_plan(Plan& pl, int64_t groups, int sms, int topk, int64_t axis) {
  pl.groups = static_cast<int>(groups);
  pl.axis = axis;
  pl.num_units = static_cast<int>(groups * pl.n_chunks);
  pl.grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(pl.num_units, sms)));
  pl.cap = candidate_capacity(topk, std::min<int64_t>(axis, pl.chunk_keys));
  size_t off = kStatusBytes;
  pl.off_cand = off;
  // two row-state slots per CTA (a unit is selected while the next one streams)
  off += round_up(static_cast<int64_t>(2) * sms * pl.R * pl.cap * 8, 256);
  pl.off_scratch = off;  // staging for a rare in-kernel compaction, per epilogue warp
  off += round_up(static_cast<int64_t>(sms) * kMaxEpiWarps * topk * 8, 256);
  pl.off_repair = off;   // per group: listed flag, then the list
  off += round_up(groups * 2 * 4, 256);
  pl.rgrid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>({groups, sms, kRepairMaxGrid})));
  if (pl.n_chunks > 1) {
    pl.off_part = off;
    off += round_up(static_cast<int64_t>(pl.num_units) * pl.R * topk * 8, 256);
    pl.off_cnt = off;
    off += round_up(static_cast<int64_t>(pl.num_units) * pl.R * 4, 256);
    pl.off_theta = off;  // per-row shared threshold, then per-row largest estimate
    off += round_up(groups * pl.R * 4, 256);
    pl.off_spec = off;
    off += round_up(groups * pl.R * 4, 256);
    // a repair recomputes whole rows: candidate room for the whole key axis
    pl.rcap = candidate_capacity(topk, axis);
    pl.off_rcand = off;
    off += round_up(static_cast<int64_t>(2) * pl.rgrid * pl.R * pl.rcap * 8, 256);
  } else {
    pl.rcap = pl.cap;
    pl.off_rcand = pl.off_cand;
  }
  pl.total = off;
}

// The fused top-k on a prepared plan: wires the workspace into `p` (whose
// inputs, tensor maps and outputs are set), clears the per-call words, and
// launches the indexer (and the merge when the key axis is split), then the
// repair launch, which recomputes, exactly and whole, any row block or
// request whose estimated threshold the checks rejected (it ends at once
// when none was listed).
int run_fused_topk(const Plan& pl, IndexerParams& p, uint8_t* wsb, bool paged, int64_t rows, cudaStream_t st) {
  const int topk = p.topk;
  p.n_chunks = pl.n_chunks;
  p.chunk_keys = pl.chunk_keys;
  p.tail_chunks = pl.tail_chunks;
  p.tail_keys = pl.tail_keys;
  p.num_units = pl.num_units;
  p.status = reinterpret_cast<int*>(wsb);
  p.cand = reinterpret_cast<uint2*>(wsb + pl.off_cand);
  p.cand_cap = pl.cap;
  p.scratch = reinterpret_cast<uint2*>(wsb + pl.off_scratch);
  p.repair_flag = reinterpret_cast<int*>(wsb + pl.off_repair);
  p.repair_list = p.repair_flag + pl.groups;
  p.speculate = 1;
  p.repair_mode = 0;
  p.wait_limit_ns = g_wait_limit_ns;
  p.debug_withhold_first_tile = g_debug_withhold;
  cudaError_t e = cudaMemsetAsync(p.repair_flag, 0, static_cast<size_t>(pl.groups) * 4, st);
  if (e != cudaSuccess) return cuda_fail(e, "repair flags reset");
  if (pl.n_chunks > 1) {
    p.part = reinterpret_cast<uint2*>(wsb + pl.off_part);
    p.part_cnt = reinterpret_cast<int*>(wsb + pl.off_cnt);
    p.row_theta = reinterpret_cast<uint32_t*>(wsb + pl.off_theta);
    p.row_spec = reinterpret_cast<uint32_t*>(wsb + pl.off_spec);
    e = cudaMemsetAsync(p.row_theta, 0, pl.off_spec + round_up(static_cast<int64_t>(pl.groups) * pl.R * 4, 256) -
                                            pl.off_theta, st);
    if (e != cudaSuccess) return cuda_fail(e, "threshold reset");
  }
  p.rows_per_unit = pl.rows_per_unit;
  e = paged ? launch_indexer_paged_topk(p, pl.R, pl.H, pl.grid, st) : launch_indexer_prefill_topk(p, pl.H, pl.grid, st);
  if (e != cudaSuccess) return cuda_fail(e, "indexer launch");
  if (pl.n_chunks > 1) {
    MergeParams mp{p.part, p.part_cnt, static_cast<int>(rows), pl.rows_per_unit, pl.R, pl.n_chunks, topk,
                   p.out_idx, p.out_vals, p.row_spec, p.status, p.repair_flag, p.repair_list,
                   p.out_slots ? p.block_table : nullptr, p.max_blocks, p.num_pages};
    e = launch_merge(mp, st);
    if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  }
  IndexerParams r = p;  // the repair: listed groups, whole rows, exact thresholds, direct output
  r.repair_mode = 1;
  r.speculate = 0;
  r.n_chunks = 1;
  r.chunk_keys = static_cast<int>(round_up(std::max<int64_t>(pl.axis, 1), kBlockKeys));
  r.tail_chunks = 0;
  r.num_units = pl.groups;
  r.cand = reinterpret_cast<uint2*>(wsb + pl.off_rcand);
  r.cand_cap = pl.rcap;
  r.part = nullptr;
  r.part_cnt = nullptr;
  r.row_theta = nullptr;
  r.row_spec = nullptr;
  r.debug_withhold_first_tile = 0;
  e = paged ? launch_indexer_paged_topk(r, pl.R, pl.H, pl.rgrid, st) : launch_indexer_prefill_topk(r, pl.H, pl.rgrid, st);
  if (e != cudaSuccess) return cuda_fail(e, "repair launch");
  return ok();
}

// Row blocks of kPrefillRows rows (4 with 64 heads); when they cannot fill
// the GPU, the key axis is cut into chunks so that about two units land on
// every SM.
Plan plan_prefill(int64_t m, int64_t n, int topk, int sms, int H = kHeads) {
  Plan pl;
  pl.H = H;
  pl.R = H == 64 ? 4 : kPrefillRows;
  pl.rows_per_unit = pl.R;
  const int64_t groups = ceil_div(m, pl.R);
  const int64_t axis = std::max<int64_t>(n, 1);
  pl.chunk_keys = static_cast<int>(round_up(axis, kBlockKeys));
  pl.n_chunks = 1;
  if (groups < sms) {
    const int64_t want = ceil_div(2 * static_cast<int64_t>(sms), groups);
    const int64_t ck = round_up(ceil_div(axis, want), kBlockKeys);
    pl.chunk_keys = static_cast<int>(ck);
    pl.n_chunks = static_cast<int>(ceil_div(axis, ck));
  }
  finish_plan(pl, groups, sms, topk, axis);
  return pl;
}

// One unit per (request, key chunk); chunks of the longest context sized so
// that about kPagedUnitsPerSm units land on every SM (context lengths differ,
// so many chunks are short or empty).  Small units even out the end of the
// schedule; a unit's rows start from the thresholds their earlier chunks
// raised, so later chunks pass few candidates.
constexpr int kPagedUnitsPerSm = 8;
constexpr int kPagedTailChunks = 4;
Plan plan_paged(int64_t B, int R, int max_blocks, int topk, int sms, int H = kHeads) {
  Plan pl;
  pl.H = H;
  pl.R = (H == 64 || R <= 4) ? 4 : 8;  // the kernel's rows; a request's R rows use the first R
  pl.rows_per_unit = R;
  const int64_t axis = static_cast<int64_t>(max_blocks) * kPageSize;
  pl.chunk_keys = static_cast<int>(round_up(axis, kBlockKeys));
  pl.n_chunks = 1;
  if (B < kPagedUnitsPerSm * static_cast<int64_t>(sms)) {
    const int64_t want = ceil_div(kPagedUnitsPerSm * static_cast<int64_t>(sms), B);
    const int64_t ck = round_up(ceil_div(axis, want), kBlockKeys);
    pl.chunk_keys = static_cast<int>(ck);
    pl.n_chunks = static_cast<int>(ceil_div(axis, ck));
    // the last kPagedTailChunks chunks each become two of half the size
    const int m = std::min<int>(kPagedTailChunks, pl.n_chunks / 4);
    const int64_t half = round_up(ceil_div(ck, 2), kBlockKeys);
    if (m > 0 && half < ck) {
      pl.tail_chunks = 2 * m;
      pl.tail_keys = static_cast<int>(half);
      pl.n_chunks += m;
    }
  }
  finish_plan(pl, B, sms, topk, axis);
  return pl;
}

int check_shape(int H, int D) {
  if ((H != 32 && H != 64) || D != kDim)
    return fail(FP8IDX_EUNSUPPORTED, "only H=32 or 64 and D=128 are supported (got H=%d, D=%d)", H, D);
  return FP8IDX_OK;
}

// Rows per request of the paged form: 1 to 8 (MTP verify widths), at most 4 with 64 heads.
int check_rows_per_request(int R, int H) {
  if (R < 1 || R > 8 || (H == 64 && R > 4))
    return fail(FP8IDX_EUNSUPPORTED, "rows per request must be in [1, %d] with H=%d (got %d)", H == 64 ? 4 : 8, H, R);
  return FP8IDX_OK;
}

int check_topk(int topk) {
  if (topk < 1 || topk > kMaxTopK)
    return fail(FP8IDX_EINVAL, "topk must be in [1, %d] (got %d)", kMaxTopK, topk);
  return FP8IDX_OK;
}

// Device address of the no-alloc scratch array on the current device,
// looked up once per device index (under a lock) and kept for the process.
int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "current device");
  constexpr int kMaxDevices = 64;
  if (dev < 0 || dev >= kMaxDevices) return fail(FP8IDX_EUNSUPPORTED, "device index %d out of range", dev);
  static std::mutex mu;
  static void* scratch_of[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (!scratch_of[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "no-alloc scratch address");
    scratch_of[dev] = ptr;
  }
  *out = scratch_of[dev];
  return FP8IDX_OK;
}

// A workspace argument of the diagnostics calls: NULL names the logits
// status block, FP8IDX_NOALLOC_WS the no-alloc scratch array.
int resolve_status_source(const void* ws, const void** src) {
  if (ws == FP8IDX_NOALLOC_WS) {
    void* p = nullptr;
    const int rc = noalloc_scratch(&p);
    if (rc != FP8IDX_OK) return rc;
    *src = p;
  } else if (!ws) {
    void* sym = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&sym, g_logits_status);
    if (e != cudaSuccess) return cuda_fail(e, "status symbol");
    *src = sym;
  } else {
    *src = ws;
  }
  return FP8IDX_OK;
}

#define FP8IDX_TRY(x)          \
  do {                         \
    int _rc = (x);             \
    if (_rc != FP8IDX_OK) return _rc; \
  } while (0)

int check_prefill_inputs(const uint8_t* q, const uint8_t* k, const float* s, const float* w,
                         const int32_t* ks, const int32_t* ke, int64_t m, int64_t n) {
  if (m < 0 || n < 0) return fail(FP8IDX_EINVAL, "negative size (m=%lld, n=%lld)", (long long)m, (long long)n);
  if (m > (int64_t(1) << 25)) return fail(FP8IDX_EINVAL, "m=%lld is too large", (long long)m);
  if (n >= (int64_t(1) << 31) - kBlockKeys) return fail(FP8IDX_EINVAL, "n=%lld is too large", (long long)n);
  if (m == 0) return FP8IDX_OK;
  if (!q || !w || !ks || !ke) return fail(FP8IDX_EINVAL, "null q, w, ks or ke");
  if (n > 0 && (!k || !s)) return fail(FP8IDX_EINVAL, "null k or s");
  if (!aligned(q, 16) || (k && !aligned(k, 16)))
    return fail(FP8IDX_EINVAL, "q and k must be 16-byte aligned");
  if (!aligned(s, 4) || !aligned(w, 4) || !aligned(ks, 4) || !aligned(ke, 4))
    return fail(FP8IDX_EINVAL, "s, w, ks and ke must be 4-byte aligned");
  return FP8IDX_OK;
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

const char* fp8idx_last_error(void) { return t_last_error.c_str(); }

int fp8idx_num_sms(void) { return device_sms(); }

void fp8idx_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns = ns; }

void fp8idx_debug_withhold_first_tile(int on) { g_debug_withhold = on ? 1 : 0; }

int fp8idx_mqa_logits(const uint8_t* q, const uint8_t* k, const float* s, const float* w,
                      const int32_t* ks, const int32_t* ke, int64_t m, int64_t n, int H, int D,
                      float* logits, int64_t ld_logits, void* stream) {
  FP8IDX_TRY(check_shape(H, D));
  FP8IDX_TRY(check_prefill_inputs(q, k, s, w, ks, ke, m, n));
  if (m == 0 || n == 0) return ok();
  if (!logits || !aligned(logits, 4)) return fail(FP8IDX_EINVAL, "logits must be non-null and 4-byte aligned");
  if (ld_logits < n) return fail(FP8IDX_EINVAL, "ld_logits (%lld) < n (%lld)", (long long)ld_logits, (long long)n);
  const int sms = device_sms();
  if (sms <= 0) return fail(FP8IDX_ECUDA, "no CUDA device");
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // One unit per 8-row block; small m splits the key axis (each unit writes
  // its own column range, so no merge is needed).
  Plan pl = plan_prefill(m, n, 1, sms, H);
  IndexerParams p;
  memset(&p, 0, sizeof(p));
  FP8IDX_TRY(make_rows128_map(&p.tmap_q, q, m * H, pl.R * H));
  FP8IDX_TRY(make_rows128_map(&p.tmap_k, k, n, kBlockKeys));
  p.s = s;
  p.w = w;
  p.ks = ks;
  p.ke = ke;
  p.n = n;
  p.m = static_cast<int>(m);
  p.rows_per_unit = pl.rows_per_unit;
  p.topk = 1;
  p.n_chunks = pl.n_chunks;
  p.chunk_keys = pl.chunk_keys;
  p.num_units = pl.num_units;
  p.logits = logits;
  p.ld_logits = ld_logits;
  int* status = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_logits_status);
  if (e != cudaSuccess) return cuda_fail(e, "status symbol");
  e = cudaMemsetAsync(status, 0, kStatusBytes, st);
  if (e != cudaSuccess) return cuda_fail(e, "status reset");
  p.status = status;
  p.wait_limit_ns = g_wait_limit_ns;
  p.debug_withhold_first_tile = g_debug_withhold;
  e = launch_indexer_prefill_logits(p, H, pl.grid, st);
  if (e != cudaSuccess) return cuda_fail(e, "mqa_logits launch");
  return ok();
}

int fp8idx_topk_rows(const float* logits, int64_t ld, const int32_t* ks, const int32_t* ke,
                     int64_t m, int64_t n, int topk, int32_t* out, void* stream) {
  FP8IDX_TRY(check_topk(topk));
  if (m < 0 || n < 0) return fail(FP8IDX_EINVAL, "negative size");
  if (m > INT32_MAX || n >= (int64_t(1) << 31)) return fail(FP8IDX_EINVAL, "size too large");
  if (m == 0) return ok();
  if (!ks || !ke || !out || (n > 0 && !logits)) return fail(FP8IDX_EINVAL, "null pointer");
  if (!aligned(logits, 4) || !aligned(ks, 4) || !aligned(ke, 4) || !aligned(out, 4))
    return fail(FP8IDX_EINVAL, "pointers must be 4-byte aligned");
  if (ld < n) return fail(FP8IDX_EINVAL, "ld (%lld) < n (%lld)", (long long)ld, (long long)n);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  TopkRowsParams p{logits, ld, ks, ke, n, static_cast<int>(m), topk, out};
  cudaError_t e = launch_topk_rows(p, st);
  if (e != cudaSuccess) return cuda_fail(e, "topk_rows launch");
  return ok();
}

size_t fp8idx_mqa_logits_topk_workspace(int64_t m, int64_t n, int H, int D, int topk) {
  if ((H != 32 && H != 64) || D != kDim || topk < 1 || topk > kMaxTopK || m < 0 || n < 0) return 0;
  const int sms = device_sms();
  if (sms <= 0) return 0;
  return plan_prefill(std::max<int64_t>(m, 1), n, topk, sms, H).total;
}

int fp8idx_mqa_logits_topk(const uint8_t* q, const uint8_t* k, const float* s, const float* w,
                           const int32_t* ks, const int32_t* ke, int64_t m, int64_t n, int H,
                           int D, int topk, int32_t* out_idx, float* out_vals, void* ws,
                           size_t ws_bytes, void* stream) {
  FP8IDX_TRY(check_shape(H, D));
  FP8IDX_TRY(check_topk(topk));
  FP8IDX_TRY(check_prefill_inputs(q, k, s, w, ks, ke, m, n));
  if (m == 0) return ok();
  if (!out_idx || !aligned(out_idx, 4) || !aligned(out_vals, 4))
    return fail(FP8IDX_EINVAL, "out_idx must be non-null; outputs 4-byte aligned");
  const int sms = device_sms();
  if (sms <= 0) return fail(FP8IDX_ECUDA, "no CUDA device");
  Plan pl = plan_prefill(m, n, topk, sms, H);
  if (!ws || !aligned(ws, 256)) return fail(FP8IDX_EINVAL, "workspace must be non-null and 256-byte aligned");
  if (ws_bytes < pl.total)
    return fail(FP8IDX_EWORKSPACE, "workspace too small (%zu < %zu bytes)", ws_bytes, pl.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  cudaError_t e = cudaMemsetAsync(ws, 0, kStatusBytes, st);
  if (e != cudaSuccess) return cuda_fail(e, "status reset");
  if (n == 0) {
    e = launch_fill_empty(out_idx, out_vals, static_cast<int>(m), topk, st);
    if (e != cudaSuccess) return cuda_fail(e, "fill launch");
    return ok();
  }
  IndexerParams p;
  memset(&p, 0, sizeof(p));
  FP8IDX_TRY(make_rows128_map(&p.tmap_q, q, m * H, pl.R * H));
  FP8IDX_TRY(make_rows128_map(&p.tmap_k, k, n, kBlockKeys));
  p.s = s;
  p.w = w;
  p.ks = ks;
  p.ke = ke;
  p.n = n;
  p.m = static_cast<int>(m);
  p.topk = topk;
  p.out_idx = out_idx;
  p.out_vals = out_vals;
  return run_fused_topk(pl, p, wsb, false, m, st);
}

size_t fp8idx_paged_mqa_logits_topk_workspace(int64_t B, int R, int max_blocks, int H, int D,
                                              int topk) {
  if ((H != 32 && H != 64) || D != kDim || topk < 1 || topk > kMaxTopK || B < 0 || max_blocks < 1 || R < 1 ||
      R > 8 || (H == 64 && R > 4))
    return 0;
  const int sms = device_sms();
  if (sms <= 0) return 0;
  return plan_paged(std::max<int64_t>(B, 1), R, max_blocks, topk, sms, H).total;
}

// The paged call; out_slots: write physical KV slots instead of positions.
static int paged_topk(const uint8_t* q, const uint8_t* k_pages, const float* s_pages, const float* w,
               const int32_t* block_table, const int32_t* seq_lens, int64_t B, int R, int max_blocks,
               int64_t num_pages, int page_size, int H, int D, int topk, int32_t* out_idx, float* out_vals,
               void* ws, size_t ws_bytes, void* stream, bool out_slots) {
  FP8IDX_TRY(check_shape(H, D));
  FP8IDX_TRY(check_topk(topk));
  if (page_size != kPageSize) return fail(FP8IDX_EUNSUPPORTED, "page_size must be 64 (got %d)", page_size);
  FP8IDX_TRY(check_rows_per_request(R, H));
  if (B < 0 || num_pages < 0 || max_blocks < 1) return fail(FP8IDX_EINVAL, "bad sizes");
  if (B * R > (int64_t(1) << 25)) return fail(FP8IDX_EINVAL, "too many rows");
  if (static_cast<int64_t>(max_blocks) * kPageSize >= (int64_t(1) << 31) - kBlockKeys ||
      num_pages * kPageSize >= (int64_t(1) << 31))
    return fail(FP8IDX_EINVAL, "paged key space too large");
  if (B == 0) return ok();
  if (!q || !w || !block_table || !seq_lens || !out_idx)
    return fail(FP8IDX_EINVAL, "null q, w, block_table, seq_lens or out_idx");
  if (num_pages > 0 && (!k_pages || !s_pages)) return fail(FP8IDX_EINVAL, "null k_pages or s_pages");
  if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(s_pages, 16))
    return fail(FP8IDX_EINVAL, "q, k_pages and s_pages must be 16-byte aligned");
  if (!aligned(s_pages, 4) || !aligned(w, 4) || !aligned(block_table, 4) || !aligned(seq_lens, 4) ||
      !aligned(out_idx, 4) || !aligned(out_vals, 4))
    return fail(FP8IDX_EINVAL, "pointers must be 4-byte aligned");
  const int sms = device_sms();
  if (sms <= 0) return fail(FP8IDX_ECUDA, "no CUDA device");
  Plan pl = plan_paged(B, R, max_blocks, topk, sms, H);
  if (!ws || !aligned(ws, 256)) return fail(FP8IDX_EINVAL, "workspace must be non-null and 256-byte aligned");
  if (ws_bytes < pl.total)
    return fail(FP8IDX_EWORKSPACE, "workspace too small (%zu < %zu bytes)", ws_bytes, pl.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  cudaError_t e = cudaMemsetAsync(ws, 0, kStatusBytes, st);
  if (e != cudaSuccess) return cuda_fail(e, "status reset");
  if (num_pages == 0) {
    e = launch_fill_empty(out_idx, out_vals, static_cast<int>(B * R), topk, st);
    if (e != cudaSuccess) return cuda_fail(e, "fill launch");
    return ok();
  }
  IndexerParams p;
  memset(&p, 0, sizeof(p));
  FP8IDX_TRY(make_rows128_map(&p.tmap_q, q, B * R * H, pl.R * H));
  FP8IDX_TRY(make_rows128_map(&p.tmap_k, k_pages, num_pages * kPageSize, kPageSize));
  p.s = s_pages;
  p.w = w;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.m = static_cast<int>(B * R);
  p.max_blocks = max_blocks;
  p.num_pages = static_cast<int>(num_pages);
  p.topk = topk;
  p.out_idx = out_idx;
  p.out_vals = out_vals;
  p.out_slots = out_slots ? 1 : 0;
  return run_fused_topk(pl, p, wsb, true, B * R, st);
}

int fp8idx_paged_mqa_logits_topk(const uint8_t* q, const uint8_t* k_pages, const float* s_pages,
                                 const float* w, const int32_t* block_table,
                                 const int32_t* seq_lens, int64_t B, int R, int max_blocks,
                                 int64_t num_pages, int page_size, int H, int D, int topk,
                                 int32_t* out_idx, float* out_vals, void* ws, size_t ws_bytes,
                                 void* stream) {
  return paged_topk(q, k_pages, s_pages, w, block_table, seq_lens, B, R, max_blocks, num_pages, page_size, H, D,
                    topk, out_idx, out_vals, ws, ws_bytes, stream, false);
}

int fp8idx_paged_mqa_logits_topk_slots(const uint8_t* q, const uint8_t* k_pages, const float* s_pages,
                                       const float* w, const int32_t* block_table,
                                       const int32_t* seq_lens, int64_t B, int R, int max_blocks,
                                       int64_t num_pages, int page_size, int H, int D, int topk,
                                       int32_t* out_slots, float* out_vals, void* ws, size_t ws_bytes,
                                       void* stream) {
  return paged_topk(q, k_pages, s_pages, w, block_table, seq_lens, B, R, max_blocks, num_pages, page_size, H, D,
                    topk, out_slots, out_vals, ws, ws_bytes, stream, true);
}

// Allocation-free form of fp8idx_mqa_logits_topk for callers that cannot
// allocate device memory at call time: code running while a CUDA graph is
// captured or replayed by a framework that owns every allocation, inference
// runtimes with a fixed memory budget planned at start-up, or plugins whose
// host forbids cudaMalloc outside initialisation.  The workspace is the fixed
// array above instead of a caller buffer.  The first call on each device
// looks up the array's device address (once, under a lock); make that first
// call before capturing a stream.  The grid shrinks until the workspace plan
// fits in the array, so large problems run on fewer SMs (slower, same
// result); a problem that does not fit even on one SM is rejected with
// FP8IDX_EWORKSPACE.  Every call reuses the same array, which keeps the last
// call's contents; the status block is cleared on entry.  Two calls that may
// run at the same time on the GPU (different streams, or different host
// threads) race on the array and must be serialised by the caller.
int fp8idx_mqa_logits_topk_noalloc(const uint8_t* q, const uint8_t* k, const float* s,
                                   const float* w, const int32_t* ks, const int32_t* ke, int64_t m,
                                   int64_t n, int H, int D, int topk, int32_t* out_idx,
                                   float* out_vals, void* stream) {
  FP8IDX_TRY(check_shape(H, D));
  FP8IDX_TRY(check_topk(topk));
  FP8IDX_TRY(check_prefill_inputs(q, k, s, w, ks, ke, m, n));
  if (m == 0) return ok();
  if (!out_idx || !aligned(out_idx, 4) || !aligned(out_vals, 4))
    return fail(FP8IDX_EINVAL, "out_idx must be non-null; outputs 4-byte aligned");
  void* scratch = nullptr;
  FP8IDX_TRY(noalloc_scratch(&scratch));
  cudaError_t e;
  int sms = device_sms();
  if (sms <= 0) return fail(FP8IDX_ECUDA, "no CUDA device");
  Plan pl;
  int g = sms;
  for (; g >= 1; --g) {
    pl = plan_prefill(m, n, topk, g, H);
    if (pl.total <= kNoAllocScratchBytes) break;
  }
  if (g < 1)
    return fail(FP8IDX_EWORKSPACE, "problem needs more than the %zu-byte fixed scratch", kNoAllocScratchBytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(scratch);
  e = cudaMemsetAsync(wsb, 0, kStatusBytes, st);
  if (e != cudaSuccess) return cuda_fail(e, "status reset");
  if (n == 0) {
    e = launch_fill_empty(out_idx, out_vals, static_cast<int>(m), topk, st);
    if (e != cudaSuccess) return cuda_fail(e, "fill launch");
    return ok();
  }
  IndexerParams p;
  memset(&p, 0, sizeof(p));
  FP8IDX_TRY(make_rows128_map(&p.tmap_q, q, m * H, pl.R * H));
  FP8IDX_TRY(make_rows128_map(&p.tmap_k, k, n, kBlockKeys));
  p.s = s;
  p.w = w;
  p.ks = ks;
  p.ke = ke;
  p.n = n;
  p.m = static_cast<int>(m);
  p.topk = topk;
  p.out_idx = out_idx;
  p.out_vals = out_vals;
  const int rc = run_fused_topk(pl, p, wsb, false, m, st);
  if (rc != FP8IDX_OK) return rc;
  return ok();
}

int fp8idx_read_device_stats(const void* ws, uint32_t* out, int count, void* stream) {
  if (!out || count < 1 || count > kStatusBytes / 4) return fail(FP8IDX_EINVAL, "bad arguments");
  const void* src = nullptr;
  FP8IDX_TRY(resolve_status_source(ws, &src));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(out, src, sizeof(uint32_t) * count, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "stats read");
  return ok();
}

int fp8idx_act_quant_store(const uint16_t* x, int64_t T, int D, const int64_t* slot, int64_t num_slots,
                           uint8_t* k_pool, float* s_pool, void* stream) {
  if (D != kDim) return fail(FP8IDX_EUNSUPPORTED, "only D=128 is supported (got D=%d)", D);
  if (T < 0 || num_slots < 0) return fail(FP8IDX_EINVAL, "negative size");
  if (T > (int64_t(1) << 34)) return fail(FP8IDX_EINVAL, "T=%lld is too large", (long long)T);
  if (T == 0) return ok();
  if (!x || !slot || !k_pool || !s_pool) return fail(FP8IDX_EINVAL, "null pointer");
  if (!aligned(x, 8) || !aligned(slot, 8) || !aligned(k_pool, 4) || !aligned(s_pool, 4))
    return fail(FP8IDX_EINVAL, "x and slot must be 8-byte aligned, k_pool and s_pool 4-byte aligned");
  cudaError_t e = launch_act_quant_store(x, T, slot, num_slots, k_pool, s_pool, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "act_quant_store launch");
  return ok();
}

int fp8idx_prepare_ragged(const int32_t* seq_len, const int32_t* q_len, const int32_t* req_idx, int B,
                          const int32_t* req_to_token, int64_t table_rows, int64_t ld_table, int32_t* ks,
                          int32_t* ke, int32_t* row_table, int64_t q_cap, int32_t* ragged, int64_t ragged_cap,
                          void* stream) {
  if (B < 0 || B > kMaxPrepBatch) return fail(FP8IDX_EINVAL, "B must be in [0, %d] (got %d)", kMaxPrepBatch, B);
  if (q_cap < 0 || ragged_cap < 0 || table_rows < 0 || ld_table < 0)
    return fail(FP8IDX_EINVAL, "negative size");
  if (q_cap > INT32_MAX || ragged_cap > INT32_MAX)
    return fail(FP8IDX_EINVAL, "capacities must stay below 2^31 (int32 key positions)");
  if (q_cap == 0 && (!ragged || ragged_cap == 0)) return ok();
  if ((B > 0 && (!seq_len || !q_len || !req_idx)) || (q_cap > 0 && (!ks || !ke)))
    return fail(FP8IDX_EINVAL, "null seq_len, q_len, req_idx, ks or ke");
  if (ragged && ragged_cap > 0 && table_rows > 0 && !req_to_token) return fail(FP8IDX_EINVAL, "null req_to_token");
  if (!aligned(seq_len, 4) || !aligned(q_len, 4) || !aligned(req_idx, 4) || !aligned(req_to_token, 4) ||
      !aligned(ks, 4) || !aligned(ke, 4) || !aligned(row_table, 4) || !aligned(ragged, 4))
    return fail(FP8IDX_EINVAL, "pointers must be 4-byte aligned");
  const int sms = device_sms();
  if (sms <= 0) return fail(FP8IDX_ECUDA, "no CUDA device");
  cudaError_t e = launch_prepare_ragged(seq_len, q_len, req_idx, B, req_to_token, table_rows, ld_table, ks, ke,
                                        row_table, q_cap, ragged, ragged ? ragged_cap : 0, sms,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prepare_ragged launch");
  return ok();
}

int fp8idx_topk_transform(const int32_t* idx, int64_t rows, int topk, const int32_t* row_base,
                          const int32_t* row_table, int rows_per_table_row, const int32_t* page_table,
                          int64_t table_rows, int64_t ld_table, int page_size, int32_t* out, void* stream) {
  if (rows < 0 || topk < 0 || table_rows < 0 || ld_table < 0) return fail(FP8IDX_EINVAL, "negative size");
  if (page_size < 1) return fail(FP8IDX_EINVAL, "page_size must be >= 1 (got %d)", page_size);
  if (!row_table && rows_per_table_row < 1)
    return fail(FP8IDX_EINVAL, "rows_per_table_row must be >= 1 without row_table");
  if (rows == 0 || topk == 0) return ok();
  if (!idx || !out || (table_rows > 0 && ld_table > 0 && !page_table))
    return fail(FP8IDX_EINVAL, "null idx, out or page_table");
  if (!aligned(idx, 4) || !aligned(out, 4) || !aligned(row_base, 4) || !aligned(row_table, 4) ||
      !aligned(page_table, 4))
    return fail(FP8IDX_EINVAL, "pointers must be 4-byte aligned");
  const int sms = device_sms();
  if (sms <= 0) return fail(FP8IDX_ECUDA, "no CUDA device");
  cudaError_t e = launch_topk_transform(idx, rows, topk, row_base, row_table, rows_per_table_row, page_table,
                                        table_rows, ld_table, page_size, out, sms,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "topk_transform launch");
  return ok();
}

int fp8idx_read_device_status(const void* ws, int* status_out, void* stream) {
  if (!status_out) return fail(FP8IDX_EINVAL, "null status_out");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const void* src = nullptr;
  FP8IDX_TRY(resolve_status_source(ws, &src));
  int v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, src, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  *status_out = v;
  return ok();
}

}  // extern "C"
