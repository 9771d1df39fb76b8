// index_prep.cu -- index preparation and the top-k transform (sm_100a).
//
// The step before and the step after the indexer, as the "reuse inference
// metadata and streamline FP8 prefill" page (LightLLM pull request: its
// description table, the `gen_nsa_ks_ke` walkthrough and the review's
// expected ragged buffer) and the `page_table_size_1` argument of
// `fast_topk_transform_fused` ("bench_mqa_logits_chunking.py" page) define
// them:
//
//   prepare:   requests laid out back to back in one ragged key space
//              (request b owns [koff_b, koff_b + seq_len[b]), its q_len[b]
//              query rows are rows [qoff_b, qoff_b + q_len[b]));
//              row t of request b: ks = koff_b,
//              ke = koff_b + clamp(seq_len[b] - q_len[b] + t + 1, 0, seq_len[b]);
//              optionally ragged[koff_b + p] = req_to_token[req_idx[b], p].
//   transform: a selected position idx (-1 = none) of row i becomes the
//              physical slot table[trow, p / P] * P + p % P, p = idx - base_i,
//              P the page size (1: a token-granular table).
//
// Both are plain integer streams.  prepare: every CTA scans the B lengths in
// shared memory, then the grid covers the rows and the ragged positions; a
// warp walks 32 consecutive positions per step and finds the request of each
// from the previous one (requests are long, so the walk rarely moves), so
// reads of a table row and writes of the ragged buffer are both coalesced.
#include <algorithm>
#include <cstdint>

#include <cuda_runtime.h>

namespace fp8idx {

namespace {

constexpr int kPrepThreads = 512;

// Exclusive prefix sums of a[0..B) into off[0..B] by one CTA (the caller bounds B
// so that 2 (B + 1) int64 offsets fit in shared memory).
__device__ void block_exclusive_scan(const int32_t* __restrict__ a, int B, int64_t* off, int64_t* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t carry = 0;
  for (int base = 0; base < B; base += kPrepThreads) {
    const int i = base + threadIdx.x;
    const int64_t v = i < B ? static_cast<int64_t>(max(__ldg(a + i), 0)) : 0;
    int64_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int64_t before = carry;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    if (i < B) off[i] = before + incl - v;
    int64_t chunk = 0;
    for (int w = 0; w < kPrepThreads / 32; ++w) chunk += warp_tot[w];
    __syncthreads();
    carry += chunk;
  }
  if (threadIdx.x == 0) off[B] = carry;
  __syncthreads();
}

// Largest b in [0, B) with off[b] <= x (off non-decreasing, off[0] = 0 <= x < off[B]).
__device__ __forceinline__ int owner_of(const int64_t* off, int B, int64_t x) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(kPrepThreads)
    prepare_kernel(const int32_t* __restrict__ seq_len, const int32_t* __restrict__ q_len,
                   const int32_t* __restrict__ req_idx, int B, const int32_t* __restrict__ table,
                   int64_t table_rows, int64_t ld, int32_t* __restrict__ ks, int32_t* __restrict__ ke,
                   int32_t* __restrict__ row_table, int64_t q_cap, int32_t* __restrict__ ragged,
                   int64_t ragged_cap) {
  extern __shared__ int64_t sh[];
  int64_t* koff = sh;              // [B + 1]
  int64_t* qoff = sh + (B + 1);    // [B + 1]
  __shared__ int64_t warp_tot[kPrepThreads / 32];
  block_exclusive_scan(seq_len, B, koff, warp_tot);
  block_exclusive_scan(q_len, B, qoff, warp_tot);
  const int64_t total_q = qoff[B], total_k = koff[B];
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kPrepThreads / 32);
  const int64_t gwarp = static_cast<int64_t>(blockIdx.x) * (kPrepThreads / 32) + (threadIdx.x >> 5);

  // ---- rows: each warp takes 32 consecutive rows per step
  for (int64_t x0 = gwarp * 32; x0 < q_cap; x0 += nwarps * 32) {
    const int64_t x = x0 + lane;
    if (x >= q_cap) break;
    int32_t s = 0, e = 0, tr = -1;
    if (x < total_q) {
      const int b = owner_of(qoff, B, x);
      const int64_t L = max(__ldg(seq_len + b), 0), Q = max(__ldg(q_len + b), 0);
      const int64_t t = x - qoff[b];
      const int64_t len = min(max(L - Q + t + 1, static_cast<int64_t>(0)), L);
      s = static_cast<int32_t>(koff[b]);
      e = static_cast<int32_t>(koff[b] + len);
      tr = __ldg(req_idx + b);
    }
    ks[x] = s;
    ke[x] = e;
    if (row_table) row_table[x] = tr;
  }

  // ---- ragged copy: each warp takes 32 * 8 consecutive positions per step
  if (!ragged) return;
  const int64_t nk = min(total_k, ragged_cap);
  constexpr int kPer = 8;
  for (int64_t x0 = gwarp * 32 * kPer; x0 < nk; x0 += nwarps * 32 * kPer) {
    int64_t x = x0 + lane;
    if (x >= nk) break;
    int b = owner_of(koff, B, x);
    int64_t next = koff[b + 1];
#pragma unroll
    for (int j = 0; j < kPer; ++j, x += 32) {
      if (x >= nk) break;
      while (x >= next) {  // the next request (rarely taken: requests are long)
        ++b;
        next = koff[b + 1];
      }
      const int64_t p = x - koff[b];
      const int64_t trow = __ldg(req_idx + b);
      ragged[x] = (trow >= 0 && trow < table_rows && p < ld) ? __ldg(table + trow * ld + p) : -1;
    }
  }
}

// One CTA per (row, run of 256 positions): the row comes from the grid, not
// from a division per element.  (idx and out may be one buffer: each element
// is read, then written, by one thread.)
constexpr int kTransformThreads = 256;

__global__ void __launch_bounds__(kTransformThreads)
    transform_kernel(const int32_t* idx, int64_t rows, int topk, const int32_t* __restrict__ row_base,
                     const int32_t* __restrict__ row_table, int rows_per_table_row,
                     const int32_t* __restrict__ table, int64_t table_rows, int64_t ld, int page_size,
                     int page_shift, int32_t* out) {
  const int x = static_cast<int>(blockIdx.x) * kTransformThreads + static_cast<int>(threadIdx.x);
  if (x >= topk) return;
  for (int64_t i = blockIdx.y; i < rows; i += gridDim.y) {
    const int64_t e = i * topk + x;
    const int32_t v = idx[e];
    int32_t slot = -1;
    if (v >= 0) {
      const int64_t p = static_cast<int64_t>(v) - (row_base ? __ldg(row_base + i) : 0);
      const int64_t trow = row_table ? __ldg(row_table + i) : i / rows_per_table_row;
      if (p >= 0 && trow >= 0 && trow < table_rows) {
        // a power-of-two page size (1 or 64 in practice) takes a shift, and a
        // position below 2^31 (always, unless the row base is negative) 32-bit
        // arithmetic
        int64_t blk, off;
        if (page_shift >= 0) {
          blk = p >> page_shift;
          off = p & (page_size - 1);
        } else if (p < (static_cast<int64_t>(1) << 31)) {
          const int32_t b32 = static_cast<int32_t>(p) / page_size;
          blk = b32;
          off = p - static_cast<int64_t>(b32) * page_size;
        } else {
          blk = p / page_size;
          off = p % page_size;
        }
        if (blk < ld) {
          const int32_t page = __ldg(table + trow * ld + blk);
          if (page >= 0) slot = page * page_size + static_cast<int32_t>(off);
        }
      }
    }
    out[e] = slot;
  }
}

}  // namespace

cudaError_t launch_prepare_ragged(const int32_t* seq_len, const int32_t* q_len, const int32_t* req_idx, int B,
                                  const int32_t* table, int64_t table_rows, int64_t ld, int32_t* ks, int32_t* ke,
                                  int32_t* row_table, int64_t q_cap, int32_t* ragged, int64_t ragged_cap,
                                  int sms, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(2) * (B + 1) * sizeof(int64_t);
  cudaError_t e = cudaFuncSetAttribute(prepare_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // enough warps for the rows and for the ragged positions (8 per lane), at most 4 CTAs per SM
  const int64_t work = std::max<int64_t>((q_cap + 31) / 32, ragged ? (ragged_cap + 255) / 256 : 0);
  const int64_t want = (work + kPrepThreads / 32 - 1) / (kPrepThreads / 32);
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, 4 * static_cast<int64_t>(sms))));
  prepare_kernel<<<grid, kPrepThreads, smem, st>>>(seq_len, q_len, req_idx, B, table, table_rows, ld, ks, ke,
                                                   row_table, q_cap, ragged, ragged_cap);
  return cudaGetLastError();
}

cudaError_t launch_topk_transform(const int32_t* idx, int64_t rows, int topk, const int32_t* row_base,
                                  const int32_t* row_table, int rows_per_table_row, const int32_t* table,
                                  int64_t table_rows, int64_t ld, int page_size, int32_t* out, int sms,
                                  cudaStream_t st) {
  if (rows <= 0 || topk <= 0) return cudaSuccess;
  const unsigned gx = static_cast<unsigned>((topk + kTransformThreads - 1) / kTransformThreads);
  // rows over grid y (at most 65535), each CTA looping over the rows it is given
  const int64_t cap = std::max<int64_t>(1, std::min<int64_t>(65535, 16 * static_cast<int64_t>(sms)));
  const unsigned gy = static_cast<unsigned>(std::min<int64_t>(rows, cap));
  const int page_shift = (page_size & (page_size - 1)) == 0 ? __builtin_ctz(static_cast<unsigned>(page_size)) : -1;
  transform_kernel<<<dim3(gx, gy), kTransformThreads, 0, st>>>(idx, rows, topk, row_base, row_table,
                                                               rows_per_table_row, table, table_rows, ld,
                                                               page_size, page_shift, out);
  return cudaGetLastError();
}

}  // namespace fp8idx
