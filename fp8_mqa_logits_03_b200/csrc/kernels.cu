// kernels.cu -- the indexer kernels for sm_100a.
//
// What is computed (the indexer call of the "bench_mqa_logits_chunking.py"
// page: `fp8_mqa_logits` then `fast_topk_transform_fused`, H = 32, D = 128):
//   L[i,j] = s[j] * sum_h w[i,h] * ReLU(q[i,h,:] . k[j,:])  on ks[i] <= j < ke[i], else -inf
//   out[i] = the top-k j of row i (larger L first, lower j on ties), padded with -1.
//
// Design (one persistent CTA per SM, warp-specialised):
//   warp 0      TMA producer: the unit's q block [R rows x H heads x 128 B]
//               into one of two q slots, then 128-key tiles [128 x 128 B]
//               through a ring of shared-memory stages (paged keys: two
//               64-token pages a tile).
//   warp 1      MMA issuer: tcgen05.mma kind::f8f6f4 with M = 128 keys,
//               N = R*H (row, head) columns, K = 128 as 4 x K32 steps, fp32
//               accumulators in TMEM, double buffered (2 x N columns).
//   warps 2..3  select group (fused top-k): takes a finished unit's row
//               state (double buffered, so it overlaps the next unit) and
//               selects each row's exact top-k: keys above the boundary bin
//               go straight out, the boundary bin is resolved in shared memory.
//               Rows are claimed from a per-slot counter; once out of units,
//               the epilogue warps claim the last units' rows too.
//   warps 4..   epilogue, warpgroups of 4 (one warp per TMEM lane quadrant,
//               so one thread per key), each owning RW rows of the unit.  Each
//               thread reads its key's head dots per row from TMEM, applies
//               ReLU, the head weights and the key scale, then either writes
//               the logit (mqa_logits) or filters it against the row's
//               running threshold into its own segment of the row's
//               candidate buffer (fused top-k).  At votes every few tiles a
//               warp counts what it appended into the row's 512-bin
//               histogram and raises the threshold to a lower bound on (or a
//               checked estimate of) the row's k-th value.
// A unit is R query rows (a row block, or one request's rows in the paged
// form) times one chunk of keys, claimed from a device counter by the
// producer and passed on through a shared-memory queue.  With one chunk per
// unit the fused kernel writes the final top-k; with several, each unit
// writes its exact partial top-k and the merge kernel selects from the union.
#include <cfloat>
#include <climits>
#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace fp8idx {

// Key scales of a page that is not in the pool: zero (never written).
__device__ __align__(128) float g_zero_scales[kPageSize];

// Warp roles: warpgroup 0 holds the TMA producer (warp 0), the MMA issuer
// (warp 1) and the select group (warps 2-3); then EWG epilogue warpgroups of
// four warps, one per TMEM lane quadrant (warp % 4), each warpgroup owning RW
// rows of the unit.  More epilogue warpgroups with fewer rows each give every
// SM sub-partition more independent warps to hide the epilogue's latencies.
template <int R, bool PAGED, int H>
struct Cfg {
  static constexpr int N = R * H;              // MMA N: (row, head) columns
  static constexpr int RW = R == 8 ? 4 : 2;    // rows per epilogue warpgroup
  static constexpr int NC = RW * H / 32;       // 32-column TMEM chunks per epilogue warp
  static constexpr int EWG = R / RW;           // epilogue warpgroups
  static constexpr int EPI_WARPS = 4 * EWG;
  static constexpr int THREADS = 32 * (4 + EPI_WARPS);
  // key-tile ring depth: what shared memory leaves next to two q blocks
  static constexpr int STAGES = R == 8 ? 4 : (H == 64 ? 5 : (PAGED ? 6 : 5));
  // paged: a ring of the tiles' key scales (two 64-token pages each), filled
  // by the producer with bulk copies beside the key tiles; more entries than
  // the producer can run ahead of the epilogue (STAGES + 2 tiles)
  static constexpr int SRING = PAGED ? (STAGES + 3 <= 8 ? 8 : 16) : 0;
  static constexpr int Q_BYTES = N * kDim;
  static constexpr int TILE_BYTES = kBlockKeys * kDim;
  static constexpr int TMEM_COLS = 2 * N <= 256 ? 256 : 512;  // double-buffered accumulators
  static constexpr uint32_t IDESC = idesc_e4m3_f32(kBlockKeys, N);
  static_assert(N <= 256 && N % 16 == 0, "MMA N out of range");
  static_assert(!PAGED || SRING >= STAGES + 3, "scale ring shorter than the producer's lead");
  static_assert(R % RW == 0 && EPI_WARPS <= kMaxEpiWarps, "epilogue layout");
  static_assert(H % 32 == 0 && (NC == 2 || NC == 4), "32-column chunks per epilogue warp");
};

constexpr int kNB = 512;         // histogram bins per row
constexpr int kSelWords = 264;   // per epilogue warp: hist[256], counter, pad
constexpr int kSelWG = 2;        // first warp of the select group
constexpr int kSelWarps = 2;     // warps in the select group
constexpr int kEpiWG = 4;        // first epilogue warp
constexpr int kSelBar = 8;       // the select group's named barrier (epilogue warpgroups use 1..EWG)
constexpr int kUpCap = kMaxTopK; // per select warp: keys above the boundary bin (fewer than topk in all)
constexpr int kAtCap = 1024;     // per select warp: keys inside the boundary bin
constexpr int kSelBatch = 16;    // candidate loads in flight per select thread

// Per (slot, row) streaming state of the fused top-k, shared by the four
// epilogue warps that own the row's keys.  A row's candidate buffer holds
// four equal segments, one per TMEM lane quadrant (key block of 32 inside
// each tile), so each warp appends with a private counter and needs no
// barrier: the histogram is counted with shared-memory atomics, the window is
// opened once by compare-and-swap, and the threshold only grows (atomicMax).
struct RowState {
  int wcnt[4];          // candidates in each segment (written when the unit ends)
  uint32_t theta;       // keep a key iff key >= theta (raised by bounds and by estimates)
  uint32_t theta_spec;  // largest threshold raised by an estimate (0: none): checked after the select
  int lo, hi;           // the row's key range inside this unit's chunk
  int vtot;             // the row's valid keys over the whole key axis
  int pad;
  unsigned long long win;  // histogram window: base | shift << 32 | 1 << 40 once open
};

// Order key of a logit computed as fma(sum, scale, +0), which is -0 only when
// a nonzero negative product rounds to zero: that -0 then orders just below
// +0, as its exact value does.  Two instructions, no -0 fix-up.
__device__ __forceinline__ uint32_t order_key_nz(float f) {
  const uint32_t b = __float_as_uint(f);
  return b ^ (static_cast<uint32_t>(static_cast<int32_t>(b) >> 31) | 0x80000000u);
}

__device__ __forceinline__ float theta_float(uint32_t key) {
  return key <= 0x007FFFFFu ? -INFINITY : key_to_float(key);
}

struct Window {
  bool open;
  uint32_t base;  // bin = min((key - base) >> shift, kNB - 1) for key >= base
  int shift;
};
__device__ __forceinline__ Window window_of(unsigned long long w) {
  return Window{(w >> 40) != 0, static_cast<uint32_t>(w), static_cast<int>((w >> 32) & 0xFF)};
}

struct SlotMeta {
  int unit, row0, nrows, pad;
};

struct SmemLayout {
  int q, stage, bar, misc, w, rows, meta, hist, esel, ssel, up, at, sring, total;
};

template <int R, bool PAGED, int H>
__host__ __device__ constexpr SmemLayout smem_layout() {
  using C = Cfg<R, PAGED, H>;
  SmemLayout L{};
  L.q = 0;  // two q blocks: the next unit's loads while this unit's MMAs run
  L.stage = 2 * C::Q_BYTES;
  L.bar = L.stage + C::STAGES * C::TILE_BYTES;
  L.misc = L.bar + 8 * (2 * C::STAGES + 38);
  L.w = L.misc + 64;
  L.rows = L.w + R * H * 4;
  L.meta = L.rows + 2 * R * static_cast<int>(sizeof(RowState));
  L.hist = L.meta + 2 * static_cast<int>(sizeof(SlotMeta));
  L.esel = L.hist + 2 * R * kNB * 4;
  L.ssel = L.esel + C::EPI_WARPS * kSelWords * 4;
  L.up = L.ssel + 320 * 4;
  L.at = L.up + kSelWarps * kUpCap * 8;
  L.sring = L.at + kSelWarps * kAtCap * 8;
  L.total = L.sring + C::SRING * kBlockKeys * 4;
  return L;
}

// ------------------------------------------------------------------ helpers

struct Unit {
  int row0;      // first query row
  int nrows;     // rows present (<= R)
  int req;       // paged: request
  int cbeg;      // chunk [cbeg, cend) of the key axis
  int cend;
  int jbeg;      // first key of the first tile
  int ntiles;
  int len;       // paged: context length (clamped)
  bool len_clamped;
};

template <int R, bool PAGED>
__device__ __forceinline__ Unit get_unit(const IndexerParams& p, int u) {
  Unit U;
  const int grp = u / p.n_chunks;
  const int c = u - grp * p.n_chunks;
  U.row0 = grp * p.rows_per_unit;  // (<= R: the MMA's row capacity; rows past nrows are idle)
  U.nrows = min(p.rows_per_unit, p.m - U.row0);
  U.req = grp;
  U.len_clamped = false;
  int lo, hi, axis;
  if (!PAGED) {
    axis = static_cast<int>(p.n);
    lo = INT_MAX;
    hi = INT_MIN;
    for (int r = 0; r < U.nrows; ++r) {
      const int a = max(__ldg(p.ks + U.row0 + r), 0);
      const int b = min(__ldg(p.ke + U.row0 + r), axis);
      if (b > a) {
        lo = min(lo, a);
        hi = max(hi, b);
      }
    }
    U.len = 0;
  } else {
    axis = p.max_blocks * kPageSize;
    const int L = __ldg(p.seq_lens + grp);
    U.len_clamped = L > axis;
    U.len = max(min(L, axis), 0);
    lo = 0;
    hi = U.len;
  }
  // chunks of chunk_keys keys, the last tail_chunks of them shorter (tail_keys):
  // the chunk-major order claims those last, so the schedule ends on small units
  const int nfull = p.n_chunks - p.tail_chunks;
  const int clen = c < nfull ? p.chunk_keys : p.tail_keys;
  U.cbeg = c < nfull ? c * p.chunk_keys : nfull * p.chunk_keys + (c - nfull) * p.tail_keys;
  U.cend = min(U.cbeg + clen, axis);
  const int jb = max(U.cbeg, lo), je = min(U.cend, hi);
  U.jbeg = jb;
  U.ntiles = je > jb ? (je - jb + kBlockKeys - 1) / kBlockKeys : 0;
  return U;
}

// Bounded wait on an mbarrier phase.  Gives up when another role has
// aborted or after `limit_ns`, flagging the device status; never traps.
// NAP_NS == 0 polls with try_wait (for the epilogue's own hand-offs, where
// the phase is normally complete already); NAP_NS > 0 passes try_wait a
// suspend-time hint of 16 NAP_NS, so the thread sleeps in hardware until the
// phase completes or the hint runs out, and a role that is ahead of the
// epilogue (MMA issue, TMA producer, idle select warps) takes few issue
// slots from it.  The abort flag and the clock are looked at every 8 tries.
template <uint32_t NAP_NS>
__device__ __noinline__ bool wait_slow(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                       int* status, unsigned long long limit_ns) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (NAP_NS == 0 ? mbar_try_wait(bar, parity) : mbar_try_wait_hint(bar, parity, 16 * NAP_NS)) return true;
    if ((it & 7) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        atomicOr(status, kStatusWaitTimeout);
        return false;
      }
    }
  }
}

// Nap lengths (ns) by role, the unit of each role's suspend-time hint: the
// epilogue polls; the MMA thread's is short (it has slack against the
// epilogue but must not delay the next tile); the producer runs stages
// ahead; idle roles sleep long.
#ifndef FP8IDX_NAP_MMA_NS
#define FP8IDX_NAP_MMA_NS 64
#endif
#ifndef FP8IDX_NAP_PRODUCER_NS
#define FP8IDX_NAP_PRODUCER_NS 256
#endif
#ifndef FP8IDX_NAP_IDLE_NS
#define FP8IDX_NAP_IDLE_NS 2048
#endif
constexpr uint32_t kSpin = 0, kNap = FP8IDX_NAP_MMA_NS, kProd = FP8IDX_NAP_PRODUCER_NS,
                   kSleep = FP8IDX_NAP_IDLE_NS;

template <uint32_t NAP_NS>
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                           int* status, unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow<NAP_NS>(bar, parity, abort_flag, status, limit_ns);
}

// Uniform OR over the threads of a named barrier.
__device__ __forceinline__ bool bar_red_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Uniform count of the threads of a named barrier whose predicate is set.
__device__ __forceinline__ uint32_t bar_red_popc(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.popc.u32 %0, %2, %3, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r;
}

// sum_h w[h] * max(x[h], 0) over the 32 heads of one (key, row), for two
// rows at once.  Heads in groups of four; the first 8 - NABS groups take the
// max on the ALU pipe and the weighted sum as packed two-lane FMAs
// (fma.rn.f32x2): one ALU issue and half an FMA issue per head.  The last
// NABS groups use 2 max(x, 0) = x + |x| instead, all on the FMA pipe (the
// linear half packed, the |x| half with the free absolute-value operand
// modifier), which moves work off the ALU pipe when it is the busier one.
// Each operation rounds once.
template <int NABS>
__device__ __forceinline__ void relu_dot32_pair(const uint32_t (&xa)[32], const uint32_t (&xb)[32],
                                                const float* wa, const float* wb, float& ra, float& rb) {
  const float4* wa4 = reinterpret_cast<const float4*>(wa);
  const float4* wb4 = reinterpret_cast<const float4*>(wb);
  uint64_t la0 = 0, la1 = 0, lb0 = 0, lb1 = 0, ma0 = 0, mb0 = 0;
  float aa0 = 0.f, aa1 = 0.f, ab0 = 0.f, ab1 = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 va = wa4[i], vb = wb4[i];
    if (i < 8 - NABS) {
      const float a0 = fmaxf(__uint_as_float(xa[4 * i + 0]), 0.f), a1 = fmaxf(__uint_as_float(xa[4 * i + 1]), 0.f);
      const float a2 = fmaxf(__uint_as_float(xa[4 * i + 2]), 0.f), a3 = fmaxf(__uint_as_float(xa[4 * i + 3]), 0.f);
      const float b0 = fmaxf(__uint_as_float(xb[4 * i + 0]), 0.f), b1 = fmaxf(__uint_as_float(xb[4 * i + 1]), 0.f);
      const float b2 = fmaxf(__uint_as_float(xb[4 * i + 2]), 0.f), b3 = fmaxf(__uint_as_float(xb[4 * i + 3]), 0.f);
      la0 = fma_f32x2(pack_f32x2(va.x, va.y), pack_f32x2(a0, a1), la0);
      lb0 = fma_f32x2(pack_f32x2(vb.x, vb.y), pack_f32x2(b0, b1), lb0);
      la1 = fma_f32x2(pack_f32x2(va.z, va.w), pack_f32x2(a2, a3), la1);
      lb1 = fma_f32x2(pack_f32x2(vb.z, vb.w), pack_f32x2(b2, b3), lb1);
    } else {
      const float a0 = __uint_as_float(xa[4 * i + 0]), a1 = __uint_as_float(xa[4 * i + 1]);
      const float a2 = __uint_as_float(xa[4 * i + 2]), a3 = __uint_as_float(xa[4 * i + 3]);
      const float b0 = __uint_as_float(xb[4 * i + 0]), b1 = __uint_as_float(xb[4 * i + 1]);
      const float b2 = __uint_as_float(xb[4 * i + 2]), b3 = __uint_as_float(xb[4 * i + 3]);
      ma0 = fma_f32x2(pack_f32x2(va.x, va.y), pack_f32x2(a0, a1), ma0);
      mb0 = fma_f32x2(pack_f32x2(vb.x, vb.y), pack_f32x2(b0, b1), mb0);
      ma0 = fma_f32x2(pack_f32x2(va.z, va.w), pack_f32x2(a2, a3), ma0);
      mb0 = fma_f32x2(pack_f32x2(vb.z, vb.w), pack_f32x2(b2, b3), mb0);
      aa0 = fmaf(va.x, fabsf(a0), aa0);
      ab0 = fmaf(vb.x, fabsf(b0), ab0);
      aa1 = fmaf(va.y, fabsf(a1), aa1);
      ab1 = fmaf(vb.y, fabsf(b1), ab1);
      aa0 = fmaf(va.z, fabsf(a2), aa0);
      ab0 = fmaf(vb.z, fabsf(b2), ab0);
      aa1 = fmaf(va.w, fabsf(a3), aa1);
      ab1 = fmaf(vb.w, fabsf(b3), ab1);
    }
  }
  float p0, p1, q0, q1;
  unpack_f32x2(add_f32x2(la0, la1), p0, p1);
  unpack_f32x2(add_f32x2(lb0, lb1), q0, q1);
  ra = p0 + p1;
  rb = q0 + q1;
  if (NABS > 0) {
    float m0, m1, n0, n1;
    unpack_f32x2(ma0, m0, m1);
    unpack_f32x2(mb0, n0, n1);
    ra += 0.5f * ((m0 + m1) + (aa0 + aa1));
    rb += 0.5f * ((n0 + n1) + (ab0 + ab1));
  }
}

// (Only meaningful for key >= base; any other key maps to some bin in range.)
__device__ __forceinline__ int hist_bin(uint32_t key, uint32_t base, int shift) {
  return static_cast<int>(min((key - base) >> shift, static_cast<uint32_t>(kNB - 1)));
}

// Find the boundary bin: the highest bin b such that at least k counted
// candidates lie in bins >= b.  Every lane returns the same result.  The
// histogram is stored plainly (bin b at h[b]); lane l reads bins 32 i + l,
// so the 16 reads are conflict-free, and the search runs over the 16 rows
// of 32 bins from the top, then over the lanes of the row that holds it.
struct Boundary {
  bool found;
  int bin;
  uint32_t above;  // candidates in bins > bin
  uint32_t inbin;
};

__device__ __forceinline__ Boundary find_boundary(const uint32_t* h, uint32_t k, int lane) {
  constexpr int kRows = kNB / 32;
  uint32_t c[kRows];
#pragma unroll
  for (int i = 0; i < kRows; ++i) c[i] = h[i * 32 + lane];
  Boundary B{false, 0, 0, 0};
  uint32_t run = 0, above_row = 0, v = 0;
  int bi = -1;
#pragma unroll
  for (int i = kRows - 1; i >= 0; --i) {
    const uint32_t tot = __reduce_add_sync(0xFFFFFFFFu, c[i]);
    const bool hit = bi < 0 && run + tot >= k;
    above_row = hit ? run : above_row;
    v = hit ? c[i] : v;
    bi = hit ? i : bi;
    run += tot;
  }
  if (bi < 0) return B;
  // inclusive suffix sum over lanes >= lane of the row's counts
  uint32_t suf = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t t = __shfl_down_sync(0xFFFFFFFFu, suf, off);
    if (lane + off < 32) suf += t;
  }
  const uint32_t ball = __ballot_sync(0xFFFFFFFFu, above_row + suf >= k);
  const int ls = 31 - __clz(static_cast<int>(ball));
  B.found = true;
  B.bin = bi * 32 + ls;
  B.inbin = __shfl_sync(0xFFFFFFFFu, v, ls);
  B.above = above_row + __shfl_sync(0xFFFFFFFFu, suf, ls) - B.inbin;
  return B;
}

// A row's four candidate segments as a select source (positions [0, 4 * wcap)).
struct SegSrc {
  const uint2* buf;
  int wcap;
  int c0, c1, c2, c3;
  __device__ __forceinline__ bool get(int e, uint64_t& K) const {
    const int s = e / wcap;
    const int i = e - s * wcap;
    const int c = s == 0 ? c0 : s == 1 ? c1 : s == 2 ? c2 : c3;
    if (i >= c) return false;
    const uint2 v = buf[e];
    K = compose_key(v.x, v.y);
    return true;
  }
};

// Two shared-memory lists back to back as a select source.
struct TwoListSrc {
  const uint2* a;
  int na;
  const uint2* b;
  int nb;
  __device__ __forceinline__ bool get(int e, uint64_t& K) const {
    uint2 v;
    if (e < na)
      v = a[e];
    else if (e - na < nb)
      v = b[e - na];
    else
      return false;
    K = compose_key(v.x, v.y);
    return true;
  }
};

// Exact top-k of one finished row by the select group (two warps; warp w
// reads segments 2w and 2w+1).  emit(pos, key, index) receives positions
// [0, returned count).  FAST (G = 1 or 2 warps, G * (kUpCap + kAtCap)
// staging pairs in up_all / at_all): keys above the histogram's boundary bin
// are in and the boundary bin is resolved exactly in shared memory; anything
// unusual, and every row when !FAST, takes a radix select over the whole buffer.
template <bool FAST, int G, class Emit>
__device__ int final_select_row(const uint2* rowbuf, int wcap, const RowState& st, const uint32_t* h,
                                int k, const Group<G>& g, uint2* up_all, uint2* at_all,
                                uint32_t* xchg, int* stats, Emit emit) {
  static_assert(!FAST || G <= 2, "the staged path exchanges counts between at most two warps");
  const int w = g.warp(), lane = g.lane();
  const int c[4] = {st.wcnt[0], st.wcnt[1], st.wcnt[2], st.wcnt[3]};
  const int cnt = c[0] + c[1] + c[2] + c[3];
  if (cnt <= k) {
#pragma unroll
    for (int s = w; s < 4; s += G) {
      const int pref = (s > 0 ? c[0] : 0) + (s > 1 ? c[1] : 0) + (s > 2 ? c[2] : 0);
      const uint2* seg = rowbuf + s * wcap;
      for (int i0 = 0; i0 < c[s]; i0 += kSelBatch * 32) {
        uint2 v[kSelBatch];
#pragma unroll
        for (int t = 0; t < kSelBatch; ++t) {
          const int i = i0 + t * 32 + lane;
          if (i < c[s]) v[t] = seg[i];
        }
#pragma unroll
        for (int t = 0; t < kSelBatch; ++t) {
          const int i = i0 + t * 32 + lane;
          if (i < c[s]) emit(pref + i, v[t].x, v[t].y);
        }
      }
    }
    return cnt;
  }
  const Window win = window_of(st.win);
  if (FAST && win.open) {
    const Boundary B = find_boundary(h, static_cast<uint32_t>(k), lane);
    if (B.found) {
      if (g.tid == 0) atomicMax(reinterpret_cast<unsigned*>(stats + kStatMaxBoundary), B.inbin);
      uint2* up_w = up_all + w * kUpCap;
      uint2* at_w = at_all + w * kAtCap;
      uint32_t nu = 0, na = 0;  // warp-uniform counters
      const uint32_t lt = (1u << lane) - 1u;
      // The boundary bin as a key interval [lo_key, hi_key): a key is above
      // the bin iff key >= hi_key (never when the bin is the top, clamped one).
      // (The bin holds at least one key, so its lower edge is below 2^32.)
      const uint32_t lo_key = static_cast<uint32_t>(
          min(static_cast<uint64_t>(win.base) + (static_cast<uint64_t>(B.bin) << win.shift), static_cast<uint64_t>(0xFFFFFFFFu)));
      const uint64_t hi64 = static_cast<uint64_t>(win.base) + (static_cast<uint64_t>(B.bin + 1) << win.shift);
      const bool has_hi = B.bin < kNB - 1 && hi64 <= 0xFFFFFFFFull;
      const uint32_t hi_key = has_hi ? static_cast<uint32_t>(hi64) : 0xFFFFFFFFu;
#pragma unroll
      for (int s = w; s < 4; s += G) {
        const uint2* seg = rowbuf + s * wcap;
        for (int i0 = 0; i0 < c[s]; i0 += kSelBatch * 32) {
          uint2 v[kSelBatch];
#pragma unroll
          for (int t = 0; t < kSelBatch; ++t) {
            const int i = i0 + t * 32 + lane;
            v[t] = i < c[s] ? seg[i] : make_uint2(0u, 0u);
          }
#pragma unroll
          for (int t = 0; t < kSelBatch; ++t) {
            const bool valid = i0 + t * 32 + lane < c[s];
            const bool up = valid && has_hi && v[t].x >= hi_key;
            const bool at = valid && !up && v[t].x >= lo_key;
            const uint32_t mu = __ballot_sync(0xFFFFFFFFu, up);
            const uint32_t ma = __ballot_sync(0xFFFFFFFFu, at);
            if (up) {
              const uint32_t q = nu + __popc(mu & lt);
              if (q < static_cast<uint32_t>(kUpCap)) up_w[q] = v[t];
            }
            if (at) {
              const uint32_t q = na + __popc(ma & lt);
              if (q < static_cast<uint32_t>(kAtCap)) at_w[q] = v[t];
            }
            nu += __popc(mu);
            na += __popc(ma);
          }
        }
      }
      uint32_t nu0 = nu, na0 = na, nu1 = 0, na1 = 0;
      if (G > 1) {
        if (lane == 0) {
          xchg[2 * w] = nu;
          xchg[2 * w + 1] = na;
        }
        g.sync();
        nu0 = xchg[0];
        na0 = xchg[1];
        nu1 = xchg[2];
        na1 = xchg[3];
      }
      const bool consistent = nu0 + nu1 == B.above && na0 + na1 == B.inbin &&
                              nu0 <= static_cast<uint32_t>(kUpCap) && nu1 <= static_cast<uint32_t>(kUpCap) &&
                              na0 <= static_cast<uint32_t>(kAtCap) && na1 <= static_cast<uint32_t>(kAtCap);
      if (consistent) {
        const uint32_t off = w == 0 ? 0u : nu0;
        const uint32_t mine = w == 0 ? nu0 : nu1;
        for (uint32_t i = lane; i < mine; i += 32) emit(static_cast<int>(off + i), up_w[i].x, up_w[i].y);
        const int need = k - static_cast<int>(B.above);
        const TwoListSrc src{at_all, static_cast<int>(na0), at_all + kAtCap, static_cast<int>(na1)};
        const int tot = static_cast<int>(na0 + na1);
        const SelectResult sel = group_select<G>(src, tot, need, g);
        const int n2 = group_emit<G>(src, tot, sel, g, [&](int pos, uint64_t K) {
          emit(static_cast<int>(B.above) + pos, composite_value(K), composite_index(K));
        });
        return static_cast<int>(B.above) + n2;
      }
    }
  }
  // general path: radix select over the whole buffer
  if (FAST && g.tid == 0) atomicAdd(stats + kStatGeneralSelects, 1);
  const SegSrc src{rowbuf, wcap, c[0], c[1], c[2], c[3]};
  const SelectResult sel = group_select<G>(src, 4 * wcap, k, g);
  return group_emit<G>(src, 4 * wcap, sel, g, [&](int pos, uint64_t K) {
    emit(pos, composite_value(K), composite_index(K));
  });
}

// Minimum of one value per thread over a select group (xchg: two words of
// scratch when the group has two warps).
template <int G>
__device__ __forceinline__ uint32_t group_min(uint32_t v, const Group<G>& g, uint32_t* xchg) {
  v = __reduce_min_sync(0xFFFFFFFFu, v);
  if (G > 1) {
    g.sync();
    if (g.lane() == 0) xchg[10 + g.warp()] = v;
    g.sync();
    v = min(xchg[10], xchg[11]);
    g.sync();
  }
  return v;
}

// A row whose threshold was raised by an estimate: the result is the row's
// top-k iff it is complete and its smallest key is at or above the largest
// estimate applied (every key at or above that estimate passed every filter).
// Otherwise the row's group (row block or request) is listed, once, for an
// exact recomputation.
__device__ __forceinline__ void check_estimate(const IndexerParams& p, int group, uint32_t spec, bool complete,
                                               uint32_t kth_key, bool leader) {
  if ((complete && kth_key >= spec) || !leader) return;
  atomicAdd(p.status + kStatRepairs, 1);
  if (atomicExch(p.repair_flag + group, 1) == 0) p.repair_list[atomicAdd(p.status + kRepairCount, 1)] = group;
}

// Exact top-k of one finished row (row rl of a slot) written out: the final
// list (-1 / -inf padded) with one key chunk, else the unit's partial list and
// its length.
template <bool FAST, int R, int G>
__device__ void write_row_topk(const IndexerParams& p, const SlotMeta& meta, int rl, const RowState& st,
                               const uint32_t* h, const uint2* rowbuf, const Group<G>& g,
                               uint2* up_all, uint2* at_all, uint32_t* xchg) {
  const int k = p.topk;
  const int wcap = p.cand_cap >> 2;
  const bool present = rl < meta.nrows;
  const int cnt = st.wcnt[0] + st.wcnt[1] + st.wcnt[2] + st.wcnt[3];
  if (present && g.tid == 0) atomicAdd(p.status + kStatCandidates, cnt);
  if (p.n_chunks == 1) {
    if (!present) return;
    const int row = meta.row0 + rl;
    int32_t* orow = p.out_idx + static_cast<int64_t>(row) * k;
    float* vrow = p.out_vals ? p.out_vals + static_cast<int64_t>(row) * k : nullptr;
    uint32_t vmin = 0xFFFFFFFFu;  // the smallest order key written (this thread's share)
    const int req = row / p.rows_per_unit;  // paged: the row's request
    const int nout = final_select_row<FAST>(rowbuf, wcap, st, h, k, g, up_all, at_all, xchg, p.status,
                                            [&](int pos, uint32_t key, uint32_t j) {
                                              orow[pos] = p.out_slots ? slot_of(p.block_table, p.max_blocks,
                                                                                p.num_pages, req,
                                                                                static_cast<int32_t>(j))
                                                                      : static_cast<int32_t>(j);
                                              if (vrow) vrow[pos] = key_to_float(key);
                                              vmin = min(vmin, key);
                                            });
    for (int pos = nout + g.tid; pos < k; pos += 32 * G) {
      orow[pos] = -1;
      if (vrow) vrow[pos] = -INFINITY;
    }
    if (st.theta_spec != 0u)
      check_estimate(p, meta.unit, st.theta_spec, nout >= min(k, st.vtot), group_min(vmin, g, xchg), g.tid == 0);
  } else {
    uint2* prow = p.part + (static_cast<size_t>(meta.unit) * R + rl) * k;
    int nout = 0;
    if (present && cnt > 0)
      nout = final_select_row<FAST>(rowbuf, wcap, st, h, k, g, up_all, at_all, xchg, p.status,
                                    [&](int pos, uint32_t key, uint32_t j) { prow[pos] = make_uint2(key, j); });
    if (g.tid == 0) p.part_cnt[static_cast<size_t>(meta.unit) * R + rl] = nout;
  }
}

// ------------------------------------------------------------------ vote-time row maintenance
//
// The epilogue's hot loop only filters and appends.  Every few tiles each
// warp, on its own schedule (no barrier), counts its newly appended
// candidates into the rows' shared histograms, makes room in a segment that
// is filling up, and reloads the rows' thresholds; warp qd of a warpgroup
// also raises the threshold of the group's row qd from that row's histogram.
// Each counted key is a real key of the row, so a histogram count taken at
// any moment (other warps may still be adding) is a lower bound and the
// threshold it gives stays a valid lower bound on the row's k-th value.

__device__ __forceinline__ unsigned long long ld_volatile_u64(const unsigned long long* p) {
  return *reinterpret_cast<const volatile unsigned long long*>(p);
}
__device__ __forceinline__ uint32_t ld_volatile_u32(const uint32_t* p) {
  return *reinterpret_cast<const volatile uint32_t*>(p);
}
__device__ __forceinline__ int ld_volatile_i32(const int* p) { return *reinterpret_cast<const volatile int*>(p); }

// Count candidates [from, to) of one warp's segment of a row into the row's
// histogram.  If the row's window is not open yet (then from == 0: nothing of
// this warp has been counted), the warp proposes one from its own candidates
// (twice their key span above their minimum) by compare-and-swap; the first
// proposal wins and every warp counts with it.  Returns the new counted mark.
__device__ __forceinline__ int fold_segment(const uint2* seg, int from, int to, RowState* st, uint32_t* h,
                                         int lane) {
  if (from >= to) return from;
  __syncwarp();  // the warp's own appends are visible to all its lanes
  unsigned long long wv = ld_volatile_u64(&st->win);
  if (!(wv >> 40)) {
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0;
    for (int e = lane; e < to; e += 32) {
      const uint32_t key = seg[e].x;
      kmin = min(kmin, key);
      kmax = max(kmax, key);
    }
    kmin = __reduce_min_sync(0xFFFFFFFFu, kmin);
    kmax = __reduce_max_sync(0xFFFFFFFFu, kmax);
    const uint64_t span = static_cast<uint64_t>(kmax - kmin);
    const int bits = 64 - __clzll(static_cast<long long>(2 * span + 1));
    const int shift = bits > 9 ? bits - 9 : 0;
    const unsigned long long mine =
        static_cast<unsigned long long>(kmin) | (static_cast<unsigned long long>(shift) << 32) | (1ull << 40);
    if (lane == 0) atomicCAS(&st->win, 0ull, mine);
    __syncwarp();
    wv = ld_volatile_u64(&st->win);
  }
  const Window w = window_of(wv);
  for (int e0 = from; e0 < to; e0 += 4 * 32) {
    uint32_t key[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = e0 + i * 32 + lane;
      key[i] = e < to ? seg[e].x : 0u;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = e0 + i * 32 + lane;
      if (e < to && key[i] >= w.base) atomicAdd(&h[hist_bin(key[i], w.base, w.shift)], 1u);
    }
  }
  return to;
}

// Count the candidates each of a warp's RW rows appended since the last
// vote into the rows' histograms.  The common case (at most 128 new keys per
// row) issues every row's loads before any count, so the read-back costs one
// L2 round trip per vote; a row whose window is still closed, or that
// appended more, goes through fold_segment.
template <int RW>
__device__ __forceinline__ void fold_rows(const uint2* seg0, int cap, int (&folded)[RW], const int (&cnt)[RW],
                                          RowState* rs, uint32_t* hs, int lane) {
  __syncwarp();  // the warp's own appends are visible to all its lanes
  uint32_t kk[RW][4];
#pragma unroll
  for (int r = 0; r < RW; ++r) {
    const uint2* seg = seg0 + static_cast<size_t>(r) * cap;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = folded[r] + i * 32 + lane;
      kk[r][i] = e < cnt[r] ? seg[e].x : 0u;
    }
  }
#pragma unroll
  for (int r = 0; r < RW; ++r) {
    if (folded[r] >= cnt[r]) continue;
    const Window w = window_of(ld_volatile_u64(&rs[r].win));
    if (!w.open || cnt[r] - folded[r] > 4 * 32) {
      folded[r] = fold_segment(seg0 + static_cast<size_t>(r) * cap, folded[r], cnt[r], rs + r, hs + r * kNB, lane);
      continue;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = folded[r] + i * 32 + lane;
      if (e < cnt[r] && kk[r][i] >= w.base) atomicAdd(&hs[r * kNB + hist_bin(kk[r][i], w.base, w.shift)], 1u);
    }
    folded[r] = cnt[r];
  }
}

// A contiguous candidate list as a select source.
struct ListSrc {
  const uint2* a;
  int n;
  __device__ __forceinline__ bool get(int e, uint64_t& K) const {
    if (e >= n) return false;
    const uint2 v = a[e];
    K = compose_key(v.x, v.y);
    return true;
  }
};

// Make room in one warp's segment of a row (cnt candidates, all counted):
// drop candidates below the row's threshold; if that leaves fewer than
// `room` free slots, keep the segment's exact top-k, staged through `scr`.
// The k-th kept key is then a lower bound on the row's k-th value, and,
// since every later key has a larger index, a later key equal to it can
// never enter the top-k: the threshold rises to just above it.  The
// histogram keeps counting the dropped keys: they are real keys of the row.
__device__ __forceinline__ int compact_segment(uint2* seg, int cnt, int room, int wcap, int k, RowState* st,
                                            uint2* scr, const Group<1>& grp, int* stats, int lane) {
  const uint32_t lt = (1u << lane) - 1u;
  const uint32_t th = ld_volatile_u32(&st->theta);
  __syncwarp();
  int n = 0;
  for (int e0 = 0; e0 < cnt; e0 += 32) {
    const int e = e0 + lane;
    const uint2 v = e < cnt ? seg[e] : make_uint2(0u, 0u);
    const bool keep = e < cnt && v.x >= th;
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep) seg[n + __popc(m & lt)] = v;  // n + rank <= e: never ahead of the reads
    n += __popc(m);
  }
  __syncwarp();
  if (n + room <= wcap) return n;
  const ListSrc src{seg, n};
  const SelectResult sel = group_select<1>(src, n, k, grp);
  uint32_t umin = 0xFFFFFFFFu;
  const int kept = group_emit<1>(src, n, sel, grp, [&](int pos, uint64_t K) {
    scr[pos] = make_uint2(composite_value(K), composite_index(K));
    umin = min(umin, composite_value(K));
  });
  umin = __reduce_min_sync(0xFFFFFFFFu, umin);
  __syncwarp();
  for (int pos = lane; pos < kept; pos += 32) seg[pos] = scr[pos];
  __syncwarp();
  if (lane == 0) {
    if (kept >= k && umin != 0xFFFFFFFFu) atomicMax(&st->theta, umin + 1);
    atomicAdd(stats + kStatCompactions, 1);
  }
  return kept;
}

// Raise a row's threshold from its histogram.  Exact: to the lower edge of
// the bin that holds the k-th counted key (at least k keys of the row lie at
// or above it).  Estimated (target < k): to the lower edge of the bin that
// holds the target-th counted key, where the target is the expected number
// of the row's top-k among the keys seen so far plus a five-sigma margin; the
// result is then recorded as an estimate to be checked after the select.
// With the key axis split over several units, thresholds are shared through
// the row's words in global memory (any unit's bound is a bound for the
// whole row; estimates are recorded there too): this unit's bound goes out as
// a reduction that returns nothing, and the row's word is read without
// waiting, its value taken up at the next vote (`gseen`), so that no vote
// waits on a round trip to L2.
__device__ __forceinline__ void raise_theta(const uint32_t* h, RowState* st, int target, bool estimate,
                                            uint32_t* row_theta, uint32_t* row_spec, uint32_t& gseen,
                                            int lane) {
  const Window w = window_of(ld_volatile_u64(&st->win));
  uint32_t th = 0;
  if (w.open) {
    const Boundary B = find_boundary(h, static_cast<uint32_t>(target), lane);
    if (B.found) {
      const uint64_t t64 = static_cast<uint64_t>(w.base) + (static_cast<uint64_t>(B.bin) << w.shift);
      th = t64 > 0xFFFFFFFFull ? 0xFFFFFFFFu : static_cast<uint32_t>(t64);
    }
  }
  if (lane == 0) {
    if (estimate && th) {
      atomicMax(&st->theta_spec, th);
      if (row_spec) atomicMax(row_spec, th);
    }
    if (row_theta) {
      if (th) atomicMax(row_theta, th);
      th = max(th, gseen);
      gseen = ld_volatile_u32(row_theta);
    }
    if (th) atomicMax(&st->theta, th);
  }
}

// The target count of an estimated threshold after `seen` of a row's `vtot`
// keys: mean + 5 sqrt(mean) + 8 with mean = k * seen / vtot (the expected
// number of the row's top-k among keys seen in random order).  Returns k
// (exact) when the estimate would not be below the exact bound.
__device__ __forceinline__ int estimate_target(int k, int seen, int vtot) {
  if (vtot <= k || seen <= 0) return k;
  const float mean = static_cast<float>(k) * static_cast<float>(seen) / static_cast<float>(vtot);
  const float c = ceilf(mean + 5.0f * sqrtf(mean) + 8.0f);
  return c < static_cast<float>(min(k, seen)) ? static_cast<int>(c) : k;
}

// ------------------------------------------------------------------ kernel

template <int R, bool PAGED, int H, int MODE>
__global__ void __launch_bounds__(Cfg<R, PAGED, H>::THREADS, 1) indexer_kernel(const __grid_constant__ IndexerParams p) {
  using C = Cfg<R, PAGED, H>;
  constexpr SmemLayout SL = smem_layout<R, PAGED, H>();
  constexpr int N = C::N;
  constexpr int RW = C::RW;
  constexpr int S = C::STAGES;
  constexpr uint32_t SR = C::SRING > 0 ? C::SRING : 1;  // scale ring entries (paged)
  static_assert(4 * (kUpCap + kAtCap) * 8 <= SL.stage + S * C::TILE_BYTES,
                "end-of-kernel select staging must fit in the q and key-tile buffers");

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base (128-byte swizzled TMA tiles), derived by pointer
  // arithmetic on the shared array so that accesses stay shared-memory ones
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* q_smem = smem + SL.q;
  uint8_t* stage_smem = smem + SL.stage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SL.bar);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* tempty = bars + 2 * S + 2;
  uint64_t* qfull = bars + 2 * S + 4;      // two q slots
  uint64_t* qempty = bars + 2 * S + 6;
  uint64_t* drain = bars + 2 * S + 8;
  uint64_t* slot_full = bars + 2 * S + 9;
  uint64_t* slot_empty = bars + 2 * S + 11;
  uint64_t* uq_full = bars + 2 * S + 13;   // unit queue, 4 entries
  uint64_t* uq_empty = bars + 2 * S + 17;
  uint64_t* sfull = bars + 2 * S + 21;     // paged: the scale ring (SRING entries)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SL.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SL.misc + 4);
  volatile int* uq = reinterpret_cast<volatile int*>(smem + SL.misc + 16);  // unit queue
  int* claim = reinterpret_cast<int*>(smem + SL.misc + 32);  // rows of each slot handed out so far
  float* w_smem = reinterpret_cast<float*>(smem + SL.w);
  RowState* rstate = reinterpret_cast<RowState*>(smem + SL.rows);
  SlotMeta* smeta = reinterpret_cast<SlotMeta*>(smem + SL.meta);
  uint32_t* hist_smem = reinterpret_cast<uint32_t*>(smem + SL.hist);
  uint32_t* esel_smem = reinterpret_cast<uint32_t*>(smem + SL.esel);
  uint32_t* ssel_smem = reinterpret_cast<uint32_t*>(smem + SL.ssel);
  uint2* up_smem = reinterpret_cast<uint2*>(smem + SL.up);
  uint2* at_smem = reinterpret_cast<uint2*>(smem + SL.at);
  float* sring = reinterpret_cast<float*>(smem + SL.sring);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // launched as a dependent grid, wait here for the grids before it on the
  // stream to complete (a no-op otherwise)
  griddep_wait();
  // a repair launch with nothing listed ends at once (the count is final: the
  // launches that list groups ran before this one on the stream)
  if (p.repair_mode && ld_volatile_i32(p.status + kRepairCount) == 0) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], C::EPI_WARPS);
      mbar_init(&slot_full[a], C::EPI_WARPS);
      mbar_init(&slot_empty[a], kSelWarps);
    }
    for (int x = 0; x < 4; ++x) {
      mbar_init(&uq_full[x], 1);
      mbar_init(&uq_empty[x], 1 + C::EPI_WARPS);  // the MMA thread and every epilogue warp
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&qfull[x], 1);
      mbar_init(&qempty[x], 1);
    }
    for (int x = 0; x < C::SRING; ++x) mbar_init(&sfull[x], 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  const unsigned long long limit = p.wait_limit_ns;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tmap_q);
      tma_prefetch_desc(&p.tmap_k);
      int stage = 0;
      uint32_t phase = 0;
      int nq = 0;  // units with tiles so far: unit nq uses q slot nq & 1
      uint32_t issued_phase[S];
      bool issued[S];
#pragma unroll
      for (int s = 0; s < S; ++s) {
        issued[s] = false;
        issued_phase[s] = 0;
      }
      bool ok = true;
      uint32_t Tp = 0;                      // the CTA's tiles issued so far
      uint32_t s_issued = 0, s_phase = 0;   // scale ring entries with a copy issued, and its phase
      // Dynamic schedule: units are claimed from a counter in the status block
      // and announced to the MMA and epilogue warps through a four-entry
      // queue; -1 ends the stream.  Whole-row units go last row block first
      // (the largest, in the causal layouts).  With a split key axis the order
      // is chunk-major: every row block's (request's) first chunk, then every
      // second one, and so on, so that full chunks come before the short last
      // ones and a row's later chunks start from the threshold its earlier
      // chunks raised.
      for (int n = 0; ok; ++n) {
        const int qs = n & 3;
        if (!wait_phase<kSleep>(&uq_empty[qs], ((n >> 2) & 1) ^ 1, abort_flag, p.status, limit)) { ok = false; break; }
        // Claim only once a q slot is free, i.e. once the MMA is done with the
        // unit before last: a CTA then holds at most one unit beyond the one
        // in flight, so that at the end no CTA sits on work another could do.
        // (An empty unit leaves its slot free; the next wait passes at once.)
        const int qs2 = nq & 1;
        if (!wait_phase<kProd>(&qempty[qs2], ((nq >> 1) & 1) ^ 1, abort_flag, p.status, limit)) { ok = false; break; }
        int u = -1;
        if (p.repair_mode) {  // the groups the checks listed, one unit each (whole rows)
          const int idx = atomicAdd(p.status + kRepairSched, 1);
          if (idx < ld_volatile_i32(p.status + kRepairCount)) u = p.repair_list[idx];
        } else {
          const int idx = atomicAdd(p.status + kSchedWord, 1);
          if (idx < p.num_units) {
            const int groups = p.num_units / p.n_chunks;
            u = p.n_chunks == 1 ? p.num_units - 1 - idx
                                : (groups - 1 - idx % groups) * p.n_chunks + idx / groups;
          }
        }
        uq[qs] = u;
        mbar_arrive(&uq_full[qs]);
        if (u < 0) break;
        const Unit U = get_unit<R, PAGED>(p, u);
        if (U.ntiles == 0) continue;
        ++nq;
        mbar_arrive_expect_tx(&qfull[qs2], C::Q_BYTES);
        tma_load_2d(q_smem + qs2 * C::Q_BYTES, &p.tmap_q, &qfull[qs2], 0, U.row0 * H);
        const int32_t* bt = PAGED ? p.block_table + static_cast<int64_t>(U.req) * p.max_blocks : nullptr;
        for (int t = 0; t < U.ntiles; ++t) {
          if (!wait_phase<kProd>(&empty[stage], phase ^ 1, abort_flag, p.status, limit)) { ok = false; break; }
          const int j0 = U.jbeg + t * kBlockKeys;
          uint8_t* dst = stage_smem + stage * C::TILE_BYTES;
          // paged: the tile's two pages through the block table
          const bool has1 = PAGED && j0 + kPageSize < U.len;
          const int32_t pg0 = PAGED ? __ldg(bt + j0 / kPageSize) : -1;
          const int32_t pg1 = has1 ? __ldg(bt + j0 / kPageSize + 1) : -1;
          const bool v0 = pg0 >= 0 && pg0 < p.num_pages;
          const bool v1 = has1 && pg1 >= 0 && pg1 < p.num_pages;
          if (p.debug_withhold_first_tile && n == 0 && t == 0) {
            // tests only: this stage never fills, so the MMA's bounded wait on
            // it runs out and the kernel takes its timeout path
          } else if (!PAGED) {
            mbar_arrive_expect_tx(&full[stage], C::TILE_BYTES);
            tma_load_2d(dst, &p.tmap_k, &full[stage], 0, j0);
          } else {
            if (!v0 || (has1 && !v1)) atomicOr(p.status, kStatusBadPage);
            mbar_arrive_expect_tx(&full[stage], (v0 ? 8192u : 0u) + (v1 ? 8192u : 0u));
            if (v0) tma_load_2d(dst, &p.tmap_k, &full[stage], 0, pg0 * kPageSize);
            if (v1) tma_load_2d(dst + 8192, &p.tmap_k, &full[stage], 0, pg1 * kPageSize);
          }
          if (PAGED) {  // the tile's key scales into the ring (a page outside the pool: zeros)
            const int e = static_cast<int>(Tp % SR);
            float* sd = sring + e * kBlockKeys;
            mbar_arrive_expect_tx(&sfull[e], has1 ? 512u : 256u);
            bulk_load(sd, v0 ? p.s + static_cast<int64_t>(pg0) * kPageSize : g_zero_scales, 256u, &sfull[e]);
            if (has1)
              bulk_load(sd + kPageSize, v1 ? p.s + static_cast<int64_t>(pg1) * kPageSize : g_zero_scales, 256u,
                        &sfull[e]);
            s_issued |= 1u << e;
            s_phase = (s_phase & ~(1u << e)) | (((Tp / SR) & 1u) << e);
          }
          ++Tp;
          issued[stage] = !(p.debug_withhold_first_tile && n == 0 && t == 0);
          issued_phase[stage] = phase;
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Never leave a copy in flight: wait for every stage's last issued load
      // and every scale ring entry's last copy.
#pragma unroll 1
      for (int s = 0; s < S; ++s) {
        if (!issued[s]) continue;
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&full[s], issued_phase[s]) && global_timer_ns() - t0 < 200000000ull) {
        }
      }
#pragma unroll 1
      for (int e = 0; e < C::SRING; ++e) {
        if (!((s_issued >> e) & 1u)) continue;
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&sfull[e], (s_phase >> e) & 1u) && global_timer_ns() - t0 < 200000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int nq = 0;  // units with tiles so far (the producer's q slot order)
      uint32_t T = 0;
      bool ok = true;
      bool any = false;
      const uint32_t q_addr = smem_u32(q_smem);
      for (int n = 0; ok; ++n) {
        const int qs = n & 3;
        if (!wait_phase<kSpin>(&uq_full[qs], (n >> 2) & 1, abort_flag, p.status, limit)) { ok = false; break; }
        const int u = uq[qs];
        mbar_arrive(&uq_empty[qs]);
        if (u < 0) break;
        const Unit U = get_unit<R, PAGED>(p, u);
        if (U.ntiles == 0) continue;
        const int qs2 = nq & 1;
        if (!wait_phase<kNap>(&qfull[qs2], (nq >> 1) & 1, abort_flag, p.status, limit)) { ok = false; break; }
        ++nq;
        tc_fence_after();
        const uint64_t bdesc = smem_desc_k128_sw128(q_addr + qs2 * C::Q_BYTES);
        for (int t = 0; t < U.ntiles; ++t, ++T) {
          const uint32_t a = T & 1, aph = (T >> 1) & 1;
          if (!wait_phase<kNap>(&tempty[a], aph ^ 1, abort_flag, p.status, limit)) { ok = false; break; }
          tc_fence_after();
          if (!wait_phase<kNap>(&full[stage], phase, abort_flag, p.status, limit)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = smem_desc_k128_sw128(smem_u32(stage_smem + stage * C::TILE_BYTES));
          const uint32_t d = tbase + a * N;
#pragma unroll
          for (int kk = 0; kk < kDim / 32; ++kk)
            mma_f8(d, adesc + 2 * kk, bdesc + 2 * kk, C::IDESC, kk > 0 ? 1u : 0u);
          mma_commit(&empty[stage]);
          mma_commit(&tfull[a]);
          any = true;
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) mma_commit(&qempty[qs2]);
      }
      if (any) {  // all MMAs retired before TMEM is released
        mma_commit(drain);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < 200000000ull) {
        }
      }
    }
  } else if (warp >= kEpiWG) {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp - kEpiWG;  // 0 .. EPI_WARPS - 1
    const int g = ew >> 2;    // warpgroup
    const int qd = warp & 3;  // TMEM lane quadrant == key block of 32 == buffer segment
    const int tid_wg = qd * 32 + lane;
    const int bar_id = 1 + g;
    float* ws_g = w_smem + g * RW * H;
    Group<1> grp{esel_smem + ew * kSelWords, nullptr, esel_smem + ew * kSelWords + 256, 0, lane};
    const int k = p.topk;
    const int cap = p.cand_cap;
    const int wcap = cap >> 2;  // segment capacity
    const uint32_t lane_addr = tbase + (static_cast<uint32_t>(qd * 32) << 16);
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t T = 0;
    bool aborted = false;

    for (int it = 0;; ++it) {
      const int qs = it & 3;
      const bool got = wait_phase<kSpin>(&uq_full[qs], (it >> 2) & 1, abort_flag, p.status, limit);
      // every warp of the group must take the same branch below (named barriers)
      if (bar_red_or(bar_id, 128, !got || aborted || *abort_flag)) {
        aborted = true;
        break;
      }
      const int u = uq[qs];
      __syncwarp();
      if (lane == 0) mbar_arrive(&uq_empty[qs]);
      const int slot = it & 1;
      if (u < 0) {
        if (MODE == kModeTopK) {
          // Out of units.  Warpgroup 0 takes rows of the last two units off
          // the select group, which may still be busy with them: each warp
          // claims a row and selects it alone, staging in the q and key-tile
          // buffers (every MMA of this CTA has completed, so they are free).
          // The CTA then does not finish on the select group's two warps.
          if (g == 0) {
            uint2* up_h = reinterpret_cast<uint2*>(smem) + qd * (kUpCap + kAtCap);
            for (int back = 2; back >= 1; --back) {
              if (it < back) continue;
              const int hslot = (it - back) & 1;
              if (!wait_phase<kSleep>(&slot_full[hslot], ((it - back) >> 1) & 1, abort_flag, p.status, limit)) break;
              const SlotMeta meta = smeta[hslot];
              for (;;) {
                int rl = 0;
                if (lane == 0) rl = atomicAdd(claim + hslot, 1);
                rl = __shfl_sync(0xFFFFFFFFu, rl, 0);
                if (rl >= R) break;
                write_row_topk<true, R>(p, meta, rl, rstate[hslot * R + rl], hist_smem + (hslot * R + rl) * kNB,
                                        p.cand + (static_cast<size_t>(blockIdx.x * 2 + hslot) * R + rl) * cap, grp,
                                        up_h, up_h + kUpCap, nullptr);
                __syncwarp();
              }
            }
          }
          // tell the select group (unit -1 in the slot)
          wait_phase<kSleep>(&slot_empty[slot], ((it >> 1) & 1) ^ 1, abort_flag, p.status, limit);
          if (g == 0 && tid_wg == 0) smeta[slot].unit = -1;
          named_bar_sync(bar_id, 128);
          __syncwarp();
          if (lane == 0) mbar_arrive(&slot_full[slot]);
        }
        break;
      }
      const Unit U = get_unit<R, PAGED>(p, u);
      RowState* rs = rstate + slot * R + g * RW;
      uint32_t* hs = hist_smem + (slot * R + g * RW) * kNB;
      uint2* cand_s = MODE == kModeTopK
                          ? p.cand + (static_cast<size_t>(blockIdx.x * 2 + slot) * R + g * RW) * cap
                          : nullptr;
      if (MODE == kModeTopK) {
        if (!wait_phase<kNap>(&slot_empty[slot], ((it >> 1) & 1) ^ 1, abort_flag, p.status, limit)) aborted = true;
      }
      // ---- per-row setup for this warpgroup's rows: the key range [lo, hi)
      // (kept in shared memory; the tile loop reads it back as a broadcast)
      if (tid_wg < RW) {
        const int rl = g * RW + tid_wg;
        int lo = 0, hi = 0, vtot = 0;
        if (rl < U.nrows) {
          const int row = U.row0 + rl;
          if (!PAGED) {
            lo = max(__ldg(p.ks + row), 0);
            hi = max(lo, min(__ldg(p.ke + row), static_cast<int>(p.n)));
          } else {
            const int e = U.len - p.rows_per_unit + rl + 1;
            hi = max(min(e, U.len), 0);
          }
          vtot = hi - lo;
          // a unit only owns the keys of its chunk (its last tile may overhang)
          lo = max(lo, U.cbeg);
          hi = max(lo, min(hi, U.cend));
        }
        rs[tid_wg].lo = lo;
        rs[tid_wg].hi = hi;
        rs[tid_wg].vtot = vtot;
      }
      for (int x = tid_wg; x < RW * H; x += 128) {
        const int rl = g * RW + x / H;
        ws_g[x] = rl < U.nrows ? __ldg(p.w + static_cast<int64_t>(U.row0 + rl) * H + x % H) : 0.f;
      }
      if (MODE == kModeTopK) {
        if (tid_wg < RW) {
          RowState& st = rs[tid_wg];
          st.wcnt[0] = st.wcnt[1] = st.wcnt[2] = st.wcnt[3] = 0;
          // with a split key axis a unit starts from the row's shared bound,
          // which the row's other chunks may have raised already
          const int rl = g * RW + tid_wg;
          st.theta = p.n_chunks > 1 && rl < U.nrows ? ld_volatile_u32(p.row_theta + U.row0 + rl) : 0u;
          st.theta_spec = 0;
          st.win = 0ull;
        }
        for (int x = tid_wg; x < RW * kNB; x += 128) hs[x] = 0;
        if (g == 0 && tid_wg == 0) {
          claim[slot] = 0;
          smeta[slot].unit = u;
          smeta[slot].row0 = U.row0;
          smeta[slot].nrows = U.nrows;
          if (PAGED && U.len_clamped) atomicOr(p.status, kStatusSeqLenTooLong);
        }
      }
      if (bar_red_or(bar_id, 128, aborted || *abort_flag)) {
        aborted = true;
        break;
      }

      if (MODE == kModeLogits) {
        // keys of this chunk that no tile covers are -inf
        const int tb = U.ntiles ? U.jbeg : U.cend;
        const int te = U.ntiles ? U.jbeg + U.ntiles * kBlockKeys : U.cend;
#pragma unroll
        for (int r = 0; r < RW; ++r) {
          if (g * RW + r >= U.nrows) continue;
          float* lrow = p.logits + static_cast<int64_t>(U.row0 + g * RW + r) * p.ld_logits;
          for (int j = U.cbeg + tid_wg; j < U.cend; j += 128)
            if (j < tb || j >= te) __stcs(lrow + j, -INFINITY);
        }
      }

      // ---- this warp's registers per row: candidates in its segment, how many of
      // them the row's histogram has counted, the key range, and the threshold
      // (reloaded from the row state at every vote)
      int cnt[RW], folded[RW], lo[RW], span[RW];
      float thf[RW];
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        cnt[r] = 0;
        folded[r] = 0;
        lo[r] = rs[r].lo;
        span[r] = rs[r].hi - rs[r].lo;
        thf[r] = MODE == kModeTopK ? theta_float(rs[r].theta) : -INFINITY;
      }
      uint2* seg0 = MODE == kModeTopK ? cand_s + qd * wcap : nullptr;  // row r's segment: seg0 + r * cap
      uint32_t gseen = 0;  // split key axis: the row's shared bound as read at this warp's last vote

      // ---- stream the unit's key tiles
      const int key0 = U.jbeg + qd * 32 + lane;
      // key scales: read a tile ahead from global memory; paged, from the
      // producer's scale ring (the tile's pages are scattered over the pool)
      auto scale_of = [&](int j) -> float { return j < p.n ? __ldg(p.s + j) : 0.f; };
      float s_next = !PAGED && U.ntiles ? scale_of(key0) : 0.f;
      int next_vote = vote_interval(0) - 1;  // the same tile sequence in every warp
      // The warp's RW rows are NC chunks of 32 TMEM columns (chunk c at column
      // g * RW * H + 32 c, its head weights at ws_g + 32 c), taken in pairs; a
      // later pair's loads are in flight while the pair before it is summed.
      // With a single pair (NC == 2), the next tile's pair is loaded as soon
      // as its accumulator is ready, before this tile's filter runs (xa, xb
      // carry it from one iteration to the next); with two pairs the
      // registers this would hold across the filter are not there.
      constexpr bool kCarry = C::NC == 2;
      constexpr int kAbsGroups = PAGED ? 0 : 2;  // head groups summed on the FMA pipe (see relu_dot32_pair)
      uint32_t xa[32], xb[32];
      if (kCarry && U.ntiles > 0) {
        if (!wait_phase<kSpin>(&tfull[T & 1], (T >> 1) & 1, abort_flag, p.status, limit)) aborted = true;
        tc_fence_after();
        const uint32_t col0 = lane_addr + (T & 1) * N + g * RW * H;
        tmem_ld32(col0, xa);
        tmem_ld32(col0 + 32, xb);
      }
      for (int t = 0; t < U.ntiles; ++t, ++T) {
        const int j = key0 + t * kBlockKeys;
        float sj = s_next;
        if (PAGED) {
          // (read before this warp releases the tile's accumulator: the
          // producer refills the entry only after every warp has done so)
          const int e = static_cast<int>(T % SR);
          if (!wait_phase<kSpin>(&sfull[e], (T / SR) & 1, abort_flag, p.status, limit)) aborted = true;
          sj = j < U.len ? sring[e * kBlockKeys + qd * 32 + lane] : 0.f;
        } else {
          s_next = scale_of(j + kBlockKeys);  // (0 past the end)
        }
        const uint32_t a = T & 1;
        // The last wait leaves the whole accumulator in registers: release it
        // to the MMA.  A row's logit sums its H / 32 chunks.  (fma with +0: an
        // exactly zero head sum gives +0 whatever the sign of the scale.)
        constexpr int NC = C::NC;
        float Lc[NC];
        {
          const uint32_t col0 = lane_addr + a * N + g * RW * H;
          if (!kCarry) {
            if (!wait_phase<kSpin>(&tfull[a], (T >> 1) & 1, abort_flag, p.status, limit)) aborted = true;
            tc_fence_after();
            tmem_ld32(col0, xa);
            tmem_ld32(col0 + 32, xb);
          }
          tmem_ld_wait();  // the first pair
          if (NC == 2) {
            tc_fence_before();
            __syncwarp();
            mbar_arrive_if(lane == 0, &tempty[a]);
            relu_dot32_pair<kAbsGroups>(xa, xb, ws_g, ws_g + 32, Lc[0], Lc[1]);
          } else {
            uint32_t xc[32], xd[32];
            tmem_ld32(col0 + 64, xc);
            tmem_ld32(col0 + 96, xd);
            relu_dot32_pair<kAbsGroups>(xa, xb, ws_g, ws_g + 32, Lc[0], Lc[1]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            mbar_arrive_if(lane == 0, &tempty[a]);
            relu_dot32_pair<kAbsGroups>(xc, xd, ws_g + 64, ws_g + 96, Lc[2], Lc[NC - 1]);
          }
        }
        float L[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) {
          float acc = Lc[r * (H / 32)];
#pragma unroll
          for (int c = 1; c < H / 32; ++c) acc += Lc[r * (H / 32) + c];
          L[r] = fmaf(acc, sj, 0.f);
        }
        if (kCarry && t + 1 < U.ntiles) {  // the next tile's pair, in flight during this tile's filter
          const uint32_t an = (T + 1) & 1;
          if (!wait_phase<kSpin>(&tfull[an], ((T + 1) >> 1) & 1, abort_flag, p.status, limit)) aborted = true;
          tc_fence_after();
          const uint32_t coln = lane_addr + an * N + g * RW * H;
          tmem_ld32(coln, xa);
          tmem_ld32(coln + 32, xb);
        }

        if (MODE == kModeLogits) {
#pragma unroll
          for (int r = 0; r < RW; ++r) {
            if (g * RW + r >= U.nrows || j >= U.cend) continue;
            float* lrow = p.logits + static_cast<int64_t>(U.row0 + g * RW + r) * p.ld_logits;
            __stcs(lrow + j, static_cast<uint32_t>(j - lo[r]) < static_cast<uint32_t>(span[r]) ? L[r] : -INFINITY);
          }
          if (aborted) break;
        } else {
          // ---- filter against the row's threshold and append to this warp's
          // segment (the row's histogram counts them at the next vote).  Stage by
          // stage over the rows, so that the rows' chains interleave ahead of
          // the stores (which keep their order).
          bool ps[RW];
          uint32_t key[RW], msk[RW];
#pragma unroll
          for (int r = 0; r < RW; ++r) {
            ps[r] = static_cast<uint32_t>(j - lo[r]) < static_cast<uint32_t>(span[r]) && L[r] >= thf[r];
            key[r] = order_key_nz(L[r]);
          }
#pragma unroll
          for (int r = 0; r < RW; ++r) msk[r] = __ballot_sync(0xFFFFFFFFu, ps[r]);
          int pos[RW];
#pragma unroll
          for (int r = 0; r < RW; ++r) {
            pos[r] = cnt[r] + __popc(msk[r] & lt);
            cnt[r] += __popc(msk[r]);
          }
#pragma unroll
          for (int r = 0; r < RW; ++r)
            st_global_v2_if(ps[r] && pos[r] < wcap, seg0 + static_cast<size_t>(r) * cap + pos[r], key[r],
                            static_cast<uint32_t>(j));

          // ---- vote: count, make room, reload the thresholds (this warp alone)
          if (t == next_vote || t + 1 == U.ntiles) {
            const int vnext = vote_interval(t + 1);
            next_vote = t + vnext;
            if (aborted || *abort_flag) {
              aborted = true;
              break;
            }
            const int room = min(vnext, U.ntiles - 1 - t) * 32;  // what may be appended before the next vote
            bool full = false;
#pragma unroll
            for (int r = 0; r < RW; ++r) {
              if (cnt[r] > wcap && lane == 0) atomicOr(p.status, kStatusCandOverflow);
              cnt[r] = min(cnt[r], wcap);
              full |= cnt[r] + room > wcap;
            }
            fold_rows<RW>(seg0, cap, folded, cnt, rs, hs, lane);
            while (full) {  // rare: one row at a time, through a single copy of the compaction
              int cr = -1, cc = 0;
#pragma unroll
              for (int r = RW - 1; r >= 0; --r)
                if (cnt[r] + room > wcap) {
                  cr = r;
                  cc = cnt[r];
                }
              if (cr < 0) break;
              uint2* scr = p.scratch + (static_cast<size_t>(blockIdx.x) * kMaxEpiWarps + ew) * k;
              const int nc = compact_segment(seg0 + static_cast<size_t>(cr) * cap, cc, room, wcap, k, rs + cr, scr,
                                             grp, p.status, lane);
#pragma unroll
              for (int r = 0; r < RW; ++r)
                if (r == cr) cnt[r] = folded[r] = nc;
            }
            if (qd < RW && g * RW + qd < U.nrows) {
              // this warp keeps the threshold of the group's row qd.  An estimate
              // takes the row's keys in tiles [0, t + 1] as seen.  Another warp
              // may already have counted tile t + 2 (this warp has released
              // tile t's accumulator), which makes the estimate a little
              // bolder; like any estimate it is checked against the result.
              const RowState* me = rs + qd;
              int target = k;
              if (p.speculate) {
                const int mlo = ld_volatile_i32(&me->lo), mhi = ld_volatile_i32(&me->hi);
                const int seen = min(mhi, U.jbeg + (t + 2) * kBlockKeys) - max(mlo, U.jbeg);
                target = estimate_target(k, max(0, min(seen, mhi - mlo)), ld_volatile_i32(&me->vtot));
              }
              const int row = U.row0 + g * RW + qd;
              raise_theta(hs + qd * kNB, rs + qd, target, target < k, p.n_chunks > 1 ? p.row_theta + row : nullptr,
                          p.n_chunks > 1 ? p.row_spec + row : nullptr, gseen, lane);
            }
#pragma unroll
            for (int r = 0; r < RW; ++r) thf[r] = theta_float(ld_volatile_u32(&rs[r].theta));
          }
        }
      }
      tmem_ld_wait();  // no TMEM load of this warp stays in flight past its tile loop
      // (an aborted warp carries on to the next unit's group vote, which ends
      // the loop for every warp of the group together)
      if (MODE == kModeTopK) {
        if (lane == 0) {
#pragma unroll
          for (int r = 0; r < RW; ++r) rs[r].wcnt[qd] = cnt[r];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&slot_full[slot]);  // releases this warp's row-state and candidate writes
      }
    }
  } else if (MODE == kModeTopK) {
    // ---------------------------------------------------------------- select group
    const int stid = (warp - kSelWG) * 32 + lane;
    constexpr int NT = 32 * kSelWarps;
    Group<kSelWarps> grp{ssel_smem, ssel_smem + 256, ssel_smem + 300, kSelBar, stid};
    uint32_t* xchg = ssel_smem + 304;
    const int cap = p.cand_cap;
    const int wcap = cap >> 2;
    for (int it = 0;; ++it) {
      const int slot = it & 1;
      const bool ok = wait_phase<kSleep>(&slot_full[slot], (it >> 1) & 1, abort_flag, p.status, limit);
      if (bar_red_or(kSelBar, NT, !ok || *abort_flag)) break;
      const SlotMeta meta = smeta[slot];
      if (meta.unit < 0) break;
      // The unit's candidate segments were written one unit ago and have
      // mostly left L2: each row's segments are brought back two rows ahead
      // of its pass (thread `stid` of the group prefetches segment `stid`).
      auto prefetch_row = [&](int rl) {
        if (stid < 4 && rl < meta.nrows) {
          const int c = min(rstate[slot * R + rl].wcnt[stid], wcap);
          const uint2* seg = p.cand + (static_cast<size_t>(blockIdx.x * 2 + slot) * R + rl) * cap + stid * wcap;
          if (c > 0) l2_prefetch_bulk(seg, static_cast<uint32_t>((c + 1) & ~1) * 8u);
        }
      };
      prefetch_row(0);
      prefetch_row(1);
      // Rows are claimed one at a time from the slot's counter: the epilogue
      // warps, once out of units, claim the last unit's remaining rows too.
      for (;;) {
        if (stid == 0) xchg[8] = static_cast<uint32_t>(atomicAdd(claim + slot, 1));
        grp.sync();
        const int rl = static_cast<int>(xchg[8]);
        if (rl >= R) break;
        prefetch_row(rl + 2);
        const RowState st = rstate[slot * R + rl];
        write_row_topk<true, R>(p, meta, rl, st, hist_smem + (slot * R + rl) * kNB,
                                p.cand + (static_cast<size_t>(blockIdx.x * 2 + slot) * R + rl) * cap, grp,
                                up_smem, at_smem, xchg);
        grp.sync();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&slot_empty[slot]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ merge

// Union of a row's partial top-k lists (one per key chunk) as a select source.
struct PartSrc {
  const uint2* base;  // partial list of chunk 0 of this row; chunk c at base + c * stride
  const int* cnt;     // count of chunk c at cnt[c * cstride]
  size_t stride;
  int cstride;
  int topk;
  __device__ __forceinline__ bool get(int e, uint64_t& K) const {
    const int c = e / topk;
    const int i = e - c * topk;
    if (i >= __ldg(cnt + static_cast<size_t>(c) * cstride)) return false;  // (i < topk always)
    const uint2 v = base[static_cast<size_t>(c) * stride + i];
    K = compose_key(v.x, v.y);
    return true;
  }
};

// A row's partial lists gathered densely in shared memory.
struct DenseSrc {
  const uint2* a;
  __device__ __forceinline__ bool get(int e, uint64_t& K) const {
    const uint2 v = a[e];
    K = compose_key(v.x, v.y);
    return true;
  }
};

constexpr int kMergeWarps = 8;
constexpr int kMergeMaxChunks = kMergeWarps * 32;  // one chunk count per thread
constexpr int kMergeStage = 12288;                 // pairs a row can gather in shared memory (96 KB: two CTAs per SM)

// One CTA per row.  The chunk counts are scanned into offsets; when the
// row's surviving pairs fit, they are gathered densely into shared memory and
// selected there, else the select reads the partial lists in place.
__global__ void __launch_bounds__(kMergeWarps * 32) merge_kernel(const MergeParams p) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t red[8 * kMergeWarps];
  __shared__ uint32_t counter;
  __shared__ int pre[kMergeMaxChunks + 1];
  __shared__ int wsum[kMergeWarps];
  extern __shared__ uint2 stage[];  // kMergeStage pairs (dynamic)
  griddep_wait();  // the indexer's partial lists are complete
  const int row = blockIdx.x;
  const int unit_row = row / p.R;  // row block / request
  const int rl = row - unit_row * p.R;
  const size_t u0 = static_cast<size_t>(unit_row) * p.n_chunks;
  const uint2* base = p.part + (u0 * p.R_part + rl) * p.topk;
  const size_t stride = static_cast<size_t>(p.R_part) * p.topk;
  const int* cnt = p.part_cnt + u0 * p.R_part + rl;
  Group<kMergeWarps> g{hist, red, &counter, 1, static_cast<int>(threadIdx.x)};
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int total = -1;  // pairs surviving in all chunks (-1: not scanned)
  if (p.n_chunks <= kMergeMaxChunks) {
    const int c = threadIdx.x;
    // a count outside [0, topk] only follows an aborted indexer launch (the
    // device status says so); clamped, it still keeps every access in bounds
    const int v = c < p.n_chunks ? min(max(__ldg(cnt + static_cast<size_t>(c) * p.R_part), 0), p.topk) : 0;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += t;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    if (c < p.n_chunks) pre[c] = before + incl - v;
    if (c == kMergeMaxChunks - 1) pre[p.n_chunks] = before + incl;
    __syncthreads();
    total = pre[p.n_chunks];
  }
  int32_t* orow = p.out_idx + static_cast<int64_t>(row) * p.topk;
  float* vrow = p.out_vals ? p.out_vals + static_cast<int64_t>(row) * p.topk : nullptr;
  uint32_t vmin = 0xFFFFFFFFu;  // the smallest order key written (this thread's share)
  auto emit = [&](int pos, uint64_t K) {
    const int32_t j = static_cast<int32_t>(composite_index(K));
    orow[pos] = p.block_table ? slot_of(p.block_table, p.max_blocks, p.num_pages, unit_row, j) : j;
    if (vrow) vrow[pos] = key_to_float(composite_value(K));
    vmin = min(vmin, composite_value(K));
  };
  int nout;
  if (total >= 0 && total <= kMergeStage) {
    for (int c = warp; c < p.n_chunks; c += kMergeWarps) {
      const uint2* src = base + static_cast<size_t>(c) * stride;
      const int n = pre[c + 1] - pre[c];
      for (int i = lane; i < n; i += 32) stage[pre[c] + i] = src[i];
    }
    __syncthreads();
    const DenseSrc src{stage};
    const SelectResult sel = group_select<kMergeWarps>(src, total, p.topk, g);
    nout = group_emit<kMergeWarps>(src, total, sel, g, emit);
  } else {
    const PartSrc src{base, cnt, stride, p.R_part, p.topk};
    const int all = p.n_chunks * p.topk;
    const SelectResult sel = group_select<kMergeWarps>(src, all, p.topk, g);
    nout = group_emit<kMergeWarps>(src, all, sel, g, emit);
  }
  for (int pos = nout + threadIdx.x; pos < p.topk; pos += blockDim.x) {
    orow[pos] = -1;
    if (vrow) vrow[pos] = -INFINITY;
  }
  // A row whose threshold was raised by an estimate (only rows with more than
  // topk keys): complete, with its smallest key at or above the largest
  // estimate applied, or its request is listed for an exact recomputation.
  const uint32_t spec = p.row_spec ? p.row_spec[row] : 0u;
  if (spec != 0u) {
    vmin = __reduce_min_sync(0xFFFFFFFFu, vmin);
    if (lane == 0) red[warp] = vmin;
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t m = 0xFFFFFFFFu;
      for (int w = 0; w < kMergeWarps; ++w) m = min(m, red[w]);
      if (nout < p.topk || m < spec) {
        atomicAdd(p.status + kStatRepairs, 1);
        if (atomicExch(p.repair_flag + unit_row, 1) == 0)
          p.repair_list[atomicAdd(p.status + kRepairCount, 1)] = unit_row;
      }
    }
  }
}

// ------------------------------------------------------------------ top-k of materialised rows

struct RowSrc {
  const float* row;
  int64_t lo;
  __device__ __forceinline__ bool get(int e, uint64_t& K) const {
    const int64_t j = lo + e;
    K = compose_key(order_key(__ldg(row + j)), static_cast<uint32_t>(j));
    return true;
  }
};

constexpr int kTopkRowsWarps = 16;

__global__ void __launch_bounds__(kTopkRowsWarps * 32) topk_rows_kernel(const TopkRowsParams p) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t red[8 * kTopkRowsWarps];
  __shared__ uint32_t counter;
  const int row = blockIdx.x;
  const int64_t lo = max(static_cast<int64_t>(p.ks[row]), static_cast<int64_t>(0));
  const int64_t hi = max(lo, min(static_cast<int64_t>(p.ke[row]), p.n));
  RowSrc src{p.logits + static_cast<int64_t>(row) * p.ld, lo};
  Group<kTopkRowsWarps> g{hist, red, &counter, 1, static_cast<int>(threadIdx.x)};
  const int total = static_cast<int>(hi - lo);
  const SelectResult sel = group_select<kTopkRowsWarps>(src, total, p.topk, g);
  int32_t* orow = p.out_idx + static_cast<int64_t>(row) * p.topk;
  const int nout = group_emit<kTopkRowsWarps>(src, total, sel, g, [&](int pos, uint64_t K) {
    orow[pos] = static_cast<int32_t>(composite_index(K));
  });
  for (int pos = nout + threadIdx.x; pos < p.topk; pos += blockDim.x) orow[pos] = -1;
}

__global__ void fill_empty_kernel(int32_t* out_idx, float* out_vals, int64_t total) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    out_idx[i] = -1;
    if (out_vals) out_vals[i] = -INFINITY;
  }
}

// ------------------------------------------------------------------ launchers

// Launch `kern`; `dependent`: as a programmatic dependent of the kernel before
// it on the stream, which lets the launch overlap that kernel's end (the
// kernel itself waits for it in griddep_wait before reading its results).
template <class Kern, class Params>
static cudaError_t launch_kernel(Kern kern, int grid, int block, size_t smem, cudaStream_t st, bool dependent,
                                 const Params& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(block));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int R, bool PAGED, int H, int MODE>
static cudaError_t launch_indexer(const IndexerParams& p, int grid, cudaStream_t st) {
  static_assert(smem_layout<R, PAGED, H>().total + 1024 <= 227 * 1024, "shared memory per CTA");
  static_assert(smem_layout<R, PAGED, H>().sring % 16 == 0, "bulk copies need 16-byte aligned destinations");
  const size_t smem = static_cast<size_t>(smem_layout<R, PAGED, H>().total) + 1024;
  auto kern = indexer_kernel<R, PAGED, H, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // the repair launch follows a kernel of the same call on the stream: launch
  // it as a dependent grid, so that its launch overlaps that kernel's end
  return launch_kernel(kern, grid, Cfg<R, PAGED, H>::THREADS, smem, st, p.repair_mode != 0, p);
}

// Instantiations: 32 heads with 8-row prefill units (4- or 8-row paged
// units); 64 heads with 4-row units (N = 4 x 64 = 256 columns).
cudaError_t launch_indexer_prefill_logits(const IndexerParams& p, int H, int grid, cudaStream_t st) {
  if (H == 64) return launch_indexer<4, false, 64, kModeLogits>(p, grid, st);
  return launch_indexer<kPrefillRows, false, 32, kModeLogits>(p, grid, st);
}
cudaError_t launch_indexer_prefill_topk(const IndexerParams& p, int H, int grid, cudaStream_t st) {
  if (H == 64) return launch_indexer<4, false, 64, kModeTopK>(p, grid, st);
  return launch_indexer<kPrefillRows, false, 32, kModeTopK>(p, grid, st);
}
cudaError_t launch_indexer_paged_topk(const IndexerParams& p, int R, int H, int grid, cudaStream_t st) {
  if (H == 64) return launch_indexer<4, true, 64, kModeTopK>(p, grid, st);
  if (R == 8) return launch_indexer<8, true, 32, kModeTopK>(p, grid, st);
  return launch_indexer<4, true, 32, kModeTopK>(p, grid, st);
}

cudaError_t launch_merge(const MergeParams& p, cudaStream_t st) {
  constexpr int smem = kMergeStage * static_cast<int>(sizeof(uint2));
  cudaError_t e = cudaFuncSetAttribute(merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_kernel(merge_kernel, p.rows, kMergeWarps * 32, smem, st, true, p);  // (after the indexer)
}

cudaError_t launch_topk_rows(const TopkRowsParams& p, cudaStream_t st) {
  topk_rows_kernel<<<p.m, kTopkRowsWarps * 32, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_fill_empty(int32_t* out_idx, float* out_vals, int rows, int topk, cudaStream_t st) {
  const int64_t total = static_cast<int64_t>(rows) * topk;
  if (total == 0) return cudaSuccess;
  const int64_t want = (total + 255) / 256;
  const int blocks = static_cast<int>(want < 4096 ? want : 4096);
  fill_empty_kernel<<<blocks, 256, 0, st>>>(out_idx, out_vals, total);
  return cudaGetLastError();
}

}  // namespace fp8idx
