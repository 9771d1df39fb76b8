// kernels.cu -- the indexer kernels for sm_100a.
//
// What is computed (the indexer call of the "bench_mqa_logits_chunking.py"
// page: `fp8_mqa_logits` then `fast_topk_transform_fused`, H = 32, D = 128):
//   L[i,j] = s[j] * sum_h w[i,h] * ReLU(q[i,h,:] . k[j,:])  on ks[i] <= j < ke[i], else -inf
//   out[i] = the top-k j of row i (larger L first, lower j on ties), padded with -1.
//
// Design (one persistent CTA per SM, warp-specialised):
//   warp 0      TMA producer: the unit's q block [R rows x 32 heads x 128 B]
//               once, then 128-key tiles [128 x 128 B] through a ring of
//               shared-memory stages (paged keys: two 64-token pages a tile).
//   warp 1      MMA issuer: tcgen05.mma kind::f8f6f4 with M = 128 keys,
//               N = R*32 (row, head) columns, K = 128 as 4 x K32 steps, fp32
//               accumulators in TMEM, double buffered (2 x N columns).
//   warps 2..9  epilogue, two warpgroups of 4 (one warp per TMEM lane
//               quadrant, so one thread per key); warpgroup g owns rows
//               [g*R/2, (g+1)*R/2) of the unit.  Each thread reads its key's
//               32 head dots per row from TMEM, applies ReLU, the head
//               weights and the key scale, then either writes the logit
//               (mqa_logits) or filters it against the row's running
//               threshold into a per-row candidate buffer (fused top-k).
// A unit is R query rows (a row block, or one request's rows in the paged
// form) times one chunk of keys.  With one chunk per unit the fused kernel
// writes the final top-k; with several, each unit writes its exact partial
// top-k and the merge kernel selects from the union.
#include <cfloat>
#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace fp8idx {

template <int R, bool PAGED>
struct Cfg {
  static constexpr int N = R * kHeads;         // MMA N: (row, head) columns
  static constexpr int RW = R / 2;             // rows per epilogue warpgroup
  static constexpr int STAGES = PAGED ? 8 : 5; // key-tile ring depth
  static constexpr int Q_BYTES = N * kDim;
  static constexpr int TILE_BYTES = kBlockKeys * kDim;
  static constexpr int TMEM_COLS = 2 * N;
  static constexpr uint32_t IDESC = idesc_e4m3_f32(kBlockKeys, N);
  static_assert(N <= 256 && N % 16 == 0, "MMA N out of range");
  static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM columns must be a power of two");
};

constexpr int kSelWords = 264;  // per epilogue warp: hist[256], counter, pad

struct SmemLayout {
  int q, stage, bar, misc, w, rows, sel, total;
};

template <int R, bool PAGED>
__host__ __device__ constexpr SmemLayout smem_layout() {
  using C = Cfg<R, PAGED>;
  SmemLayout L{};
  L.q = 0;
  L.stage = C::Q_BYTES;
  L.bar = L.stage + C::STAGES * C::TILE_BYTES;
  L.misc = L.bar + 8 * (2 * C::STAGES + 8);
  L.w = L.misc + 64;
  L.rows = L.w + R * kHeads * 4;
  L.sel = L.rows + 2 * R * 4;
  L.total = L.sel + 8 * kSelWords * 4;
  return L;
}

// ------------------------------------------------------------------ helpers

struct Unit {
  int row0;      // first query row
  int nrows;     // rows present (<= R)
  int req;       // paged: request
  int64_t cbeg;  // chunk [cbeg, cend) of the key axis
  int64_t cend;
  int64_t jbeg;  // first key of the first tile
  int ntiles;
  int64_t len;   // paged: context length (clamped)
};

template <int R, bool PAGED>
__device__ __forceinline__ Unit get_unit(const IndexerParams& p, int u) {
  Unit U;
  const int grp = u / p.n_chunks;
  const int c = u - grp * p.n_chunks;
  U.row0 = grp * R;
  U.nrows = min(R, p.m - U.row0);
  U.req = grp;
  int64_t lo, hi, axis;
  if (!PAGED) {
    axis = p.n;
    lo = INT64_MAX;
    hi = INT64_MIN;
    for (int r = 0; r < U.nrows; ++r) {
      int64_t a = max(static_cast<int64_t>(__ldg(p.ks + U.row0 + r)), static_cast<int64_t>(0));
      int64_t b = min(static_cast<int64_t>(__ldg(p.ke + U.row0 + r)), p.n);
      if (b > a) {
        lo = min(lo, a);
        hi = max(hi, b);
      }
    }
    U.len = 0;
  } else {
    axis = static_cast<int64_t>(p.max_blocks) * kPageSize;
    int64_t L = __ldg(p.seq_lens + grp);
    L = max(min(L, axis), static_cast<int64_t>(0));
    U.len = L;
    lo = 0;
    hi = L;
  }
  U.cbeg = static_cast<int64_t>(c) * p.chunk_keys;
  U.cend = min(U.cbeg + p.chunk_keys, axis);
  const int64_t jb = max(U.cbeg, lo), je = min(U.cend, hi);
  U.jbeg = jb;
  U.ntiles = je > jb ? static_cast<int>((je - jb + kBlockKeys - 1) / kBlockKeys) : 0;
  return U;
}

// Bounded wait on an mbarrier phase.  Gives up when another role has
// aborted or after `limit_ns`, flagging the device status; never traps.
__device__ __noinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                      int* status, unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  uint32_t it = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++it & 31) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        atomicOr(status, kStatusWaitTimeout);
        return false;
      }
    }
  }
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

// sum_h w[h] * max(x[h], 0) over the 32 heads of one (key, row).
__device__ __forceinline__ float relu_dot32(const uint32_t (&x)[32], const float* wsm) {
  const float4* w4 = reinterpret_cast<const float4*>(wsm);
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 wv = w4[i];
    a0 = fmaf(wv.x, fmaxf(__uint_as_float(x[4 * i + 0]), 0.f), a0);
    a1 = fmaf(wv.y, fmaxf(__uint_as_float(x[4 * i + 1]), 0.f), a1);
    a2 = fmaf(wv.z, fmaxf(__uint_as_float(x[4 * i + 2]), 0.f), a2);
    a3 = fmaf(wv.w, fmaxf(__uint_as_float(x[4 * i + 3]), 0.f), a3);
  }
  return (a0 + a1) + (a2 + a3);
}

// A row's candidate buffer as a select source.
struct BufSrc {
  const uint2* buf;
  __device__ __forceinline__ bool get(int e, uint64_t& K) const {
    const uint2 v = buf[e];
    K = compose_key(v.x, v.y);
    return true;
  }
};

// ------------------------------------------------------------------ kernel

template <int R, bool PAGED, int MODE>
__global__ void __launch_bounds__(kThreads, 1) indexer_kernel(const __grid_constant__ IndexerParams p) {
  using C = Cfg<R, PAGED>;
  constexpr SmemLayout SL = smem_layout<R, PAGED>();
  constexpr int N = C::N;
  constexpr int RW = C::RW;
  constexpr int S = C::STAGES;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* q_smem = smem + SL.q;
  uint8_t* stage_smem = smem + SL.stage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SL.bar);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* tempty = bars + 2 * S + 2;
  uint64_t* qfull = bars + 2 * S + 4;
  uint64_t* qempty = bars + 2 * S + 5;
  uint64_t* drain = bars + 2 * S + 6;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SL.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SL.misc + 4);
  float* w_smem = reinterpret_cast<float*>(smem + SL.w);
  int* cnt_smem = reinterpret_cast<int*>(smem + SL.rows);
  uint32_t* theta_smem = reinterpret_cast<uint32_t*>(smem + SL.rows + R * 4);
  uint32_t* sel_smem = reinterpret_cast<uint32_t*>(smem + SL.sel);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
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
      uint32_t phase = 0, qphase = 0;
      uint32_t issued_phase[S];
      bool issued[S];
#pragma unroll
      for (int s = 0; s < S; ++s) {
        issued[s] = false;
        issued_phase[s] = 0;
      }
      bool ok = true;
      for (int i = blockIdx.x; ok && i < p.num_units; i += gridDim.x) {
        const int u = p.num_units - 1 - i;
        const Unit U = get_unit<R, PAGED>(p, u);
        if (U.ntiles == 0) continue;
        if (!wait_bar(qempty, qphase ^ 1, abort_flag, p.status, limit)) { ok = false; break; }
        qphase ^= 1;
        mbar_arrive_expect_tx(qfull, C::Q_BYTES);
        tma_load_2d(q_smem, &p.tmap_q, qfull, 0, U.row0 * kHeads);
        for (int t = 0; t < U.ntiles; ++t) {
          if (!wait_bar(&empty[stage], phase ^ 1, abort_flag, p.status, limit)) { ok = false; break; }
          const int64_t j0 = U.jbeg + static_cast<int64_t>(t) * kBlockKeys;
          uint8_t* dst = stage_smem + stage * C::TILE_BYTES;
          if (!PAGED) {
            mbar_arrive_expect_tx(&full[stage], C::TILE_BYTES);
            tma_load_2d(dst, &p.tmap_k, &full[stage], 0, static_cast<int32_t>(j0));
          } else {
            const int64_t lp = j0 / kPageSize;
            const int32_t* bt = p.block_table + static_cast<int64_t>(U.req) * p.max_blocks;
            int32_t pg0 = __ldg(bt + lp);
            int32_t pg1 = (j0 + kPageSize < U.len) ? __ldg(bt + lp + 1) : -1;
            bool v0 = pg0 >= 0 && pg0 < p.num_pages;
            bool v1 = pg1 >= 0 && pg1 < p.num_pages;
            if (!v0 || (j0 + kPageSize < U.len && !v1)) atomicOr(p.status, kStatusBadPage);
            mbar_arrive_expect_tx(&full[stage], (v0 ? 8192u : 0u) + (v1 ? 8192u : 0u));
            if (v0) tma_load_2d(dst, &p.tmap_k, &full[stage], 0, pg0 * kPageSize);
            if (v1) tma_load_2d(dst + 8192, &p.tmap_k, &full[stage], 0, pg1 * kPageSize);
          }
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Never leave a copy in flight: wait for every stage's last issued load.
#pragma unroll 1
      for (int s = 0; s < S; ++s) {
        if (!issued[s]) continue;
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&full[s], issued_phase[s]) && global_timer_ns() - t0 < 200000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, qphase = 0;
      uint32_t T = 0;
      bool ok = true;
      bool any = false;
      const uint32_t q_addr = smem_u32(q_smem);
      for (int i = blockIdx.x; ok && i < p.num_units; i += gridDim.x) {
        const int u = p.num_units - 1 - i;
        const Unit U = get_unit<R, PAGED>(p, u);
        if (U.ntiles == 0) continue;
        if (!wait_bar(qfull, qphase, abort_flag, p.status, limit)) { ok = false; break; }
        qphase ^= 1;
        tc_fence_after();
        const uint64_t bdesc = smem_desc_k128_sw128(q_addr);
        for (int t = 0; t < U.ntiles; ++t, ++T) {
          const uint32_t a = T & 1, aph = (T >> 1) & 1;
          if (!wait_bar(&tempty[a], aph ^ 1, abort_flag, p.status, limit)) { ok = false; break; }
          tc_fence_after();
          if (!wait_bar(&full[stage], phase, abort_flag, p.status, limit)) { ok = false; break; }
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
        if (ok) mma_commit(qempty);
      }
      if (any) {  // all MMAs retired before TMEM is released
        mma_commit(drain);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < 200000000ull) {
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp - 2;  // 0..7
    const int g = ew >> 2;    // warpgroup
    const int qd = warp & 3;  // TMEM lane quadrant == key block of 32
    const int tid_wg = qd * 32 + lane;
    const int bar_id = 1 + g;
    float* ws_g = w_smem + g * RW * kHeads;
    int* cnt_g = cnt_smem + g * RW;
    uint32_t* th_g = theta_smem + g * RW;
    Group<1> grp{sel_smem + ew * kSelWords, nullptr, sel_smem + ew * kSelWords + 256, 0, lane};
    const int k = p.topk;
    const int cap = p.cand_cap;
    uint2* cand_g = p.cand ? p.cand + (static_cast<size_t>(blockIdx.x) * R + g * RW) * cap : nullptr;
    const uint32_t lane_addr = tbase + (static_cast<uint32_t>(qd * 32) << 16);
    uint32_t T = 0;
    bool aborted = false;

    for (int i = blockIdx.x; i < p.num_units; i += gridDim.x) {
      const int u = p.num_units - 1 - i;
      const Unit U = get_unit<R, PAGED>(p, u);
      // ---- per-row setup for this warpgroup's rows
      int64_t lo_r[RW], hi_r[RW];
      bool rv[RW];
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        const int rl = g * RW + r;
        rv[r] = rl < U.nrows;
        lo_r[r] = 0;
        hi_r[r] = 0;
        if (rv[r]) {
          const int row = U.row0 + rl;
          if (!PAGED) {
            int64_t a = max(static_cast<int64_t>(__ldg(p.ks + row)), static_cast<int64_t>(0));
            int64_t b = min(static_cast<int64_t>(__ldg(p.ke + row)), p.n);
            lo_r[r] = a;
            hi_r[r] = max(a, b);
          } else {
            int64_t e = U.len - R + rl + 1;
            hi_r[r] = max(min(e, U.len), static_cast<int64_t>(0));
          }
          // a unit only owns the keys of its chunk (its last tile may overhang)
          lo_r[r] = max(lo_r[r], U.cbeg);
          hi_r[r] = min(hi_r[r], U.cend);
        }
      }
      if (tid_wg < RW * kHeads) {
        const int rl = g * RW + tid_wg / kHeads;
        ws_g[tid_wg] = rl < U.nrows ? __ldg(p.w + static_cast<int64_t>(U.row0 + rl) * kHeads + tid_wg % kHeads) : 0.f;
      }
      if (tid_wg < RW) {
        cnt_g[tid_wg] = 0;
        th_g[tid_wg] = 0;
      }
      named_bar_sync(bar_id, 128);

      if (MODE == kModeLogits) {
        // keys of this chunk that no tile covers are -inf
        const int64_t tb = U.ntiles ? U.jbeg : U.cend;
        const int64_t te = U.ntiles ? U.jbeg + static_cast<int64_t>(U.ntiles) * kBlockKeys : U.cend;
#pragma unroll
        for (int r = 0; r < RW; ++r) {
          if (!rv[r]) continue;
          float* lrow = p.logits + static_cast<int64_t>(U.row0 + g * RW + r) * p.ld_logits;
          for (int64_t j = U.cbeg + tid_wg; j < U.cend; j += 128)
            if (j < tb || j >= te) __stcs(lrow + j, -INFINITY);
        }
      }

      // ---- stream the unit's key tiles
      const int64_t key0 = U.jbeg + qd * 32 + lane;
      auto scale_of = [&](int64_t j) -> float {
        if (!PAGED) return j < p.n ? __ldg(p.s + j) : 0.f;
        if (j >= U.len) return 0.f;
        const int32_t pg = __ldg(p.block_table + static_cast<int64_t>(U.req) * p.max_blocks + j / kPageSize);
        if (pg < 0 || pg >= p.num_pages) return 0.f;
        return __ldg(p.s + static_cast<int64_t>(pg) * kPageSize + (j % kPageSize));
      };
      float s_next = U.ntiles ? scale_of(key0) : 0.f;
      for (int t = 0; t < U.ntiles; ++t, ++T) {
        const int64_t j = key0 + static_cast<int64_t>(t) * kBlockKeys;
        const float sj = s_next;
        if (t + 1 < U.ntiles) s_next = scale_of(j + kBlockKeys);
        const uint32_t a = T & 1, aph = (T >> 1) & 1;
        if (!wait_bar(&tfull[a], aph, abort_flag, p.status, limit)) aborted = true;
        tc_fence_after();
        float L[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) {
          uint32_t x[32];
          tmem_ld32(lane_addr + a * N + (g * RW + r) * kHeads, x);
          tmem_ld_wait();
          L[r] = relu_dot32(x, ws_g + r * kHeads) * sj;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[a]);

        if (MODE == kModeLogits) {
#pragma unroll
          for (int r = 0; r < RW; ++r) {
            if (!rv[r] || j >= U.cend) continue;
            float* lrow = p.logits + static_cast<int64_t>(U.row0 + g * RW + r) * p.ld_logits;
            __stcs(lrow + j, (j >= lo_r[r] && j < hi_r[r]) ? L[r] : -INFINITY);
          }
          if (bar_red_or(bar_id, 128, aborted || *abort_flag)) {
            aborted = true;
            break;
          }
        } else {
#pragma unroll
          for (int r = 0; r < RW; ++r) {
            const uint32_t key = order_key(L[r]);
            const bool pass = rv[r] && j >= lo_r[r] && j < hi_r[r] && key >= th_g[r];
            const uint32_t msk = __ballot_sync(0xFFFFFFFFu, pass);
            if (msk) {
              const int leader = __ffs(static_cast<int>(msk)) - 1;
              int base = 0;
              if (lane == leader) base = atomicAdd(&cnt_g[r], __popc(msk));
              base = __shfl_sync(0xFFFFFFFFu, base, leader);
              if (pass)
                cand_g[static_cast<size_t>(r) * cap + base + __popc(msk & ((1u << lane) - 1u))] =
                    make_uint2(key, static_cast<uint32_t>(j));
            }
          }
          if (bar_red_or(bar_id, 128, aborted || *abort_flag)) {
            aborted = true;
            break;
          }
          // Keep room for one more tile per row: compact rows that are near full
          // to their exact top-k; later keys only enter above the k-th value.
          bool need = false;
#pragma unroll
          for (int r = 0; r < RW; ++r) need |= cnt_g[r] > cap - kBlockKeys;
          if (need) {
            if (qd < RW && cnt_g[qd] > cap - kBlockKeys) {
              uint2* buf = cand_g + static_cast<size_t>(qd) * cap;
              const int cnt = cnt_g[qd];
              const SelectResult sel = group_select<1>(BufSrc{buf}, cnt, k, grp);
              uint32_t umin = 0xFFFFFFFFu;
              const int kept = group_emit<1>(BufSrc{buf}, cnt, sel, grp, [&](int pos, uint64_t K) {
                buf[pos] = make_uint2(composite_value(K), composite_index(K));
                umin = min(umin, composite_value(K));
              });
              umin = __reduce_min_sync(0xFFFFFFFFu, umin);
              if (lane == 0) {
                cnt_g[qd] = kept;
                if (kept >= k) th_g[qd] = max(th_g[qd], umin == 0xFFFFFFFFu ? umin : umin + 1);
              }
            }
            named_bar_sync(bar_id, 128);
          }
        }
      }
      if (aborted) break;

      if (MODE == kModeTopK) {
        // ---- exact top-k of each row's candidates
        if (qd < RW) {
          const int r = qd;
          const int rl = g * RW + r;
          const uint2* buf = cand_g + static_cast<size_t>(r) * cap;
          const int cnt = cnt_g[r];
          if (p.n_chunks == 1) {
            if (rl < U.nrows) {
              const int row = U.row0 + rl;
              int32_t* orow = p.out_idx + static_cast<int64_t>(row) * k;
              float* vrow = p.out_vals ? p.out_vals + static_cast<int64_t>(row) * k : nullptr;
              const SelectResult sel = group_select<1>(BufSrc{buf}, cnt, k, grp);
              const int nout = group_emit<1>(BufSrc{buf}, cnt, sel, grp, [&](int pos, uint64_t K) {
                orow[pos] = static_cast<int32_t>(composite_index(K));
                if (vrow) vrow[pos] = key_to_float(composite_value(K));
              });
              for (int pos = nout + lane; pos < k; pos += 32) {
                orow[pos] = -1;
                if (vrow) vrow[pos] = -INFINITY;
              }
            }
          } else {
            uint2* prow = p.part + (static_cast<size_t>(u) * R + rl) * k;
            int nout = 0;
            if (rl < U.nrows && cnt > 0) {
              const SelectResult sel = group_select<1>(BufSrc{buf}, cnt, k, grp);
              nout = group_emit<1>(BufSrc{buf}, cnt, sel, grp, [&](int pos, uint64_t K) {
                prow[pos] = make_uint2(composite_value(K), composite_index(K));
              });
            }
            if (lane == 0) p.part_cnt[static_cast<size_t>(u) * R + rl] = nout;
          }
        }
        named_bar_sync(bar_id, 128);
      }
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
    if (i >= __ldg(cnt + static_cast<size_t>(c) * cstride)) return false;
    const uint2 v = base[static_cast<size_t>(c) * stride + i];
    K = compose_key(v.x, v.y);
    return true;
  }
};

constexpr int kMergeWarps = 8;

__global__ void __launch_bounds__(kMergeWarps * 32) merge_kernel(const MergeParams p) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t red[8 * kMergeWarps];
  __shared__ uint32_t counter;
  const int row = blockIdx.x;
  const int unit_row = row / p.R;  // row block / request
  const int rl = row - unit_row * p.R;
  const size_t u0 = static_cast<size_t>(unit_row) * p.n_chunks;
  PartSrc src{p.part + (u0 * p.R + rl) * p.topk, p.part_cnt + u0 * p.R + rl,
              static_cast<size_t>(p.R) * p.topk, p.R, p.topk};
  Group<kMergeWarps> g{hist, red, &counter, 1, static_cast<int>(threadIdx.x)};
  const int total = p.n_chunks * p.topk;
  const SelectResult sel = group_select<kMergeWarps>(src, total, p.topk, g);
  int32_t* orow = p.out_idx + static_cast<int64_t>(row) * p.topk;
  float* vrow = p.out_vals ? p.out_vals + static_cast<int64_t>(row) * p.topk : nullptr;
  const int nout = group_emit<kMergeWarps>(src, total, sel, g, [&](int pos, uint64_t K) {
    orow[pos] = static_cast<int32_t>(composite_index(K));
    if (vrow) vrow[pos] = key_to_float(composite_value(K));
  });
  for (int pos = nout + threadIdx.x; pos < p.topk; pos += blockDim.x) {
    orow[pos] = -1;
    if (vrow) vrow[pos] = -INFINITY;
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

template <int R, bool PAGED, int MODE>
static cudaError_t launch_indexer(const IndexerParams& p, int grid, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(smem_layout<R, PAGED>().total) + 1024;
  auto kern = indexer_kernel<R, PAGED, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_indexer_prefill_logits(const IndexerParams& p, int grid, cudaStream_t st) {
  return launch_indexer<8, false, kModeLogits>(p, grid, st);
}
cudaError_t launch_indexer_prefill_topk(const IndexerParams& p, int grid, cudaStream_t st) {
  return launch_indexer<8, false, kModeTopK>(p, grid, st);
}
cudaError_t launch_indexer_paged_topk(const IndexerParams& p, int R, int grid, cudaStream_t st) {
  if (R == 8) return launch_indexer<8, true, kModeTopK>(p, grid, st);
  return launch_indexer<4, true, kModeTopK>(p, grid, st);
}

cudaError_t launch_merge(const MergeParams& p, cudaStream_t st) {
  merge_kernel<<<p.rows, kMergeWarps * 32, 0, st>>>(p);
  return cudaGetLastError();
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
