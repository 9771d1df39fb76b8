// quant.cu -- key quantisation into the paged key pool (sm_100a).
//
// The producer side of the paged keys: the `act_quant` step and the fp8
// k-pool stores named on the "Serve GLM-5.3-Flash on SM80" page (commit
// notes).  For each bf16 key row x[t, 0:128]:
//   s_t   = max(max_d |x[t,d]|, 1e-4) / 448            (fp32)
//   q_t,d = e4m3(x[t,d] / s_t), nearest even, saturating at +-448
// and the codes and the scale go to pool slot slot[t] (page slot / 64, row
// slot % 64).  A slot outside [0, num_slots) is not stored.  NaN elements
// are left out of the row maximum and get a NaN code (0x7F or 0xFF).
//
// One warp per 4 tokens: each lane first loads 4 bf16 (8 bytes) of each of
// the 4 rows, so that a warp has 1 KB in flight (the rows are read in
// coalesced 256-byte passes); then per row the warp reduces |x| to the row
// maximum with one redux, each lane converts its 4 quotients with two packed
// cvt.e4m3x2 and stores 4 code bytes, and lane 0 stores the scale.  The
// kernel is a plain HBM stream (256 B read, 132 B written per token).
#include <cstdint>

#include "ptx.cuh"

namespace fp8idx {

namespace {

constexpr int kQuantWarps = 8;   // warps per CTA
constexpr int kTokPerWarp = 4;   // tokens per warp, loaded together

__device__ __forceinline__ uint16_t e4m3x2_rn_sat(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint32_t abs_bits_no_nan(float f) {
  const uint32_t b = __float_as_uint(f) & 0x7FFFFFFFu;
  return b > 0x7F800000u ? 0u : b;
}

__global__ void __launch_bounds__(kQuantWarps * 32)
    act_quant_store_kernel(const uint16_t* __restrict__ x, int64_t T, const int64_t* __restrict__ slot,
                           int64_t num_slots, uint8_t* __restrict__ k_pool, float* __restrict__ s_pool) {
  const int64_t t0 = (static_cast<int64_t>(blockIdx.x) * kQuantWarps + (threadIdx.x >> 5)) * kTokPerWarp;
  const int lane = threadIdx.x & 31;
  uint2 raw[kTokPerWarp];
  int64_t sl[kTokPerWarp];
#pragma unroll
  for (int i = 0; i < kTokPerWarp; ++i) {
    const int64_t t = t0 + i;
    sl[i] = t < T ? __ldg(slot + t) : -1;
    raw[i] = t < T ? __ldg(reinterpret_cast<const uint2*>(x + t * 128) + lane) : make_uint2(0u, 0u);
  }
#pragma unroll
  for (int i = 0; i < kTokPerWarp; ++i) {
    if (sl[i] < 0 || sl[i] >= num_slots) continue;  // the same for the whole warp
    const float f0 = __uint_as_float(raw[i].x << 16), f1 = __uint_as_float(raw[i].x & 0xFFFF0000u);
    const float f2 = __uint_as_float(raw[i].y << 16), f3 = __uint_as_float(raw[i].y & 0xFFFF0000u);
    // |x| as bits: non-negative floats order like their bit patterns; a NaN
    // (bits above +inf's) counts as 0, so the row maximum is over the rest
    uint32_t a = max(max(abs_bits_no_nan(f0), abs_bits_no_nan(f1)), max(abs_bits_no_nan(f2), abs_bits_no_nan(f3)));
    a = __reduce_max_sync(0xFFFFFFFFu, a);
    const float sc = fmaxf(__uint_as_float(a), 1e-4f) / 448.0f;
    const uint32_t lo = e4m3x2_rn_sat(f0 / sc, f1 / sc);
    const uint32_t hi = e4m3x2_rn_sat(f2 / sc, f3 / sc);
    reinterpret_cast<uint32_t*>(k_pool + sl[i] * 128)[lane] = lo | (hi << 16);
    if (lane == 0) s_pool[sl[i]] = sc;
  }
}

}  // namespace

cudaError_t launch_act_quant_store(const uint16_t* x, int64_t T, const int64_t* slot, int64_t num_slots,
                                   uint8_t* k_pool, float* s_pool, cudaStream_t st) {
  const int64_t per_cta = static_cast<int64_t>(kQuantWarps) * kTokPerWarp;
  const int64_t blocks = (T + per_cta - 1) / per_cta;
  act_quant_store_kernel<<<static_cast<unsigned>(blocks), kQuantWarps * 32, 0, st>>>(x, T, slot, num_slots,
                                                                                     k_pool, s_pool);
  return cudaGetLastError();
}

}  // namespace fp8idx
