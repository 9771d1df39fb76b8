// select.cuh -- exact top-k selection by a group of warps.
//
// The order is the indexer's: larger logit first, and among equal logits the
// lower key index first.  Each candidate becomes one 64-bit composite key
//     K = (order_key(logit) << 32) | (0xFFFFFFFF - index)
// so that "better" is simply "larger K" and all keys of a row are distinct.
// A most-significant-digit radix select (8-bit digits) finds the shortest
// prefix P of length plen such that exactly k candidates have a prefix >= P;
// it skips the leading bits that all candidates share and stops as soon as
// the bin holding the k-th candidate is taken whole.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace fp8idx {

// Monotone map float -> uint32 (a < b  <=>  key(a) < key(b)); -0 maps like +0.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  if ((b << 1) == 0) b = 0;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_to_float(uint32_t u) {
  uint32_t b = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
  return __uint_as_float(b);
}

__device__ __forceinline__ uint64_t compose_key(uint32_t u, uint32_t j) {
  return (static_cast<uint64_t>(u) << 32) | static_cast<uint64_t>(0xFFFFFFFFu - j);
}
__device__ __forceinline__ uint32_t composite_index(uint64_t K) {
  return 0xFFFFFFFFu - static_cast<uint32_t>(K);
}
__device__ __forceinline__ uint32_t composite_value(uint64_t K) {
  return static_cast<uint32_t>(K >> 32);
}

struct SelectResult {
  uint64_t prefix;  // selected iff plen == 0 or (K >> (64 - plen)) >= prefix
  int plen;
  int count;  // number of candidates seen
};

__device__ __forceinline__ bool is_selected(uint64_t K, const SelectResult& s) {
  return s.plen == 0 || (K >> (64 - s.plen)) >= s.prefix;
}

// Shared scratch of one group: hist[256] and red[8 * G] words, plus a counter.
template <int G>
struct Group {
  uint32_t* hist;
  uint32_t* red;
  uint32_t* counter;
  int bar_id;  // named barrier id (unused when G == 1)
  int tid;     // thread index inside the group, [0, 32 * G)

  __device__ __forceinline__ void sync() const {
    if (G == 1)
      __syncwarp();
    else
      named_bar_sync(bar_id, 32 * G);
  }
  __device__ __forceinline__ int lane() const { return tid & 31; }
  __device__ __forceinline__ int warp() const { return tid >> 5; }
};

// Src must provide:  __device__ bool get(int e, uint64_t& K) const;  (false: no candidate at e)
template <int G, class Src>
__device__ SelectResult group_select(const Src& src, int total, int k, const Group<G>& g) {
  const int lane = g.lane();
  // ---- pass 0: count candidates and find the bits they all share
  uint32_t cnt = 0;
  uint64_t kor = 0, kand = ~0ull;
  for (int e = g.tid; e < total; e += 32 * G) {
    uint64_t K;
    if (src.get(e, K)) {
      ++cnt;
      kor |= K;
      kand &= K;
    }
  }
  cnt = __reduce_add_sync(0xFFFFFFFFu, cnt);
  uint32_t orl = __reduce_or_sync(0xFFFFFFFFu, static_cast<uint32_t>(kor));
  uint32_t orh = __reduce_or_sync(0xFFFFFFFFu, static_cast<uint32_t>(kor >> 32));
  uint32_t anl = __reduce_and_sync(0xFFFFFFFFu, static_cast<uint32_t>(kand));
  uint32_t anh = __reduce_and_sync(0xFFFFFFFFu, static_cast<uint32_t>(kand >> 32));
  if (G > 1) {
    if (lane == 0) {
      uint32_t* r = g.red + 5 * g.warp();
      r[0] = cnt; r[1] = orl; r[2] = orh; r[3] = anl; r[4] = anh;
    }
    g.sync();
    cnt = 0; orl = 0; orh = 0; anl = ~0u; anh = ~0u;
#pragma unroll 1
    for (int w = 0; w < G; ++w) {
      const uint32_t* r = g.red + 5 * w;
      cnt += r[0]; orl |= r[1]; orh |= r[2]; anl &= r[3]; anh &= r[4];
    }
    g.sync();
  }
  SelectResult res;
  res.count = static_cast<int>(cnt);
  res.prefix = 0;
  res.plen = 0;
  if (static_cast<int>(cnt) <= k) return res;  // everything is selected

  const uint64_t kor_all = (static_cast<uint64_t>(orh) << 32) | orl;
  const uint64_t kand_all = (static_cast<uint64_t>(anh) << 32) | anl;
  int plen = __clzll(static_cast<long long>(kor_all ^ kand_all));  // < 64: keys are distinct
  uint64_t prefix = plen ? (kand_all >> (64 - plen)) : 0;
  uint32_t need = static_cast<uint32_t>(k);

  while (true) {
    const int dbits = (64 - plen) < 8 ? (64 - plen) : 8;
    const int shift = 64 - plen - dbits;
    const uint64_t dmask = (1ull << dbits) - 1;
    for (int i = g.tid; i < 256; i += 32 * G) g.hist[i] = 0;
    g.sync();
    for (int e = g.tid; e < total; e += 32 * G) {
      uint64_t K;
      if (src.get(e, K) && (plen == 0 || (K >> (64 - plen)) == prefix))
        atomicAdd(&g.hist[(K >> shift) & dmask], 1u);
    }
    g.sync();
    // Every warp finds the digit redundantly: lane l owns bins [8l, 8l + 8).
    uint32_t b[8];
    uint32_t tot = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      b[i] = g.hist[lane * 8 + i];
      tot += b[i];
    }
    uint32_t suf = tot;  // inclusive suffix sum over lanes >= lane
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      uint32_t t = __shfl_down_sync(0xFFFFFFFFu, suf, off);
      if (lane + off < 32) suf += t;
    }
    const uint32_t ball = __ballot_sync(0xFFFFFFFFu, suf >= need);
    const int lstar = 31 - __clz(static_cast<int>(ball));
    uint32_t dstar = 0, above = 0, inbin = 0;
    if (lane == lstar) {
      uint32_t run = suf - tot;
#pragma unroll
      for (int i = 7; i >= 0; --i) {
        if (run + b[i] >= need) {
          dstar = static_cast<uint32_t>(lane * 8 + i);
          inbin = b[i];
          break;
        }
        run += b[i];
      }
      above = run;
    }
    dstar = __shfl_sync(0xFFFFFFFFu, dstar, lstar);
    above = __shfl_sync(0xFFFFFFFFu, above, lstar);
    inbin = __shfl_sync(0xFFFFFFFFu, inbin, lstar);
    g.sync();  // everyone has read hist before the next pass clears it
    prefix = (prefix << dbits) | dstar;
    plen += dbits;
    need -= above;
    if (inbin == need || plen >= 64) break;
  }
  res.prefix = prefix;
  res.plen = plen;
  return res;
}

// Calls emit(pos, K) for every selected candidate, pos in [0, min(k, count)).
// Positions are handed out in the order a single warp meets the candidates
// (so with G == 1 a candidate never moves to a higher position, which makes
// in-place compaction safe).  Returns the number emitted.
template <int G, class Src, class Emit>
__device__ int group_emit(const Src& src, int total, const SelectResult& sel, const Group<G>& g,
                          Emit emit) {
  const int lane = g.lane();
  if (g.tid == 0) *g.counter = 0;
  g.sync();
  for (int base = 0; base < total; base += 32 * G) {
    const int e = base + g.tid;
    uint64_t K = 0;
    const bool ok = e < total && src.get(e, K) && is_selected(K, sel);
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, ok);
    if (m) {
      const int leader = __ffs(static_cast<int>(m)) - 1;
      uint32_t pos0 = 0;
      if (lane == leader) pos0 = atomicAdd(g.counter, static_cast<uint32_t>(__popc(m)));
      pos0 = __shfl_sync(0xFFFFFFFFu, pos0, leader);
      if (ok) emit(static_cast<int>(pos0 + __popc(m & ((1u << lane) - 1u))), K);
    }
  }
  g.sync();
  const int n = static_cast<int>(*g.counter);
  g.sync();
  return n;
}

}  // namespace fp8idx
