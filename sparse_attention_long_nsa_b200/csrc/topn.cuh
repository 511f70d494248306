// Warp-level top-n block selection for one (query position, KV head).
//
// Candidates are blocks 0..jt (jt = t / l'). When all fit in top_n they are all
// taken; otherwise the first `ff` blocks and the `fl` blocks ending at jt are
// forced and the remaining top_n - ff - fl slots go to the highest scores, ties
// to the lower block index ("Разреженное внимание — NSA и DSA", ai.flicky.cc,
// section "NSA: три ветви", selection branch). The threshold is found by a
// 32-step radix select over the order-preserving bit pattern of the scores;
// ties are taken in index order with ballots; the output is ascending and
// padded with -1.
#pragma once

#include "common.cuh"

namespace nsa {

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// All 32 lanes call it. imp: scores of blocks 0..jt (generic pointer).
template <int PER>
__device__ __forceinline__ void warp_topn(const float* imp, int jt, int top_n, int ff, int fl, int32_t* out,
                                          int lane) {
  const int K = jt + 1;
  if (K <= top_n) {
    for (int i = lane; i < top_n; i += 32) out[i] = i < K ? i : -1;
    return;
  }
  const int need = top_n - ff - fl;   // K > top_n >= ff + fl: forced sets are disjoint
  uint32_t key[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int j = i * 32 + lane;
    const bool cand = j < K && j >= ff && j <= jt - fl;
    key[i] = cand ? order_key(imp[j]) : 0u;   // 0 sorts below every real score
  }
  uint32_t x = 0;   // need-th largest candidate key
  if (need > 0) {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t y = x | (1u << bit);
      int c = 0;
#pragma unroll
      for (int i = 0; i < PER; ++i) c += key[i] >= y;
      c = __reduce_add_sync(0xffffffffu, c);
      if (c >= need) x = y;
    }
  }
  int gt = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) gt += (need > 0) && key[i] > x;
  gt = __reduce_add_sync(0xffffffffu, gt);
  int ties_left = need - gt;
  int pos = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int j = i * 32 + lane;
    const bool forced = j < K && (j < ff || j > jt - fl);
    const bool eq = need > 0 && key[i] == x && key[i] != 0u;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const int before = __popc(eqm & ((1u << lane) - 1u));
    const bool take_eq = eq && before < ties_left;
    ties_left -= min(__popc(eqm), max(ties_left, 0));
    const bool chosen = forced || (need > 0 && key[i] > x) || take_eq;
    const uint32_t cm = __ballot_sync(0xffffffffu, chosen);
    if (chosen) out[pos + __popc(cm & ((1u << lane) - 1u))] = j;
    pos += __popc(cm);
  }
  for (int i = pos + lane; i < top_n; i += 32) out[i] = -1;
}

// Same selection for any jt, reading the scores from memory on every pass
// instead of holding them in registers (used beyond 1024 candidate blocks).
__device__ __forceinline__ void warp_topn_mem(const float* imp, int jt, int top_n, int ff, int fl, int32_t* out,
                                              int lane) {
  const int K = jt + 1;
  if (K <= top_n) {
    for (int i = lane; i < top_n; i += 32) out[i] = i < K ? i : -1;
    return;
  }
  const int need = top_n - ff - fl;
  auto key_of = [&](int j) -> uint32_t {
    const bool cand = j < K && j >= ff && j <= jt - fl;
    return cand ? order_key(imp[j]) : 0u;
  };
  uint32_t x = 0;
  if (need > 0) {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t y = x | (1u << bit);
      int c = 0;
      for (int j = lane; j < K; j += 32) c += key_of(j) >= y;
      c = __reduce_add_sync(0xffffffffu, c);
      if (c >= need) x = y;
    }
  }
  int gt = 0;
  for (int j = lane; j < K; j += 32) gt += (need > 0) && key_of(j) > x;
  gt = __reduce_add_sync(0xffffffffu, gt);
  int ties_left = need - gt;
  int pos = 0;
  for (int j0 = 0; j0 < K; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < K ? key_of(j) : 0u;
    const bool forced = j < K && (j < ff || j > jt - fl);
    const bool eq = need > 0 && key == x && key != 0u;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const int before = __popc(eqm & ((1u << lane) - 1u));
    const bool take_eq = eq && before < ties_left;
    ties_left -= min(__popc(eqm), max(ties_left, 0));
    const bool chosen = forced || (need > 0 && key > x) || take_eq;
    const uint32_t cm = __ballot_sync(0xffffffffu, chosen);
    if (chosen) out[pos + __popc(cm & ((1u << lane) - 1u))] = j;
    pos += __popc(cm);
  }
  for (int i = pos + lane; i < top_n; i += 32) out[i] = -1;
}

}  // namespace nsa
