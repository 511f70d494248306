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

// All 32 lanes call it. imp: scores of blocks 0..jt (generic pointer). The free
// slots are filled in top_n - ff - fl rounds of a warp arg-max: each round takes
// the largest remaining score (the lowest block index among equal ones), marks
// it in a per-lane bitmask and removes it; the marked and forced blocks are then
// written in ascending order.
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
  uint32_t chosen = 0u;   // bit i: block i*32 + lane taken
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int j = i * 32 + lane;
    const bool cand = j < K && j >= ff && j <= jt - fl;
    const bool forced = j < K && (j < ff || j > jt - fl);
    key[i] = cand ? order_key(imp[j]) : 0u;   // every real score maps above 0
    if (forced) chosen |= 1u << i;
  }
  // (up to 8 scores per lane the scans are short chains; above that they are
  // split into 8 independent chains joined by a tree)
  constexpr int NP = PER <= 8 ? 1 : 8;
  for (int round = 0; round < need; ++round) {
    uint32_t part[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) part[p] = key[p];
#pragma unroll
    for (int i = NP; i < PER; ++i) part[i % NP] = max(part[i % NP], key[i]);
#pragma unroll
    for (int w = NP / 2; w >= 1; w >>= 1)
#pragma unroll
      for (int p = 0; p < w; ++p) part[p] = max(part[p], part[p + w]);
    const uint32_t M = __reduce_max_sync(0xffffffffu, part[0]);
    uint32_t eq[NP];   // bit i: key[i] == M
#pragma unroll
    for (int p = 0; p < NP; ++p) eq[p] = 0u;
#pragma unroll
    for (int i = 0; i < PER; ++i) eq[i % NP] |= (key[i] == M ? 1u : 0u) << i;
#pragma unroll
    for (int w = NP / 2; w >= 1; w >>= 1)
#pragma unroll
      for (int p = 0; p < w; ++p) eq[p] |= eq[p + w];
    // this lane's lowest block holding M, then the lowest over the warp
    const uint32_t li = eq[0] ? (uint32_t)((__ffs(eq[0]) - 1) * 32 + lane) : 0xffffffffu;
    const uint32_t jmin = __reduce_min_sync(0xffffffffu, li);
    const uint32_t take = (lane == (int)(jmin & 31u)) ? (1u << (jmin >> 5)) : 0u;
    chosen |= take;
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if ((take >> i) & 1u) key[i] = 0u;
  }
  int pos = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const bool c = (chosen >> i) & 1u;
    const uint32_t cm = __ballot_sync(0xffffffffu, c);
    if (c) out[pos + __popc(cm & ((1u << lane) - 1u))] = i * 32 + lane;
    pos += __popc(cm);
  }
  for (int i = pos + lane; i < top_n; i += 32) out[i] = -1;
}

// Same selection with the scores in registers (PER per lane, block i*32 + lane in
// key[i]) and the threshold found by a 32-step radix search over the order keys
// instead of arg-max rounds: every step counts the keys at or above a candidate
// threshold with one warp reduction, so the chain is 32 short steps whatever the
// number of free slots. Then every key above the threshold and the first equal
// ones in block order are taken (ties to the lower index), output ascending.
template <int PER>
__device__ __forceinline__ void warp_topn_radix(const float* imp, int jt, int top_n, int ff, int fl, int32_t* out,
                                                int lane) {
  const int K = jt + 1;
  if (K <= top_n) {
    for (int i = lane; i < top_n; i += 32) out[i] = i < K ? i : -1;
    return;
  }
  const int need = top_n - ff - fl;   // K > top_n >= ff + fl: forced sets are disjoint
  uint32_t key[PER];
  uint32_t forced = 0u;   // bit i: block i*32 + lane is forced
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int j = i * 32 + lane;
    const bool cand = j < K && j >= ff && j <= jt - fl;
    key[i] = cand ? order_key(imp[j]) : 0u;   // every real score maps above 0
    if (j < K && (j < ff || j > jt - fl)) forced |= 1u << i;
  }
  uint32_t x = 0u;   // the need-th largest key
  if (need > 0) {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t y = x | (1u << bit);
      int c = 0;
#pragma unroll
      for (int i = 0; i < PER; ++i) c += key[i] >= y ? 1 : 0;
      if ((int)__reduce_add_sync(0xffffffffu, (uint32_t)c) >= need) x = y;
    }
  }
  int gt = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) gt += (need > 0 && key[i] > x) ? 1 : 0;
  int ties_left = need - (int)__reduce_add_sync(0xffffffffu, (uint32_t)gt);
  int pos = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const bool eq = need > 0 && key[i] == x && key[i] != 0u;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const bool take_eq = eq && __popc(eqm & ((1u << lane) - 1u)) < ties_left;
    ties_left -= min(__popc(eqm), max(ties_left, 0));
    const bool chosen = ((forced >> i) & 1u) || (need > 0 && key[i] > x) || take_eq;
    const uint32_t cm = __ballot_sync(0xffffffffu, chosen);
    if (chosen) out[pos + __popc(cm & ((1u << lane) - 1u))] = i * 32 + lane;
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

// Dispatch on the number of candidates 0..jt (register version up to 1024).
__device__ __forceinline__ void warp_topn_any(const float* imp, int jt, int top_n, int ff, int fl, int32_t* out,
                                              int lane) {
  const int per = (jt + 32) / 32;
  if (per <= 1) warp_topn<1>(imp, jt, top_n, ff, fl, out, lane);
  else if (per <= 2) warp_topn<2>(imp, jt, top_n, ff, fl, out, lane);
  else if (per <= 4) warp_topn<4>(imp, jt, top_n, ff, fl, out, lane);
  else if (per <= 8) warp_topn<8>(imp, jt, top_n, ff, fl, out, lane);
  else if (per <= 16) warp_topn_radix<16>(imp, jt, top_n, ff, fl, out, lane);
  else if (per <= 32) warp_topn_radix<32>(imp, jt, top_n, ff, fl, out, lane);
  else warp_topn_mem(imp, jt, top_n, ff, fl, out, lane);
}

// Ascending bitonic sort of one int per lane across the warp.
__device__ __forceinline__ int warp_sort_asc(int v, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j >= 1; j >>= 1) {
      const int o = __shfl_xor_sync(0xffffffffu, v, j);
      const bool up = (lane & k) == 0;          // direction of this k-block
      const bool lower = (lane & j) == 0;       // this lane keeps the smaller of the pair when up
      v = (lower == up) ? min(v, o) : max(v, o);
    }
  }
  return v;
}

// Best `need` free candidates of one slice of blocks, by warp arg-max rounds
// (ties to the lower block index). Writes round r's (key, block) to ck[r], ci[r];
// key 0 once the slice has no candidate left.
template <int PER>
__device__ __forceinline__ void slice_best(const float* imp, int lo, int hi, int ff, int last_free, int need,
                                           uint32_t* ck, int* ci, int lane) {
  uint32_t key[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int j = lo + i * 32 + lane;
    key[i] = (j < hi && j >= ff && j <= last_free) ? order_key(imp[j]) : 0u;
  }
  for (int round = 0; round < need; ++round) {
    uint32_t m = key[0];
#pragma unroll
    for (int i = 1; i < PER; ++i) m = max(m, key[i]);
    const uint32_t M = __reduce_max_sync(0xffffffffu, m);
    uint32_t eq = 0u;
#pragma unroll
    for (int i = 0; i < PER; ++i) eq |= (key[i] == M ? 1u : 0u) << i;
    const uint32_t li = eq ? (uint32_t)((__ffs(eq) - 1) * 32 + lane) : 0xffffffffu;
    const uint32_t pmin = __reduce_min_sync(0xffffffffu, li);   // lowest position = lowest block
    if (lane == (int)(pmin & 31u)) {
      const int i0 = (int)(pmin >> 5);
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (i == i0) key[i] = 0u;
    }
    if (lane == 0) {
      ck[round] = M;
      ci[round] = M ? lo + (int)pmin : 0x7fffffff;
    }
  }
}

// CTA-wide selection with the same result as warp_topn (block 0 .. ff-1 and the
// fl blocks ending at jt forced; the other top_n - ff - fl slots to the highest
// scores, ties to the lower index; ascending, -1 padded). Each of the nw warps
// picks the best candidates of its slice of the blocks, then warp 0 picks among
// those (a block in the overall best set is among the best of its own slice).
// ck/ci: shared scratch of nw * 32 entries each. Every thread of the CTA calls it
// (it synchronises the CTA); returns false when the candidates do not fit
// (more than nw * 512 blocks), and then writes nothing.
__device__ inline bool cta_topn(const float* imp, int jt, int top_n, int ff, int fl, int32_t* out, uint32_t* ck,
                                int* ci, int nw, int warp, int lane) {
  const int K = jt + 1;
  if (K <= top_n) {
    if (warp == 0)
      for (int i = lane; i < top_n; i += 32) out[i] = i < K ? i : -1;
    return true;
  }
  const int per = (K + 32 * nw - 1) / (32 * nw);
  if (per > 16) return false;
  const int need = top_n - ff - fl;
  const int pw = per <= 1 ? 1 : per <= 2 ? 2 : per <= 4 ? 4 : per <= 8 ? 8 : 16;
  const int lo = warp * 32 * pw, hi = min(K, lo + 32 * pw);
  if (warp < nw && lo < K && need > 0) {
    uint32_t* wk = ck + warp * 32;
    int* wi = ci + warp * 32;
    switch (pw) {
      case 1: slice_best<1>(imp, lo, hi, ff, jt - fl, need, wk, wi, lane); break;
      case 2: slice_best<2>(imp, lo, hi, ff, jt - fl, need, wk, wi, lane); break;
      case 4: slice_best<4>(imp, lo, hi, ff, jt - fl, need, wk, wi, lane); break;
      case 8: slice_best<8>(imp, lo, hi, ff, jt - fl, need, wk, wi, lane); break;
      default: slice_best<16>(imp, lo, hi, ff, jt - fl, need, wk, wi, lane); break;
    }
  }
  __syncthreads();
  if (warp == 0) {
    const int nsl = (K + 32 * pw - 1) / (32 * pw);   // slices that ran
    // lane l holds entry r = l of every slice: key k[w], block b[w]
    uint32_t k[8];
    int bidx[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const bool v = w < nsl && lane < need;
      k[w] = v ? ck[w * 32 + lane] : 0u;
      bidx[w] = v ? ci[w * 32 + lane] : 0x7fffffff;
    }
    int mine = 0x7fffffff;   // block chosen in round `lane`
    for (int round = 0; round < need; ++round) {
      uint32_t m = 0u;
#pragma unroll
      for (int w = 0; w < 8; ++w) m = max(m, k[w]);
      const uint32_t M = __reduce_max_sync(0xffffffffu, m);
      int bm = 0x7fffffff;
#pragma unroll
      for (int w = 0; w < 8; ++w)
        if (k[w] == M) bm = min(bm, bidx[w]);
      const int B = (int)__reduce_min_sync(0xffffffffu, (uint32_t)bm);
#pragma unroll
      for (int w = 0; w < 8; ++w)
        if (bidx[w] == B) k[w] = 0u;
      if (lane == round) mine = B;
    }
    // forced blocks in the lanes after the chosen ones
    const int f = lane - need;
    if (f >= 0 && f < ff) mine = f;
    if (f >= ff && f < ff + fl) mine = jt - fl + 1 + (f - ff);
    const int v = warp_sort_asc(mine, lane);
    if (lane < top_n) out[lane] = v == 0x7fffffff ? -1 : v;
  }
  return true;
}

}  // namespace nsa
