// pkm_select.cuh -- exact top-k over the product candidates of two sorted per-half
// lists, shared by the large-batch and small-batch gather kernels.
//
// A key's score is its left score plus its right score ("Product Keys Give
// Transformers Million-Slot Memory Layers", "Why top-k of each half is enough"); key
// (i, j) is left sub-key i joined with right sub-key j, flat slot i*n + j ("Implied
// keys vs stored sub-keys"). With both lists sorted best first, the pair at list
// positions (a, b) is beaten by every pair (a', b') with a' <= a and b' <= b, so only
// pairs with (a + 1)(b + 1) <= k can be among the best k: sum_a floor(k / (a + 1))
// candidates (119 for k = 32) instead of k^2.
#pragma once

#include "pkm_common.cuh"

namespace pkm {

// Candidate pairs (a, b) with (a+1)(b+1) <= k number at most 119 for k <= 32.
constexpr int kMaxPairs = 128;

// Fill pairs[] with a | (b << 8) for every candidate pair; returns their number. One
// thread.
__device__ __forceinline__ int build_pairs(int k, int* pairs) {
  int p = 0;
  for (int a = 0; a < k; ++a)
    for (int b = 0; (a + 1) * (b + 1) <= k; ++b) pairs[p++] = a | (b << 8);
  return p;
}

// Lane j holds entry j of the left list (s1, i1) and of the right list (s2, i2), each
// sorted best first (padding: score -inf, id kIdPad). On return lane j holds the j-th
// best candidate (score, flat slot) by (score desc, slot asc).
__device__ __forceinline__ void select_candidates(float s1, int i1, float s2, int i2,
                                                  const int* pairs, int npairs, int n,
                                                  float& bs, int& bi) {
  const int lane = threadIdx.x & 31;
  bs = -INFINITY;
  bi = kIdPad;
  for (int c0 = 0; c0 < npairs; c0 += 32) {
    const int p = c0 + lane;
    const int ab = p < npairs ? pairs[p] : 0;
    const int a = ab & 0xff, b = ab >> 8;
    const float sa = __shfl_sync(0xffffffffu, s1, a);
    const int ia = __shfl_sync(0xffffffffu, i1, a);
    const float sb = __shfl_sync(0xffffffffu, s2, b);
    const int ib = __shfl_sync(0xffffffffu, i2, b);
    // Padding ids can only surface when scores are NaN; they never form a slot.
    const bool real = p < npairs && ia >= 0 && ia < n && ib >= 0 && ib < n;
    float cs = real ? sa + sb : -INFINITY;
    int ci = real ? ia * n + ib : kIdPad;
    warp_sort32(cs, ci);
    warp_merge32(bs, bi, cs, ci);
  }
}

}  // namespace pkm
