// Warp-level top-k of one token's logits with the renormalised softmax weights.
#pragma once

#include "common.cuh"

namespace beam {

// v: this lane's logits, expert e = lane + 32 i (entries with e >= E are ignored).
// k rounds of a warp arg-max (larger logit first, equal logits -> lower expert index);
// softmax is monotone, so these are the top-k of the softmax, and the renormalised weights
// p_j / sum_chosen p equal a softmax over the chosen logits.  Lanes j < k write slot j of
// ids / wout (descending weight).
template <int EPL>
__device__ __forceinline__ void warp_topk(const float (&v)[EPL], int E, int k, int lane, int32_t* ids,
                                          float* wout) {
  uint32_t taken = 0;
  float sel_v[16];
  int sel_e[16];
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (!((taken >> i) & 1u) && e < E && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    sel_v[j] = bv;
    sel_e[j] = be;
  }
  float z[16], sum = 0.0f;
  for (int j = 0; j < k; ++j) {
    z[j] = expf(sel_v[j] - sel_v[0]);
    sum += z[j];
  }
  for (int j = lane; j < k; j += 32) {
    ids[j] = sel_e[j];
    wout[j] = z[j] / sum;
  }
}

}  // namespace beam
