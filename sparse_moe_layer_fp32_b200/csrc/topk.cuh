// Warp-level top-k of one token's logits with the renormalised softmax weights.
#pragma once

#include "common.cuh"

namespace beam {

// Order-preserving map of an FP32 value to an unsigned key (larger value -> larger key);
// every finite value and -inf map above 0, which marks "not a candidate".
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// v: this lane's logits, expert e = lane + 32 i (entries with e >= E are ignored).
// k rounds of a warp arg-max (larger logit first, equal logits -> lower expert index): a
// warp max of the keys, then one ballot per register slot finds the lowest expert holding
// it.  softmax is monotone, so these are the top-k of the softmax, and the renormalised
// weights p_j / sum_chosen p equal a softmax over the chosen logits.  Lane j < k ends up
// holding slot j and writes ids[j] / wout[j] (descending weight).
template <int EPL>
__device__ __forceinline__ void warp_topk(const float (&v)[EPL], int E, int k, int lane, int32_t* ids,
                                          float* wout) {
  uint32_t key[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) key[i] = lane + 32 * i < E ? order_key(v[i]) : 0u;
  int my_e = 0;
  float my_v = 0.0f, v0 = 0.0f;
  for (int j = 0; j < k; ++j) {
    uint32_t m = key[0];
#pragma unroll
    for (int i = 1; i < EPL; ++i) m = max(m, key[i]);
    const uint32_t top = __reduce_max_sync(0xffffffffu, m);
    int best = 0;
#pragma unroll
    for (int i = EPL - 1; i >= 0; --i) {  // the lowest slot (then lane) that holds the maximum
      const uint32_t b = __ballot_sync(0xffffffffu, key[i] == top);
      if (b) best = 32 * i + __ffs(b) - 1;
    }
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if (best == lane + 32 * i) key[i] = 0u;
    const float val = key_value(top);
    if (j == 0) v0 = val;
    if (lane == j) {
      my_e = best;
      my_v = val;
    }
  }
  const float z = lane < k ? expf(my_v - v0) : 0.0f;
  float sum = z;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < k) {
    ids[lane] = my_e;
    wout[lane] = z / sum;
  }
}

}  // namespace beam
