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
// Each lane first sorts its EPL candidates (descending key, equal keys keep the lower
// expert first); then k rounds take the warp maximum of the lanes' heads, the lowest
// expert index among the heads equal to it wins (equal logits -> lower expert index), and
// the winning lane pops its head.  softmax is monotone, so these are the top-k of the
// softmax, and the renormalised weights p_j / sum_chosen p equal a softmax over the chosen
// logits.  Lane j < k ends up holding slot j and writes ids[j] / wout[j] (descending
// weight).
template <int EPL>
__device__ __forceinline__ void warp_topk(const float (&v)[EPL], int E, int k, int lane, int32_t* ids,
                                          float* wout) {
  uint32_t key[EPL];
  int idx[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    idx[i] = lane + 32 * i;
    key[i] = idx[i] < E ? order_key(v[i]) : 0u;
  }
  // odd-even transposition sort; a swap needs a strictly larger key, so it is stable
#pragma unroll
  for (int p = 0; p < EPL; ++p) {
#pragma unroll
    for (int i = p & 1; i + 1 < EPL; i += 2) {
      const bool sw = key[i + 1] > key[i];
      const uint32_t ka = sw ? key[i + 1] : key[i], kb = sw ? key[i] : key[i + 1];
      const int ia = sw ? idx[i + 1] : idx[i], ib = sw ? idx[i] : idx[i + 1];
      key[i] = ka;
      key[i + 1] = kb;
      idx[i] = ia;
      idx[i + 1] = ib;
    }
  }
  int my_e = 0;
  float my_v = 0.0f, v0 = 0.0f;
  for (int j = 0; j < k; ++j) {
    const uint32_t top = __reduce_max_sync(0xffffffffu, key[0]);
    const uint32_t best = __reduce_min_sync(0xffffffffu, key[0] == top ? static_cast<uint32_t>(idx[0]) : 0xffffffffu);
    if (key[0] == top && static_cast<uint32_t>(idx[0]) == best) {  // pop the head
#pragma unroll
      for (int i = 0; i + 1 < EPL; ++i) {
        key[i] = key[i + 1];
        idx[i] = idx[i + 1];
      }
      key[EPL - 1] = 0u;
    }
    const float val = key_value(top);
    if (j == 0) v0 = val;
    if (lane == j) {
      my_e = static_cast<int>(best);
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
