// One token's top-k selection over its expert logits, done by one warp.
// Used by the forward's routers and by the allocation-free router, so that
// both pick the same experts.
#pragma once

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

namespace moe {

constexpr int kTopkMaxExperts = 256;
constexpr int kTopkPerLane = kTopkMaxExperts / 32;

// Total order of the selection: larger logit first, then lower index.
__device__ __forceinline__ bool topk_better(float va, int ea, float vb, int eb) {
  return va > vb || (va == vb && ea < eb);
}

struct TopkResult {
  int my_e;     // lane i < k: the i-th chosen expert
  float my_p;   // lane i < k: its softmax probability over all experts
  float psum;   // sum of the k chosen probabilities (every lane)
};

// lgt[0..E): the token's logits (shared memory), k <= E <= 256. Softmax over
// all E experts, then the k largest logits, equal logits to the lower expert
// index. A NaN logit (from a NaN or infinite input row) ranks as -inf, and an
// expert is chosen at most once, so the k ids are always distinct and in
// [0, E) whatever the values; the weights of such a token are then NaN.
__device__ __forceinline__ TopkResult topk_warp(const float* lgt, int E, int k, int lane) {
  float v[kTopkPerLane];
#pragma unroll
  for (int j = 0; j < kTopkPerLane; ++j) {
    const int e = lane + 32 * j;
    const float l = e < E ? lgt[e] : -INFINITY;
    v[j] = isnan(l) ? -INFINITY : l;
  }
  float mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < kTopkPerLane; ++j) mx = fmaxf(mx, v[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float z = 0.f;
#pragma unroll
  for (int j = 0; j < kTopkPerLane; ++j)
    if (lane + 32 * j < E) z += expf(v[j] - mx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);

  TopkResult r{-1, 0.f, 0.f};
  uint32_t taken = 0;  // bit j: expert lane + 32 j already chosen
  for (int i = 0; i < k; ++i) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < kTopkPerLane; ++j) {
      const int e = lane + 32 * j;
      if (e < E && !((taken >> j) & 1u) && topk_better(v[j], e, bv, be)) {
        bv = v[j];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (topk_better(ov, oe, bv, be)) {
        bv = ov;
        be = oe;
      }
    }
    // an untaken expert with a value >= -inf always exists (k <= E), so be
    // is valid; the clamp only guards the indexing that follows
    be = min(max(be, 0), E - 1);
#pragma unroll
    for (int j = 0; j < kTopkPerLane; ++j)
      if (lane + 32 * j == be) taken |= 1u << j;
    const float p = expf(bv - mx) / z;
    r.psum += p;
    if (lane == i) {
      r.my_e = be;
      r.my_p = p;
    }
  }
  return r;
}

}  // namespace moe
