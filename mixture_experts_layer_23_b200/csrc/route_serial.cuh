// Softmax + top-k of one token, computed serially by one thread over its E logits in increasing
// expert order.  Every router entry point uses this routine, so identical logits give identical
// expert ids and gate weights whichever entry point produced them.
//
// Top-k gate of tutorial ch.4 "分布式训练", section "框架" (Tutel gate_type {'type': 'top', 'k'}):
// the k largest logits, best first; equal logits go to the lower expert index.  Gate weights:
// gate_norm 0 -> softmax over all E logits read at the chosen experts; gate_norm 1 -> softmax over
// the k chosen logits only.
#pragma once
#include <math.h>
#include <stdint.h>

namespace moe {

struct TopK8 {
  float v[8];  // best logits so far, descending; ties keep the earlier (lower) expert first
  int e[8];
  float m;     // running max of all logits (online softmax)
  float s;     // running sum of exp(logit - m)
};

__device__ __forceinline__ void topk_init(TopK8& t) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    t.v[j] = -INFINITY;
    t.e[j] = 0x7fffffff;
  }
  t.m = -INFINITY;
  t.s = 0.f;
}

// Feed logit v of expert e; experts must arrive in increasing index order.
__device__ __forceinline__ void topk_push(TopK8& t, float v, int e) {
  if (v > t.m) {
    t.s = t.s * expf(t.m - v) + 1.f;
    t.m = v;
  } else {
    t.s += expf(v - t.m);
  }
  if (v > t.v[7]) {
    // insert at the first slot holding a strictly smaller logit (an equal, earlier expert stays
    // ahead) and shift the tail down by one; walking from the end reads only unmodified slots
#pragma unroll
    for (int j = 7; j > 0; --j) {
      if (v > t.v[j - 1]) {
        t.v[j] = t.v[j - 1];
        t.e[j] = t.e[j - 1];
      } else if (v > t.v[j]) {
        t.v[j] = v;
        t.e[j] = e;
      }
    }
    if (v > t.v[0]) {
      t.v[0] = v;
      t.e[0] = e;
    }
  }
}

__device__ __forceinline__ void topk_finish(const TopK8& t, int k, int gate_norm,
                                            int32_t* __restrict__ idx_out,
                                            float* __restrict__ w_out) {
  if (gate_norm == 0) {
    const float inv = 1.f / t.s;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < k) {
        idx_out[j] = t.e[j];
        w_out[j] = expf(t.v[j] - t.m) * inv;
      }
  } else {
    float z = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < k) z += expf(t.v[j] - t.v[0]);
    const float inv = 1.f / z;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < k) {
        idx_out[j] = t.e[j];
        w_out[j] = expf(t.v[j] - t.v[0]) * inv;
      }
  }
}

}  // namespace moe
