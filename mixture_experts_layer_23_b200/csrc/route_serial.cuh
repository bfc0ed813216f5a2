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

// The KS best logits so far (KS >= k; the first k entries do not depend on KS, so a caller that
// knows k at compile time keeps only that many slots and shortens every insertion).
template <int KS>
struct TopK {
  float v[KS];  // descending; ties keep the earlier (lower) expert first
  int e[KS];
};
using TopK8 = TopK<8>;

template <int KS>
__device__ __forceinline__ void topk_init(TopK<KS>& t) {
#pragma unroll
  for (int j = 0; j < KS; ++j) {
    t.v[j] = -INFINITY;
    t.e[j] = 0x7fffffff;
  }
}

// Feed logit v of expert e; experts must arrive in increasing index order.
template <int KS>
__device__ __forceinline__ void topk_push(TopK<KS>& t, float v, int e) {
  if (v > t.v[KS - 1]) {
    // insert at the first slot holding a strictly smaller logit (an equal, earlier expert stays
    // ahead) and shift the tail down by one; walking from the end reads only unmodified slots
#pragma unroll
    for (int j = KS - 1; j > 0; --j) {
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

// The softmax over all E logits is taken in two passes: the top-k pass above finds the largest
// logit (t.v[0]), and a second pass adds exp(l - t.v[0]) over the logits in increasing expert
// order.  The exponentials of that pass do not depend on one another, so they overlap; an online
// softmax inside the top-k pass would put one exponential per expert on a serial chain.
template <int KS>
__device__ __forceinline__ float softmax_term(const TopK<KS>& t, float l) {
  return expf(l - t.v[0]);
}

// Gate weights of the k best experts.  gate_norm 0: softmax over all E logits, `den` being the
// sum of softmax_term over them (in increasing expert order); gate_norm 1: softmax over the k
// chosen logits only (`den` unused).
template <int KS>
__device__ __forceinline__ void topk_finish(const TopK<KS>& t, int k, int gate_norm, float den,
                                            int32_t* __restrict__ idx_out,
                                            float* __restrict__ w_out) {
  if (gate_norm == 0) {
    const float inv = 1.f / den;
#pragma unroll
    for (int j = 0; j < KS; ++j)
      if (j < k) {
        idx_out[j] = t.e[j];
        w_out[j] = expf(t.v[j] - t.v[0]) * inv;
      }
  } else {
    float z = 0.f;
#pragma unroll
    for (int j = 0; j < KS; ++j)
      if (j < k) z += expf(t.v[j] - t.v[0]);
    const float inv = 1.f / z;
#pragma unroll
    for (int j = 0; j < KS; ++j)
      if (j < k) {
        idx_out[j] = t.e[j];
        w_out[j] = expf(t.v[j] - t.v[0]) * inv;
      }
  }
}

}  // namespace moe
