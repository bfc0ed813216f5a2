// Host driver for the library's per-token softmax + top-k routine (route_serial.cuh), compiled as
// plain C++: reads "T E k gate_norm" and T*E logits from stdin, prints for each token its k expert
// ids and k gate weights.  Used by tests/test_route_serial_host.py against the CPU oracle.
// With the argument "kslots" the routine keeps the fewest slots the tensor-core router keeps for
// this k (2, 4, 6 or 8) instead of 8.
#define __device__
#define __forceinline__ inline
#include <cstdio>
#include <cstring>
#include <vector>

#include "../../mixture_experts_layer_23_b200/csrc/route_serial.cuh"

template <int KS>
static void route_row(const std::vector<float>& row, int k, int gate_norm) {
  const int E = (int)row.size();
  moe::TopK<KS> st;
  moe::topk_init(st);
  for (int e = 0; e < E; ++e) moe::topk_push(st, row[e], e);
  float den = 0.f;   // second pass: softmax denominator over all E logits, in expert order
  for (int e = 0; e < E; ++e) den += moe::softmax_term(st, row[e]);
  int idx[8];
  float w[8];
  moe::topk_finish(st, k, gate_norm, den, idx, w);
  for (int j = 0; j < k; ++j) printf("%d ", idx[j]);
  for (int j = 0; j < k; ++j) printf("%.9g ", w[j]);
  printf("\n");
}

int main(int argc, char** argv) {
  const bool kslots = argc > 1 && strcmp(argv[1], "kslots") == 0;
  int T, E, k, gate_norm;
  if (scanf("%d %d %d %d", &T, &E, &k, &gate_norm) != 4) return 1;
  std::vector<float> row(E);
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e)
      if (scanf("%f", &row[e]) != 1) return 1;
    if (!kslots || k > 6) route_row<8>(row, k, gate_norm);
    else if (k > 4) route_row<6>(row, k, gate_norm);
    else if (k > 2) route_row<4>(row, k, gate_norm);
    else route_row<2>(row, k, gate_norm);
  }
  return 0;
}
