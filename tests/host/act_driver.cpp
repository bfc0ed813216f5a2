// Host driver for the bf16 epilogues' activation functions (act_fast.cuh), compiled as plain C++
// (exact expf and division stand in for the fast intrinsics): reads u values from stdin, prints
// "gelu gelu_grad sigmoid" per value.  Used by tests/test_act_fast_host.py.
#define MOE_ACT_HOST_TEST
#include <cstdio>

#include "../../mixture_experts_layer_23_b200/csrc/act_fast.cuh"

int main() {
  float u;
  while (scanf("%f", &u) == 1)
    printf("%.9g %.9g %.9g\n", moe::fast::gelu(u), moe::fast::gelu_grad(u), moe::fast::sigmoid(u));
  return 0;
}
