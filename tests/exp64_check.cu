// Host-side check of jf::exp_nonpos_f64 (the same source the row-statistics kernel compiles):
// reads doubles from stdin, prints exp_nonpos_f64 of each with 17 significant digits.
#include <cstdio>

#include "../tree_verify_attention_jf_b200/csrc/jf_math.cuh"

int main() {
  double x;
  while (std::scanf("%lf", &x) == 1) std::printf("%.17g\n", jf::exp_nonpos_f64(x));
  return 0;
}
