// Host-side check of jf::exp_nonpos_f64 (the same source the row-statistics kernel compiles):
// reads doubles from stdin, prints exp_nonpos_f64 of each with 17 significant digits.  With the
// argument "table" it prints the 128 table entries instead.
#include <cstdio>
#include <cstring>

#include "../tree_verify_attention_jf_b200/csrc/jf_math.cuh"

int main(int argc, char** argv) {
  static const double tab[128] = JF_EXP2_FRAC128;
  if (argc > 1 && std::strcmp(argv[1], "table") == 0) {
    for (int j = 0; j < 128; ++j) std::printf("%a\n", tab[j]);
    return 0;
  }
  double x;
  while (std::scanf("%lf", &x) == 1) std::printf("%.17g\n", jf::exp_nonpos_f64(x, tab));
  return 0;
}
