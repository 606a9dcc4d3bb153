// Host-side check of jf::exp_nonpos_f64 (the same source the row-statistics kernel compiles):
// reads doubles from stdin, prints exp_nonpos_f64 of each with 17 significant digits.  With the
// argument "table" it prints the 32 table entries instead.
#include <cstdio>
#include <cstring>

#include "../tree_verify_attention_jf_b200/csrc/jf_math.cuh"

int main(int argc, char** argv) {
  static const double tab[32] = JF_EXP2_FRAC32;
  if (argc > 1 && std::strcmp(argv[1], "table") == 0) {
    for (int j = 0; j < 32; ++j) std::printf("%a\n", tab[j]);
    return 0;
  }
  double x;
  while (std::scanf("%lf", &x) == 1) std::printf("%.17g\n", jf::exp_nonpos_f64(x, tab));
  return 0;
}
