// CPU check of the emulated exp2 used by the prefill softmax: prints the
// maximum relative error against std::exp2 (double) over a dense sweep of
// [-125, 9] and a few exact points.  Built and run by tests/test_exp2_poly.py.
#include <cmath>
#include <cstdio>

#include "../../long_context_attention_dca_b200/csrc/exp2_poly.cuh"

int main() {
  double max_rel = 0.0;
  double worst_x = 0.0;
  const int n = 2000000;
  for (int i = 0; i <= n; ++i) {
    const float x = (float)(-125.0 + 134.0 * (double)i / n);
    const double ref = std::exp2((double)x);
    const double got = (double)dca::exp2_poly3(x);
    const double rel = std::fabs(got - ref) / ref;
    if (rel > max_rel) {
      max_rel = rel;
      worst_x = x;
    }
  }
  // integers are exact powers of two up to the polynomial's value at 0
  double max_int_rel = 0.0;
  for (int k = -125; k <= 8; ++k) {
    const double rel = std::fabs((double)dca::exp2_poly3((float)k) - std::exp2((double)k)) /
                       std::exp2((double)k);
    if (rel > max_int_rel) max_int_rel = rel;
  }
  const float below = dca::exp2_poly3(-1000.0f);
  const float neg_inf = dca::exp2_poly3(-INFINITY);
  std::printf("%.9e %.9e %.9e %.9e %.9e\n", max_rel, worst_x, max_int_rel, (double)below,
              (double)neg_inf);
  return 0;
}
