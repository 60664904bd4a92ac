// Exhaustive host-side check of the quantiser's cell-table encoder.
//
// Compiles the kernel's own constants header (nf4_constants.cuh) as plain
// C++ and, for every binary32 x in [-1.0001, 1.0001], compares the code the
// kernel's formula gives (cell = rint(16 x + 16) by one fused multiply-add,
// then base + one compare) with the nearest of the 16 levels passed on the
// command line (binary64 distance, ties to the lower code: the normalise-
// and-round-to-nearest step of NF4 quantisation).  Prints the number of
// mismatches; exit status 1 on any.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#define __constant__
#include "nf4_constants.cuh"

static uint32_t kernel_code(float x) {
  const float y = std::fmaf(x, 16.0f, 12582928.0f);
  uint32_t yb;
  std::memcpy(&yb, &y, 4);
  uint32_t idx = yb - 0x4B400000u;
  if (idx > static_cast<uint32_t>(qlora::kNF4Cells - 1)) idx = qlora::kNF4Cells - 1;
  return qlora::kNF4CellTable.base[idx] + ((x > qlora::kNF4CellTable.thr[idx]) ? 1u : 0u);
}

int main(int argc, char** argv) {
  if (argc != 17) { std::fprintf(stderr, "usage: %s level0 .. level15\n", argv[0]); return 2; }
  double lv[16];
  for (int i = 0; i < 16; ++i) lv[i] = std::strtod(argv[i + 1], nullptr);
  // every non-negative binary32 up to 1.0001, with both signs
  float lim = 1.0001f;
  uint32_t top;
  std::memcpy(&top, &lim, 4);
  long bad = 0;
#pragma omp parallel for reduction(+ : bad) schedule(static, 1 << 20)
  for (int64_t i = 0; i <= 2 * static_cast<int64_t>(top) + 1; ++i) {
    const uint32_t b = static_cast<uint32_t>(i >> 1) | ((i & 1) ? 0x80000000u : 0u);
    float x;
    std::memcpy(&x, &b, 4);
    int best = 0;
    double bd = std::fabs(static_cast<double>(x) - lv[0]);
    for (int k = 1; k < 16; ++k) {
      const double d = std::fabs(static_cast<double>(x) - lv[k]);
      if (d < bd) { bd = d; best = k; }
    }
    if (kernel_code(x) != static_cast<uint32_t>(best)) ++bad;
  }
  std::printf("values %lld mismatches %ld nan_code %u\n", 2 * static_cast<long long>(top) + 2, bad,
              kernel_code(std::nanf("")));
  return bad != 0;
}
