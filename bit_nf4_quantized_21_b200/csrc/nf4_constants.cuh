// nf4_constants.cuh -- the NF4 codebook and its decision thresholds, as data.
//
// NF4 places its 16 levels at quantiles of a normal distribution, dense near
// zero ("QLoRA", learning-llms.pages.dev/topics/qlora, the bullet on NF4;
// "QLoRA", infra.bea.ai, §1 subsection "Key Innovation: NF4").
// The exact quantiles are those of the QLoRA paper's construction: 8
// positive levels, 7 negative, an exact zero at code 7, endpoints -1/+1.
// gen_nf4_constants.py (beside this file) prints these literals and states
// the construction; the thresholds are the level midpoints rounded toward
// -inf to binary32, so that  code(x) = #{i : x > t_i}  is the nearest level
// with ties going to the lower code.
#pragma once
#include <cstdint>

#define QLORA_NF4_LEVELS \
    -0x1.0000000000000p+0f,  /* 0: -1.000000000 */ \
    -0x1.6473620000000p-1f,  /* 1: -0.696192801 */ \
    -0x1.0cd65c0000000p-1f,  /* 2: -0.525072932 */ \
    -0x1.94653c0000000p-2f,  /* 3: -0.394917428 */ \
    -0x1.2344960000000p-2f,  /* 4: -0.284441322 */ \
    -0x1.7a6a7a0000000p-3f,  /* 5: -0.184773400 */ \
    -0x1.74f0d20000000p-4f,  /* 6: -0.091049977 */ \
    0x0.0p+0f,               /* 7: +0.000000000 */ \
    0x1.45f6020000000p-4f,   /* 8: +0.079580314 */ \
    0x1.4995be0000000p-3f,   /* 9: +0.160930142 */ \
    0x1.f809b40000000p-3f,   /* 10: +0.246112257 */ \
    0x1.5a066c0000000p-2f,   /* 11: +0.337915123 */ \
    0x1.c3496a0000000p-2f,   /* 12: +0.440709740 */ \
    0x1.200f520000000p-1f,   /* 13: +0.562616885 */ \
    0x1.7227600000000p-1f,   /* 14: +0.722956657 */ \
    0x1.0000000000000p+0f,   /* 15: +1.000000000 */

#define QLORA_NF4_THRESHOLDS \
    -0x1.b239b20000000p-1f,  /* 0: -0.848096430 */ \
    -0x1.38a4e00000000p-1f,  /* 1: -0.610632896 */ \
    -0x1.d708fa0000000p-2f,  /* 2: -0.459995180 */ \
    -0x1.5bd4ea0000000p-2f,  /* 3: -0.339679390 */ \
    -0x1.e079d40000000p-3f,  /* 4: -0.234607369 */ \
    -0x1.1a71720000000p-3f,  /* 5: -0.137911692 */ \
    -0x1.74f0d20000000p-5f,  /* 6: -0.045524988 */ \
    0x1.45f6020000000p-5f,   /* 7: +0.039790157 */ \
    0x1.ec90be0000000p-4f,   /* 8: +0.120255224 */ \
    0x1.a0cfb80000000p-3f,   /* 9: +0.203521192 */ \
    0x1.2b05a20000000p-2f,   /* 10: +0.292013675 */ \
    0x1.8ea7ea0000000p-2f,   /* 11: +0.389312416 */ \
    0x1.00da020000000p-1f,   /* 12: +0.501663268 */ \
    0x1.491b580000000p-1f,   /* 13: +0.642786741 */ \
    0x1.b913b00000000p-1f,   /* 14: +0.861478329 */

namespace qlora {

// host copies (codebook query) and device copies (kernels read them as
// constant-bank operands)
constexpr float kNF4Level[16] = {QLORA_NF4_LEVELS};
constexpr float kNF4Threshold[15] = {QLORA_NF4_THRESHOLDS};
__constant__ float c_nf4_level[16] = {QLORA_NF4_LEVELS};
__constant__ float c_nf4_threshold[15] = {QLORA_NF4_THRESHOLDS};

// The encoder's cell table.  x in [-1, 1] (|x| may exceed 1 by a rounding)
// is cut into 33 cells of width 1/16 centred on the multiples of 1/16:
// cell i = rint(16 x + 16) holds x in [(2i - 33)/32, (2i - 31)/32].  Each
// cell holds at most one threshold (consecutive thresholds are >= 0.08
// apart), so
//   #{j : x > t_j} = base_i + (x > thr_i)
// with base_i = #{j : t_j < (2i - 33)/32} and thr_i the cell's threshold
// (2.0, above every x, when it has none).  Every threshold lies >= 1.6e-3
// from a cell edge, far more than any rounding of x next to an edge, so a
// value there gets the same count in either cell.  33 entries of 4 bytes
// fit the 32 shared-memory banks with only cells 0 and 32 (x = -1, x = 1)
// sharing one.
constexpr int kNF4Cells = 33;
struct NF4CellTable {
  float thr[kNF4Cells];
  uint32_t base[kNF4Cells];
};
constexpr float nf4_cell_lo(int i) { return static_cast<float>(2 * i - 33) / 32.0f; }
constexpr float nf4_cell_hi(int i) { return static_cast<float>(2 * i - 31) / 32.0f; }
constexpr NF4CellTable make_nf4_cells() {
  NF4CellTable t{};
  for (int i = 0; i < kNF4Cells; ++i) {
    uint32_t base = 0;
    float thr = 2.0f;
    for (int j = 0; j < 15; ++j) {
      if (kNF4Threshold[j] < nf4_cell_lo(i)) ++base;
      else if (kNF4Threshold[j] < nf4_cell_hi(i) && thr == 2.0f) thr = kNF4Threshold[j];
    }
    t.thr[i] = thr;
    t.base[i] = base;
  }
  return t;
}
constexpr NF4CellTable kNF4CellTable = make_nf4_cells();
constexpr bool nf4_cells_ok() {
  for (int i = 0; i < kNF4Cells; ++i) {
    int inside = 0;
    for (int j = 0; j < 15; ++j) {
      if (kNF4Threshold[j] >= nf4_cell_lo(i) && kNF4Threshold[j] < nf4_cell_hi(i)) ++inside;
      const float d1 = kNF4Threshold[j] - nf4_cell_lo(i), d2 = kNF4Threshold[j] - nf4_cell_hi(i);
      if ((d1 < 1e-5f && d1 > -1e-5f) || (d2 < 1e-5f && d2 > -1e-5f)) return false;   // too near an edge
    }
    if (inside > 1) return false;
  }
  return kNF4CellTable.base[0] == 0 && kNF4CellTable.base[32] == 15 && kNF4CellTable.base[16] == 7 &&
         kNF4CellTable.thr[0] == 2.0f && kNF4CellTable.thr[32] == 2.0f;
}
static_assert(nf4_cells_ok(), "NF4 encoder cell table");
__constant__ NF4CellTable c_nf4_cells = kNF4CellTable;

// every entry present (a lost initializer would silently read as 0)
static_assert(kNF4Level[0] == -1.0f && kNF4Level[7] == 0.0f && kNF4Level[15] == 1.0f, "NF4 levels");
static_assert(kNF4Level[14] > 0.72f && kNF4Level[8] > 0.0f, "NF4 levels");
static_assert(kNF4Threshold[0] < -0.84f && kNF4Threshold[14] > 0.86f && kNF4Threshold[7] > 0.0f,
              "NF4 thresholds");

}  // namespace qlora
