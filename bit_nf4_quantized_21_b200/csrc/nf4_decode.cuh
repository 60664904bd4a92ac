// nf4_decode.cuh -- register-only NF4 -> bf16 decoding, shared by the
// standalone dequantiser, the fused GEMM and the decode kernel.
//
// For one 64-weight block with block scale `scale`, the 16 possible bf16
// outputs bf16_rne(fp32(level[c] * scale)) are computed once (16 fp32
// multiplies, 8 cvt.rn.bf16x2) and split into a table of low bytes and a
// table of high bytes, 16 bytes each (4 registers each).  A byte permute
// (prmt) then looks up 4 codes at a time: the code's low 3 bits pick a byte
// within one 8-entry half of the table, and its high bit picks the half.
// The result is bit-identical to evaluating the definition per element.
#pragma once
#include <cstdint>
#include "nf4_constants.cuh"
#include "ptx.cuh"

namespace qlora {

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

struct NF4Table {
  uint32_t lo[4];  // low byte of the bf16 of code 4q .. 4q+3 in word q
  uint32_t hi[4];  // high byte
};

__device__ __forceinline__ NF4Table nf4_table(float scale) {
  uint32_t p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    p[i] = pack_bf16x2(__fmul_rn(c_nf4_level[2 * i], scale), __fmul_rn(c_nf4_level[2 * i + 1], scale));
  NF4Table t;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    t.lo[q] = prmt(p[2 * q], p[2 * q + 1], 0x6420u);
    t.hi[q] = prmt(p[2 * q], p[2 * q + 1], 0x7531u);
  }
  return t;
}

// The decode's three right shifts are done as high halves of multiplies
// (x >> k == mulhi(x, 2^(32 - k))): a multiply issues on the FMA pipe, while
// every byte permute and mask of the lookup issues on the integer pipe, which
// is the decode's bottleneck.  The multipliers are read from constant memory
// so that the compiler cannot turn the multiplies back into shifts.
__constant__ uint32_t c_nf4_shr[2] = {0x80000000u /* >> 1 */, 0x00010000u /* >> 16 */};
struct NF4Shr {
  uint32_t m1, m16;
};
__device__ __forceinline__ NF4Shr nf4_shr() { return NF4Shr{c_nf4_shr[0], c_nf4_shr[1]}; }

// 8 codes (one 32-bit word; code i in bits 4i..4i+3) -> 8 bf16 in 4 words,
// element 2j in the low half of word j.
__device__ __forceinline__ void nf4_decode8(uint32_t w, const NF4Table& t, uint32_t (&o)[4],
                                            NF4Shr sh = NF4Shr{0x80000000u, 0x00010000u}) {
  const uint32_t idx = w & 0x77777777u;                                      // low 3 bits of every code
  const uint32_t half = (__umulhi(w, sh.m1) & 0x44444444u) | 0x32103210u;    // byte i from word A or B
  // prmt reads only the low 16 bits (four nibbles) of its selector, so the
  // upper half of idx / half needs no masking for h = 0
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t s = h ? __umulhi(idx, sh.m16) : idx;
    const uint32_t g = h ? __umulhi(half, sh.m16) : half;
    const uint32_t lo = prmt(prmt(t.lo[0], t.lo[1], s), prmt(t.lo[2], t.lo[3], s), g);
    const uint32_t hi = prmt(prmt(t.hi[0], t.hi[1], s), prmt(t.hi[2], t.hi[3], s), g);
    o[2 * h] = prmt(lo, hi, 0x5140u);
    o[2 * h + 1] = prmt(lo, hi, 0x7362u);
  }
}

// Second-level scale formats (the weight's double_quant field): none (fp32
// block absmax), linear 8-bit (q * s2), and FP8 E4M3 codes (E4M3(q) * s2,
// "QLoRA", infra.bea.ai, §1 subsection "Double Quantization", which
// quantises the block scales to FP8).
constexpr int kDqNone = 0, kDqU8 = 1, kDqE4M3 = 2;

// Value of an E4M3 code 0..126 (bias 7, 3 mantissa bits; no sign, no NaN:
// the quantiser writes only non-negative finite codes): the exponent field
// moves to fp32's bias, the 3 mantissa bits to the top of fp32's mantissa;
// exponent field 0 is the subnormal range m * 2^-9.
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
  const uint32_t e = c >> 3, m = c & 7u;
  return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : static_cast<float>(m) * 0x1p-9f;
}
// The stored 8-bit value of a block's absmax as a float.
__device__ __forceinline__ float dq_value(uint32_t q, int dq) {
  return dq == kDqE4M3 ? e4m3_to_f32(q) : static_cast<float>(q);
}

// Block scale of the stored format.
__device__ __forceinline__ float nf4_block_scale(const uint8_t* __restrict__ q8,
                                                 const float* __restrict__ s2,
                                                 const float* __restrict__ absmax_f32, int dq,
                                                 int64_t b) {
  if (dq) return __fmul_rn(dq_value(__ldg(q8 + b), dq), __ldg(s2 + (b >> 8)));
  return __ldg(absmax_f32 + b);
}

}  // namespace qlora
