// merge.cuh -- folding a trained adapter back into the frozen NF4 base:
// W' = dequant(W_4bit) + s B A, re-quantised to NF4.
//
// "QLoRA" (learning-llms page), the fine-print bullet on merging: folding
// BA into W assumed both in one precision; adding a bf16 update into 4-bit
// weights forces a re-quantisation.  katajob.com, "What it costs": merge
// friction -- merging a high-precision delta into a low-precision weight
// means re-quantising.  This is that merge: each merged weight is formed in
// fp32 with a fixed operation order, written to an fp32 buffer, and the
// buffer is then quantised by the ordinary quantiser (codec.cuh).  Per
// element (n, k), every operation an IEEE fp32 operation with one rounding:
//   acc = 0;  for j = 0 .. r-1:  acc = acc + B[n, j] * A[j, k]
//   W'[n, k] = W^[n, k] + s * acc
// where W^ is the bf16 dequantised weight (nf4_decode.cuh) and s = alpha / r.
// Two forms: k_merge_nf4 writes W' to an fp32 buffer (one thread per 8
// consecutive weights), which the caller's quantiser pass then encodes; or
// MergeSrc feeds the quantiser kernel (codec.cuh) the same W' values formed
// in registers, so the merge is one pass that reads the 4-bit weight and
// writes the 4-bit result, with the same codes and scales bit for bit.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "nf4_decode.cuh"
#include "codec.cuh"

namespace qlora {

constexpr int kMergeThreads = 256;

__global__ void __launch_bounds__(kMergeThreads)
    k_merge_nf4(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ q8, const float* __restrict__ s2,
                const float* __restrict__ absmax_f32, int dq, int64_t N, int64_t K,
                const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ B, int r, float s,
                float* __restrict__ out) {
  const int64_t K8 = K / 8;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= N * K8) return;
  const int64_t n = idx / K8, k0 = (idx - n * K8) * 8;
  const int64_t e0 = n * K + k0;                       // first element (row-major)
  const NF4Table tab = nf4_table(nf4_block_scale(q8, s2, absmax_f32, dq, e0 / 64));
  uint32_t wh[4];
  nf4_decode8(__ldg(reinterpret_cast<const uint32_t*>(codes + e0 / 2)), tab, wh);
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
  for (int j = 0; j < r; ++j) {
    const float b = __bfloat162float(B[n * r + j]);
    const uint4 av = __ldg(reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j) * K + k0));
    const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(b, __uint_as_float(aw[i] << 16)));
      acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(b, __uint_as_float(aw[i] & 0xFFFF0000u)));
    }
  }
  float w[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[2 * i] = __fadd_rn(__uint_as_float(wh[i] << 16), __fmul_rn(s, acc[2 * i]));
    w[2 * i + 1] = __fadd_rn(__uint_as_float(wh[i] & 0xFFFF0000u), __fmul_rn(s, acc[2 * i + 1]));
  }
  float4* dst = reinterpret_cast<float4*>(out + e0);
  dst[0] = make_float4(w[0], w[1], w[2], w[3]);
  dst[1] = make_float4(w[4], w[5], w[6], w[7]);
}

// 16 merged weights of one block, for the quantiser kernel.
struct Merged16 {
  float v[16];
};
__device__ __forceinline__ void widen16(const Merged16& m, float (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = m.v[i];
}
__device__ __forceinline__ uint32_t mag_bits16(const Merged16& m) {
  uint32_t b = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) b = max(b, __float_as_uint(m.v[i]) & 0x7FFFFFFFu);
  return b;
}

// W' = W^ + s B A as a weight source of the quantiser kernel: load(e0)
// forms the 16 merged weights e0 .. e0 + 15 (one block's quarter, one row)
// in the order above.  The source weight's format (dq) is its own; the
// quantiser writes the output in the output's format.
struct MergeSrc {
  const uint8_t* codes;
  const uint8_t* q8;
  const float* s2;
  const float* absmax_f32;
  int dq;
  int64_t K;
  const __nv_bfloat16* A;   // [r, K]
  const __nv_bfloat16* B;   // [N, r]
  int r;
  float s;
  static constexpr int kMinBlocks = 2;
  __device__ __forceinline__ Merged16 load(int64_t e0) const {
    const int64_t n = e0 / K, k0 = e0 - n * K;
    const NF4Table tab = nf4_table(nf4_block_scale(q8, s2, absmax_f32, dq, e0 / 64));
    const uint2 cw = __ldg(reinterpret_cast<const uint2*>(codes + e0 / 2));
    uint32_t wl[4], wu[4];
    nf4_decode8(cw.x, tab, wl);
    nf4_decode8(cw.y, tab, wu);
    const uint32_t wh[8] = {wl[0], wl[1], wl[2], wl[3], wu[0], wu[1], wu[2], wu[3]};
    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0.0f;
    for (int j = 0; j < r; ++j) {
      const float b = __bfloat162float(B[n * r + j]);
      const uint4* ap = reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j) * K + k0);
      const uint4 a0 = __ldg(ap), a1 = __ldg(ap + 1);
      const uint32_t aw[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(b, __uint_as_float(aw[i] << 16)));
        acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(b, __uint_as_float(aw[i] & 0xFFFF0000u)));
      }
    }
    Merged16 m;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      m.v[2 * i] = __fadd_rn(__uint_as_float(wh[i] << 16), __fmul_rn(s, acc[2 * i]));
      m.v[2 * i + 1] = __fadd_rn(__uint_as_float(wh[i] & 0xFFFF0000u), __fmul_rn(s, acc[2 * i + 1]));
    }
    return m;
  }
};

}  // namespace qlora
