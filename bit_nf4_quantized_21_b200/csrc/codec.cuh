// codec.cuh -- the one-shot NF4 quantiser and the standalone dequantiser.
//
// Both are HBM-bound streaming kernels.  Per weight the quantiser reads 2 B
// (bf16; 4 B for fp32) and writes 0.5 B of codes plus 1/64 B of q8; the
// dequantiser reads 0.516 B and writes 2 B.
#pragma once
#include <cfloat>
#include <cstdint>
#include "nf4_decode.cuh"

namespace qlora {

constexpr int kQuantThreads = 256;  // one CTA per 256-block group

// The 8 weights a thread holds per block, kept as loaded (a bf16 uint4
// is 4 registers instead of 8 floats) and widened only when encoded.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> { uint4 u; };
template <> struct Raw8<float> { float4 a, b; };
__device__ __forceinline__ Raw8<__nv_bfloat16> load_raw8(const __nv_bfloat16* p) {
  return {__ldg(reinterpret_cast<const uint4*>(p))};
}
__device__ __forceinline__ Raw8<float> load_raw8(const float* p) {
  return {__ldg(reinterpret_cast<const float4*>(p)), __ldg(reinterpret_cast<const float4*>(p) + 1)};
}
__device__ __forceinline__ void widen8(const Raw8<__nv_bfloat16>& r, float (&v)[8]) {
  const uint32_t w[4] = {r.u.x, r.u.y, r.u.z, r.u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void widen8(const Raw8<float>& r, float (&v)[8]) {
  v[0] = r.a.x; v[1] = r.a.y; v[2] = r.a.z; v[3] = r.a.w;
  v[4] = r.b.x; v[5] = r.b.y; v[6] = r.b.z; v[7] = r.b.w;
}

// Nearest NF4 level of a normalised weight: code = #{i : x > t_i}, from the
// cell table (nf4_constants.cuh): cell = rint(32 x + 32.5), found with one
// fused multiply-add and the 1.5 * 2^23 rounding trick (the sum's low
// mantissa bits are the integer), then one compare against the cell's
// threshold.  The index is clamped to the table (a NaN x, from a block with
// an infinite absmax, reads the last cell; such blocks are flagged).
__device__ __forceinline__ uint32_t nf4_encode(float x, const uint2* s_cell) {
  const float y = __fadd_rn(__fmaf_rn(x, 32.0f, 32.5f), 12582912.0f);
  const uint32_t idx = min(static_cast<uint32_t>(__float_as_int(y)) - 0x4B400000u, 65u);
  const uint2 e = s_cell[idx];
  return e.y + ((x > __uint_as_float(e.x)) ? 1u : 0u);
}

// E4M3 code of a non-negative float: round to nearest even, values above
// 448 saturate to 448 (the hardware conversion of two floats packs the
// second operand into the low byte).
__device__ __forceinline__ uint32_t f32_to_e4m3(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return static_cast<uint32_t>(r) & 0xFFu;
}

// K1.  Grid: one CTA per group of 256 blocks (16384 weights).  Eight threads
// share a 64-weight block (8 weights each, one 16-byte load of bf16), so a
// warp reads 4 whole blocks = 512 contiguous bytes and writes 128 contiguous
// bytes of codes.  The block absmax is a warp-shuffle max over the 8 lanes.
// All 8 of a thread's loads are issued before any is used and are kept as
// loaded (32 registers for bf16), which leaves room for 5 CTAs per SM: with
// 8 x 16 B in flight per thread that is 160 KB per SM (HBM needs tens of KB
// per SM in flight).  The encoding is ~11 instructions per weight.
template <typename T>
__global__ void __launch_bounds__(kQuantThreads, sizeof(T) == 2 ? 5 : 3)
    k_quantize_nf4(const T* __restrict__ w, int64_t nblocks, int dq, uint8_t* __restrict__ codes,
                   uint8_t* __restrict__ q8, float* __restrict__ s2,
                   float* __restrict__ absmax_out, int* status) {
  __shared__ uint2 s_cell[66];
  __shared__ float s_absmax[256];
  __shared__ float s_wmax[kQuantThreads / 32];
  const int tid = threadIdx.x;
  if (tid < 66) s_cell[tid] = make_uint2(__float_as_uint(c_nf4_cells.c[tid].thr), c_nf4_cells.c[tid].base);

  const int64_t g = blockIdx.x;
  const int64_t b0 = g * 256;
  const int nb = static_cast<int>((nblocks - b0) < 256 ? (nblocks - b0) : 256);
  const int sub = tid & 7;
  bool nonfinite = false;

  Raw8<T> raw[8];
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int lb = it * 32 + (tid >> 3);
    if (lb < nb) raw[it] = load_raw8(w + (b0 + lb) * 64 + sub * 8);
  }
  __syncthreads();   // the cell table is in shared memory
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int lb = it * 32 + (tid >> 3);
    const bool valid = lb < nb;
    const int64_t b = b0 + lb;
    float v[8];
    widen8(raw[it], v);
    uint32_t mbits = 0;
    if (valid) {
#pragma unroll
      for (int i = 0; i < 8; ++i) mbits = max(mbits, __float_as_uint(v[i]) & 0x7FFFFFFFu);
    }
    // max over the 8 lanes of the block (integer order = magnitude order,
    // with inf/NaN patterns above every finite value)
    mbits = max(mbits, __shfl_xor_sync(0xFFFFFFFFu, mbits, 1));
    mbits = max(mbits, __shfl_xor_sync(0xFFFFFFFFu, mbits, 2));
    mbits = max(mbits, __shfl_xor_sync(0xFFFFFFFFu, mbits, 4));
    if (!valid) continue;
    if (mbits >= 0x7F800000u) nonfinite = true;
    const float absmax = __uint_as_float(mbits);
    uint32_t word;
    if (!(absmax >= FLT_MIN)) {
      word = 0x77777777u;  // zero (or subnormal) block: every weight is code 7
    } else {
      const float inv = __frcp_rn(absmax);
      word = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) word |= nf4_encode(__fmul_rn(v[i], inv), s_cell) << (4 * i);
    }
    reinterpret_cast<uint32_t*>(codes)[b * 8 + sub] = word;
    if (sub == 0) s_absmax[lb] = absmax;
  }
  if (nonfinite && status) atomicOr(status, QLORA_DEV_NONFINITE);
  __syncthreads();

  const float a = (tid < nb) ? s_absmax[tid] : 0.0f;
  if (absmax_out && tid < nb) absmax_out[b0 + tid] = a;
  if (!dq) return;
  float m = a;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((tid & 31) == 0) s_wmax[tid >> 5] = m;
  __syncthreads();
  m = s_wmax[0];
#pragma unroll
  for (int i = 1; i < kQuantThreads / 32; ++i) m = fmaxf(m, s_wmax[i]);
  // linear 8-bit: s2 = m / 255, q = min(255, rint(absmax / s2));
  // FP8 E4M3: s2 = m / 448 (E4M3's largest finite value), q = E4M3 code of
  // absmax / s2, round to nearest even, saturating
  const bool fp8 = dq == kDqE4M3;
  const float step = (m >= FLT_MIN) ? __fdiv_rn(m, fp8 ? 448.0f : 255.0f) : 0.0f;
  if (tid < nb) {
    uint32_t q = 0;
    if (step > 0.0f) {
      const float v = __fdiv_rn(a, step);
      q = fp8 ? f32_to_e4m3(v) : static_cast<uint32_t>(fminf(rintf(v), 255.0f));
    }
    q8[b0 + tid] = static_cast<uint8_t>(q);
  }
  if (tid == 0) s2[g] = step;
}

// K2.  One thread per 64-weight block: two 16-byte loads of codes, one
// table build, 64 bf16 out.  Each warp stages its 32 blocks (4 KB) in shared
// memory (16-byte chunks XOR-swizzled by row) so that the global stores are
// 512 contiguous bytes per instruction.
constexpr int kDeqThreads = 256;

__global__ void __launch_bounds__(kDeqThreads)
    k_dequantize_nf4(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ q8,
                     const float* __restrict__ s2, const float* __restrict__ absmax_f32, int dq,
                     int64_t nblocks, __nv_bfloat16* __restrict__ out) {
  __shared__ uint4 stage[kDeqThreads / 32][32 * 8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t wbase = (static_cast<int64_t>(blockIdx.x) * kDeqThreads) + warp * 32;
  const int64_t b = wbase + lane;
  if (b < nblocks) {
    const uint4* cp = reinterpret_cast<const uint4*>(codes + b * 32);
    const uint4 c0 = __ldg(cp), c1 = __ldg(cp + 1);
    const NF4Table t = nf4_table(nf4_block_scale(q8, s2, absmax_f32, dq, b));
    const NF4Shr sh = nf4_shr();
    const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t o[4];
      nf4_decode8(cw[c], t, o, sh);
      stage[warp][lane * 8 + (c ^ (lane & 7))] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  __syncwarp();
  uint4* dst = reinterpret_cast<uint4*>(out);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int flat = i * 32 + lane;
    const int row = flat >> 3, c = flat & 7;
    if (wbase + row < nblocks)
      dst[(wbase + row) * 8 + c] = stage[warp][row * 8 + (c ^ (row & 7))];
  }
}

}  // namespace qlora
