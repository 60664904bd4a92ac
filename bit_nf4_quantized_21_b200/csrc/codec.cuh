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

// The 16 weights a thread holds per block, kept as loaded (bf16: two uint4,
// 8 registers instead of 16 floats) and widened only when encoded.
template <typename T> struct Raw16;
template <> struct Raw16<__nv_bfloat16> { uint4 a, b; };
template <> struct Raw16<float> { float4 a, b, c, d; };
__device__ __forceinline__ Raw16<__nv_bfloat16> load_raw16(const __nv_bfloat16* p) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
  return {__ldg(q), __ldg(q + 1)};
}
__device__ __forceinline__ Raw16<float> load_raw16(const float* p) {
  const float4* q = reinterpret_cast<const float4*>(p);
  return {__ldg(q), __ldg(q + 1), __ldg(q + 2), __ldg(q + 3)};
}
__device__ __forceinline__ void widen16(const Raw16<__nv_bfloat16>& r, float (&v)[16]) {
  const uint32_t w[8] = {r.a.x, r.a.y, r.a.z, r.a.w, r.b.x, r.b.y, r.b.z, r.b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void widen16(const Raw16<float>& r, float (&v)[16]) {
  const float4 q[4] = {r.a, r.b, r.c, r.d};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[4 * i] = q[i].x; v[4 * i + 1] = q[i].y; v[4 * i + 2] = q[i].z; v[4 * i + 3] = q[i].w;
  }
}
// The largest |weight| of the 16 as a binary32 bit pattern.  Integer order
// of sign-cleared patterns is magnitude order, with inf and NaN patterns
// above every finite value; bf16 pairs are compared two at a time as
// 16-bit lanes, then widened.
__device__ __forceinline__ uint32_t mag_bits16(const Raw16<__nv_bfloat16>& r) {
  const uint32_t w[8] = {r.a.x, r.a.y, r.a.z, r.a.w, r.b.x, r.b.y, r.b.z, r.b.w};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = __vmaxu2(m, w[i] & 0x7FFF7FFFu);
  return max(m & 0xFFFFu, m >> 16) << 16;
}
__device__ __forceinline__ uint32_t mag_bits16(const Raw16<float>& r) {
  const float4 q[4] = {r.a, r.b, r.c, r.d};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = max(m, __float_as_uint(q[i].x) & 0x7FFFFFFFu);
    m = max(m, __float_as_uint(q[i].y) & 0x7FFFFFFFu);
    m = max(m, __float_as_uint(q[i].z) & 0x7FFFFFFFu);
    m = max(m, __float_as_uint(q[i].w) & 0x7FFFFFFFu);
  }
  return m;
}

// Nearest NF4 level of a normalised weight: code = #{i : x > t_i}, from the
// cell table (nf4_constants.cuh): cell = rint(16 x + 16), found with one
// fused multiply-add whose addend 1.5 * 2^23 + 16 leaves the rounded sum's
// low mantissa bits equal to the integer, then one compare against the
// cell's threshold.  Both table reads are 4-byte loads from the same
// address register.  The index is clamped to the table (a NaN x, from a
// block with an infinite absmax, reads the last cell; such blocks are
// flagged).
__device__ __forceinline__ uint32_t nf4_encode(float x, const NF4CellTable* s_cell) {
  const float y = __fmaf_rn(x, 16.0f, 12582928.0f);
  const uint32_t idx = min(static_cast<uint32_t>(__float_as_int(y)) - 0x4B400000u, static_cast<uint32_t>(kNF4Cells - 1));
  const float thr = s_cell->thr[idx];
  return s_cell->base[idx] + ((x > thr) ? 1u : 0u);
}

// E4M3 code of a non-negative float: round to nearest even, values above
// 448 saturate to 448 (the hardware conversion of two floats packs the
// second operand into the low byte).
__device__ __forceinline__ uint32_t f32_to_e4m3(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return static_cast<uint32_t>(r) & 0xFFu;
}

// Where the weights come from: a bf16 or fp32 matrix in global memory
// (the quantiser), or values a source computes itself (the fused adapter
// merge, merge.cuh).  load(e0) returns the 16 weights e0 .. e0 + 15 of one
// block in a form widen16 / mag_bits16 accept.
template <typename T> struct PtrSrc {
  const T* p;
  static constexpr int kMinBlocks = sizeof(T) == 2 ? 4 : 3;   // CTAs per SM the registers allow
  __device__ __forceinline__ Raw16<T> load(int64_t e0) const { return load_raw16(p + e0); }
};

// K1.  Grid: one CTA per group of 256 blocks (16384 weights).  Four threads
// share a 64-weight block (16 weights each, two 16-byte loads of bf16), so a
// warp reads 8 whole blocks = 1 KB contiguous and writes 256 contiguous
// bytes of codes.  The block absmax is a shuffle max over the 4 lanes; the
// per-block work (shuffles, reciprocal, checks, stores) is spread over 16
// weights per thread.  All 4 of a thread's block loads are issued before
// any is used and are kept as loaded (32 registers for bf16); 4 CTAs per SM
// keep 128 B per thread, 128 KB per SM, in flight.
// The encoding is ~10 instructions per weight.
template <typename Src>
__global__ void __launch_bounds__(kQuantThreads, Src::kMinBlocks)
    k_quantize_nf4(const Src src, int64_t nblocks, int dq, uint8_t* __restrict__ codes,
                   uint8_t* __restrict__ q8, float* __restrict__ s2,
                   float* __restrict__ absmax_out, int* status) {
  __shared__ NF4CellTable s_cell;
  __shared__ float s_absmax[256];
  __shared__ float s_wmax[kQuantThreads / 32];
  const int tid = threadIdx.x;
  if (tid < kNF4Cells) {
    s_cell.thr[tid] = c_nf4_cells.thr[tid];
    s_cell.base[tid] = c_nf4_cells.base[tid];
  }

  const int64_t g = blockIdx.x;
  const int64_t b0 = g * 256;
  const int nb = static_cast<int>((nblocks - b0) < 256 ? (nblocks - b0) : 256);
  const int sub = tid & 3;   // weights 16 sub .. 16 sub + 15 of the block
  bool nonfinite = false;

  decltype(src.load(0)) raw[4];
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int lb = it * 64 + (tid >> 2);
    if (lb < nb) raw[it] = src.load((b0 + lb) * 64 + sub * 16);
  }
  __syncthreads();   // the cell table is in shared memory
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int lb = it * 64 + (tid >> 2);
    const bool valid = lb < nb;
    uint32_t mbits = valid ? mag_bits16(raw[it]) : 0u;
    mbits = max(mbits, __shfl_xor_sync(0xFFFFFFFFu, mbits, 1));
    mbits = max(mbits, __shfl_xor_sync(0xFFFFFFFFu, mbits, 2));
    if (!valid) continue;
    if (mbits >= 0x7F800000u) nonfinite = true;
    const float absmax = __uint_as_float(mbits);
    uint2 word;
    if (!(absmax >= FLT_MIN)) {
      word = make_uint2(0x77777777u, 0x77777777u);  // zero (or subnormal) block: every weight is code 7
    } else {
      const float inv = __frcp_rn(absmax);
      float v[16];
      widen16(raw[it], v);
      uint32_t h[2] = {0, 0};
#pragma unroll
      for (int i = 0; i < 16; ++i) h[i >> 3] |= nf4_encode(__fmul_rn(v[i], inv), &s_cell) << (4 * (i & 7));
      word = make_uint2(h[0], h[1]);
    }
    reinterpret_cast<uint2*>(codes)[(b0 + lb) * 4 + sub] = word;
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
