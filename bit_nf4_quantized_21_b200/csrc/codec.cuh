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

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Nearest NF4 level of a normalised weight: code = #{i : x > t_i}, found by a
// 4-step binary search over the 15 sorted thresholds; the first step's
// threshold (t_7) comes from a register, the other three from shared memory.
__device__ __forceinline__ uint32_t nf4_encode(float x, const float* s_thr, float t7) {
  uint32_t c = (x > t7) ? 8u : 0u;
  c += (x > s_thr[c + 3]) ? 4u : 0u;
  c += (x > s_thr[c + 1]) ? 2u : 0u;
  c += (x > s_thr[c]) ? 1u : 0u;
  return c;
}

// K1.  Grid: one CTA per group of 256 blocks (16384 weights).  Eight threads
// share a 64-weight block (8 weights each, one 16-byte load of bf16), so a
// warp reads 4 whole blocks = 512 contiguous bytes and writes 128 contiguous
// bytes of codes.  The block absmax is a warp-shuffle max over the 8 lanes.
// All 8 of a thread's loads are issued before any is used, so every thread
// keeps 8 x 16 B in flight (HBM needs tens of KB per SM in flight).
template <typename T>
__global__ void __launch_bounds__(kQuantThreads)
    k_quantize_nf4(const T* __restrict__ w, int64_t nblocks, int dq, uint8_t* __restrict__ codes,
                   uint8_t* __restrict__ q8, float* __restrict__ s2,
                   float* __restrict__ absmax_out, int* status) {
  __shared__ float s_thr[16];
  __shared__ float s_absmax[256];
  __shared__ float s_wmax[kQuantThreads / 32];
  const int tid = threadIdx.x;
  if (tid < 15) s_thr[tid] = c_nf4_threshold[tid];
  __syncthreads();

  const int64_t g = blockIdx.x;
  const int64_t b0 = g * 256;
  const int nb = static_cast<int>((nblocks - b0) < 256 ? (nblocks - b0) : 256);
  const int sub = tid & 7;
  const float t7 = c_nf4_threshold[7];
  bool nonfinite = false;

  float v[8][8];
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int lb = it * 32 + (tid >> 3);
    if (lb < nb) load8<T>(w + (b0 + lb) * 64 + sub * 8, v[it]);
  }
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int lb = it * 32 + (tid >> 3);
    const bool valid = lb < nb;
    const int64_t b = b0 + lb;
    uint32_t mbits = 0;
    if (valid) {
#pragma unroll
      for (int i = 0; i < 8; ++i) mbits = max(mbits, __float_as_uint(v[it][i]) & 0x7FFFFFFFu);
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
      for (int i = 0; i < 8; ++i) word |= nf4_encode(__fmul_rn(v[it][i], inv), s_thr, t7) << (4 * i);
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
  const float step = (m >= FLT_MIN) ? __fdiv_rn(m, 255.0f) : 0.0f;
  if (tid < nb) {
    float q = 0.0f;
    if (step > 0.0f) q = fminf(rintf(__fdiv_rn(a, step)), 255.0f);
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
    const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t o[4];
      nf4_decode8(cw[c], t, o);
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
