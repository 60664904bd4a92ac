// dropout.cuh -- LoRA dropout on the adapter input.
//
// "QLoRA" (infra.bea.ai), §3 "Implementation", configures the adapters with
// lora_dropout = 0.05 in a PEFT LoraConfig and defines nothing further.  This
// library reads it as inverted dropout on the adapter's input only: the
// frozen path sees X unchanged, the adapter sees X * keep, and the kept
// elements are scaled by 1 / (1 - p).  Because X * keep is still exactly
// bf16, the 1 / (1 - p) is applied to the fp32 products instead:
//   T  = (X * keep) A^T / (1 - p)
//   dA = s G^T (X * keep) / (1 - p)
//   dX = dY W^ + s ((G A) * keep) / (1 - p)
// One mask per call, regenerated wherever it is needed from a counter-based
// generator: element e = m K + k (row-major over X [M, K]) is kept iff the
// top 32 bits of word e mod 4 of Philox-4x64-10 at counter (e div 4, 0, 0, 0)
// under key (seed, 0) are >= ceil(p 2^32).  Philox-4x64-10 is the generator
// of Salmon, Moraes, Dror and Shaw ("Parallel random numbers: as easy as 1,
// 2, 3", SC 2011): ten rounds of two 64 x 64 -> 128-bit products on a
// four-word counter, the two-word key bumped by two Weyl constants after
// every round.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace qlora {

constexpr uint64_t kPhiloxM0 = 0xD2E7470EE14C6C93ull;   // round multipliers
constexpr uint64_t kPhiloxM1 = 0xCA5A826395121157ull;
constexpr uint64_t kPhiloxW0 = 0x9E3779B97F4A7C15ull;   // key increments
constexpr uint64_t kPhiloxW1 = 0xBB67AE8584CAA73Bull;

// The four 64-bit words of Philox-4x64-10 at counter (c0, 0, 0, 0), key (k0, 0).
__device__ __forceinline__ void philox4x64_10(uint64_t c0, uint64_t k0, uint64_t (&x)[4]) {
  uint64_t a = c0, b = 0, c = 0, d = 0, ka = k0, kb = 0;
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint64_t hi0 = __umul64hi(kPhiloxM0, a), lo0 = kPhiloxM0 * a;
    const uint64_t hi1 = __umul64hi(kPhiloxM1, c), lo1 = kPhiloxM1 * c;
    a = hi1 ^ b ^ ka;
    b = lo1;
    c = hi0 ^ d ^ kb;
    d = lo0;
    ka += kPhiloxW0;
    kb += kPhiloxW1;
  }
  x[0] = a; x[1] = b; x[2] = c; x[3] = d;
}

// Keep bits of elements 4 q .. 4 q + 3 (bit i = element 4 q + i).
__device__ __forceinline__ uint32_t dropout_keep4(uint64_t q, uint64_t seed, uint64_t thr) {
  uint64_t x[4];
  philox4x64_10(q, seed, x);
  uint32_t bits = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) bits |= ((x[i] >> 32) >= thr ? 1u : 0u) << i;
  return bits;
}

constexpr int kDropThreads = 256;

// Xd = X * keep over n elements (n % 8 == 0): each thread takes 8 elements
// (one 16-byte load and store, two Philox blocks); a dropped element becomes +0.
__global__ void __launch_bounds__(kDropThreads)
    k_dropout_x(const __nv_bfloat16* __restrict__ X, __nv_bfloat16* __restrict__ Xd, int64_t n, uint64_t seed,
                uint64_t thr) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kDropThreads;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * kDropThreads + threadIdx.x; v * 8 < n; v += stride) {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(X) + v);
    const uint32_t keep = dropout_keep4(2 * v, seed, thr) | (dropout_keep4(2 * v + 1, seed, thr) << 4);
    uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = (keep >> (2 * i)) & 1u ? 0x0000FFFFu : 0u;
      const uint32_t hi = (keep >> (2 * i + 1)) & 1u ? 0xFFFF0000u : 0u;
      w[i] &= lo | hi;
    }
    reinterpret_cast<uint4*>(Xd)[v] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// The keep mask itself, one byte per element (1 kept, 0 dropped), n % 4 == 0.
__global__ void __launch_bounds__(kDropThreads)
    k_dropout_mask(uint8_t* __restrict__ keep, int64_t n, uint64_t seed, uint64_t thr) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kDropThreads;
  for (int64_t q = static_cast<int64_t>(blockIdx.x) * kDropThreads + threadIdx.x; q * 4 < n; q += stride) {
    const uint32_t b = dropout_keep4(q, seed, thr);
    reinterpret_cast<uint32_t*>(keep)[q] = (b & 1u) | ((b & 2u) << 7) | ((b & 4u) << 14) | ((b & 8u) << 21);
  }
}

// dX [M, K] = bf16( dXf + c (G A)[m, k] keep[m, k] ),  c = s / (1 - p),
// with (G A)[m, k] = sum_j G[m, j] A[j, k] in fp32 in j order and dXf the
// frozen-path product dY W^ in fp32.  Thread = 8 consecutive k of one row
// (K % 64 == 0, so a row holds whole groups of 8).
__global__ void __launch_bounds__(kDropThreads)
    k_dropout_dx(const float* __restrict__ dXf, const float* __restrict__ G, const __nv_bfloat16* __restrict__ A,
                 int64_t M, int64_t K, int r, float c, uint64_t seed, uint64_t thr, __nv_bfloat16* __restrict__ dX) {
  const int64_t groups = M * (K / 8);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kDropThreads;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * kDropThreads + threadIdx.x; v < groups; v += stride) {
    const int64_t m = v / (K / 8), k0 = (v - m * (K / 8)) * 8;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    const float* g = G + m * r;
    for (int j = 0; j < r; ++j) {
      const float gj = __ldg(g + j);
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(A + j * K + k0));
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(gj, __uint_as_float(aw[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = fmaf(gj, __uint_as_float(aw[i] & 0xFFFF0000u), acc[2 * i + 1]);
      }
    }
    const int64_t e = m * K + k0;   // a multiple of 8: two whole Philox blocks
    const uint32_t keep = dropout_keep4(e / 4, seed, thr) | (dropout_keep4(e / 4 + 1, seed, thr) << 4);
    const float4 f0 = __ldg(reinterpret_cast<const float4*>(dXf + e));
    const float4 f1 = __ldg(reinterpret_cast<const float4*>(dXf + e) + 1);
    const float base[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float y0 = base[2 * i], y1 = base[2 * i + 1];
      if ((keep >> (2 * i)) & 1u) y0 = __fadd_rn(y0, __fmul_rn(c, acc[2 * i]));
      if ((keep >> (2 * i + 1)) & 1u) y1 = __fadd_rn(y1, __fmul_rn(c, acc[2 * i + 1]));
      out[i] = pack_bf16x2(y0, y1);
    }
    *reinterpret_cast<uint4*>(dX + e) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

}  // namespace qlora
