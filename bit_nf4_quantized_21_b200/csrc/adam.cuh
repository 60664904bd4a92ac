// adam.cuh -- the adapter optimiser step: Adam with fp32 state.
//
// "QLoRA" (infra.bea.ai), "How QLoRA Works", precision table: the adapters
// A, B and their gradients are bf16 and the optimiser (Adam) keeps fp32
// state, 12 bytes per adapter parameter -- an fp32 master copy and the two
// moments.  The pages print no update rule; this is Adam as published
// (Kingma & Ba: moment averages with bias correction), with optional
// decoupled weight decay (AdamW, Loshchilov & Hutter) applied to the
// master copy before the moment step.  Per element, in this order, all
// fp32 with IEEE rounding:
//   g      = grad * grad_scale
//   theta  = master * decay                 (decay = 1 - lr * weight_decay)
//   m      = beta1 * m + (1 - beta1) * g
//   v      = beta2 * v + (1 - beta2) * g * g
//   denom  = sqrt(v) * rsqrt_bc2 + eps      (rsqrt_bc2 = 1 / sqrt(1 - beta2^t))
//   master = theta - step_size * (m / denom)   (step_size = lr / (1 - beta1^t))
//   param  = bf16_rne(master)               (when a bf16 copy is kept)
// The per-step scalars (decay, step_size, rsqrt_bc2) are computed once on
// the host in double precision and rounded to fp32.
//
// HBM-bound elementwise work: 4 elements per thread per iteration with
// 16-byte loads and stores, grid-stride over a grid sized to the SM count.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "ptx.cuh"

namespace qlora {

constexpr int kAdamThreads = 256;

struct AdamArgs {
  float* master;               // [n] fp32, updated in place
  float* m;                    // [n] fp32 first moment
  float* v;                    // [n] fp32 second moment
  __nv_bfloat16* param;        // [n] bf16 copy of master (nullable)
  const void* grad;            // [n] fp32 or bf16
  int grad_bf16;
  int64_t n;
  float grad_scale, decay, beta1, one_minus_beta1, beta2, one_minus_beta2, eps, step_size, rsqrt_bc2;
  int* status;
};

__device__ __forceinline__ float adam_one(const AdamArgs& a, float g, float& master, float& m, float& v, bool& bad) {
  g = __fmul_rn(g, a.grad_scale);
  bad |= !isfinite(g);
  const float theta = __fmul_rn(master, a.decay);
  m = __fadd_rn(__fmul_rn(a.beta1, m), __fmul_rn(a.one_minus_beta1, g));
  v = __fadd_rn(__fmul_rn(a.beta2, v), __fmul_rn(a.one_minus_beta2, __fmul_rn(g, g)));
  const float denom = __fadd_rn(__fmul_rn(__fsqrt_rn(v), a.rsqrt_bc2), a.eps);
  master = __fsub_rn(theta, __fmul_rn(a.step_size, __fdiv_rn(m, denom)));
  return master;
}

__device__ __forceinline__ float adam_grad(const AdamArgs& a, int64_t i) {
  if (a.grad_bf16) return __bfloat162float(static_cast<const __nv_bfloat16*>(a.grad)[i]);
  return static_cast<const float*>(a.grad)[i];
}

__global__ void __launch_bounds__(kAdamThreads) k_adam_step(const AdamArgs a) {
  const int64_t n4 = a.n / 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  bool bad = false;
  for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < n4; q += stride) {
    float4 w = reinterpret_cast<const float4*>(a.master)[q];
    float4 m = reinterpret_cast<const float4*>(a.m)[q];
    float4 v = reinterpret_cast<const float4*>(a.v)[q];
    float g[4];
    if (a.grad_bf16) {
      const uint2 gb = reinterpret_cast<const uint2*>(a.grad)[q];
      g[0] = __uint_as_float(gb.x << 16); g[1] = __uint_as_float(gb.x & 0xFFFF0000u);
      g[2] = __uint_as_float(gb.y << 16); g[3] = __uint_as_float(gb.y & 0xFFFF0000u);
    } else {
      const float4 gf = reinterpret_cast<const float4*>(a.grad)[q];
      g[0] = gf.x; g[1] = gf.y; g[2] = gf.z; g[3] = gf.w;
    }
    adam_one(a, g[0], w.x, m.x, v.x, bad);
    adam_one(a, g[1], w.y, m.y, v.y, bad);
    adam_one(a, g[2], w.z, m.z, v.z, bad);
    adam_one(a, g[3], w.w, m.w, v.w, bad);
    reinterpret_cast<float4*>(a.master)[q] = w;
    reinterpret_cast<float4*>(a.m)[q] = m;
    reinterpret_cast<float4*>(a.v)[q] = v;
    if (a.param) {
      const __nv_bfloat162 p01 = __floats2bfloat162_rn(w.x, w.y), p23 = __floats2bfloat162_rn(w.z, w.w);
      uint2 pb;
      pb.x = *reinterpret_cast<const uint32_t*>(&p01);
      pb.y = *reinterpret_cast<const uint32_t*>(&p23);
      reinterpret_cast<uint2*>(a.param)[q] = pb;
    }
  }
  // the ragged tail (n % 4 elements), one per thread of the first block
  if (blockIdx.x == 0 && threadIdx.x < static_cast<unsigned>(a.n - 4 * n4)) {
    const int64_t i = 4 * n4 + threadIdx.x;
    float w = a.master[i], m = a.m[i], v = a.v[i];
    adam_one(a, adam_grad(a, i), w, m, v, bad);
    a.master[i] = w; a.m[i] = m; a.v[i] = v;
    if (a.param) a.param[i] = __float2bfloat16_rn(w);
  }
  if (bad && a.status) atomicOr(a.status, QLORA_DEV_NONFINITE);
}

}  // namespace qlora
