// skinny.cuh -- the rank-r adapter products on tcgen05 tensor cores.
//
// One kernel computes C[p, q] = sum_j Aop(p, j) * Bop(q, j) for a tall
// operand (P rows) against a narrow one (Q <= 256 columns per CTA), split
// over the contraction j across CTAs; each CTA writes its fp32 partial tile
// and a finishing kernel adds the splits in a fixed order (deterministic, no
// float atomics).  The four uses (s = alpha/r):
//
//   T  = X A^T     p = token m,  j = k,  Aop = X   (K-major), Bop = A (K-major)
//   G  = dY B      p = token m,  j = n,  Aop = dY  (K-major), Bop = B (MN-major)
//   dA = s G^T X   p = k,        j = m,  Aop = X^T (MN-major), Bop = [G_hi|G_lo] (MN-major)
//   dB = s dY^T T  p = n,        j = m,  Aop = dY^T (MN-major), Bop = [T_hi|T_lo] (MN-major)
//
// For dA and dB the fp32 G and T are split into two bf16 terms (hi = bf16(v),
// lo = bf16(v - hi)) that share one accumulator, so the adapter gradients
// carry ~16 mantissa bits of G and T instead of bf16's 8.
//
// Tile: 128 rows of P, one 64-deep contraction chunk per pipeline stage.
// Warps: 0 = TMA producer, 1 = TMEM allocator + MMA issuer, 2..5 = epilogue.
#pragma once
#include "ptx.cuh"

namespace qlora {

constexpr int kSkBM = 128;
constexpr int kSkThreads = 192;
constexpr uint32_t kSkABytes = kSkBM * 64 * 2;   // 16 KB

struct SkinnyArgs {
  int64_t P;          // rows of C
  int Qn;             // columns of C handled by one CTA (multiple of 16; of 64 for MN-major B)
  int64_t Qtot;       // leading dimension of the partial buffer
  int num_chunks;     // 64-deep contraction chunks in total
  int chunks_per_split;
  int stages;
  float* partial;     // [splits][P][Qtot]
  int* status;
};

template <int A_MN, int B_MN>
__global__ void __launch_bounds__(kSkThreads, 1)
    k_skinny(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
             const SkinnyArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = args.stages;
  const uint32_t b_bytes = static_cast<uint32_t>(args.Qn) * 128u;
  const uint32_t stage_bytes = kSkABytes + b_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + S * stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* acc_full = bars + 2 * S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t p0 = static_cast<int64_t>(blockIdx.x) * kSkBM;
  const int q0 = blockIdx.z * 256;
  const int split = blockIdx.y;
  const int c_begin = split * args.chunks_per_split;
  const int nch = min(args.num_chunks, c_begin + args.chunks_per_split) - c_begin;
  const int qv = min(args.Qn, static_cast<int>(args.Qtot - q0));   // valid columns of this chunk
  const uint32_t tcols = args.Qn <= 32 ? 32u : (args.Qn <= 64 ? 64u : (args.Qn <= 128 ? 128u : 256u));

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(acc_full), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < nch; ++it) {
        const int s = it % S;
        if (it >= S && !mbar_wait(smem_u32(&empty[s]), ((it / S) + 1) & 1, abort_flag, args.status)) break;
        const uint32_t fb = smem_u32(&full[s]);
        const uint32_t a_dst = smem_u32(base + s * stage_bytes);
        const uint32_t b_dst = a_dst + kSkABytes;
        const int j0 = (c_begin + it) * 64;
        mbar_arrive_expect_tx(fb, stage_bytes);
        if (A_MN) {
          tma_load_2d(a_dst, &tm_a, fb, static_cast<int32_t>(p0), j0);
          tma_load_2d(a_dst + 8192, &tm_a, fb, static_cast<int32_t>(p0) + 64, j0);
        } else {
          tma_load_2d(a_dst, &tm_a, fb, j0, static_cast<int32_t>(p0));
        }
        if (B_MN) {
          for (int h = 0; h < args.Qn / 64; ++h) tma_load_2d(b_dst + h * 8192, &tm_b, fb, q0 + 64 * h, j0);
        } else {
          tma_load_2d(b_dst, &tm_b, fb, j0, q0);
        }
        ++issued;
      }
      if (*abort_flag) {
        for (int it = max(0, issued - S); it < issued; ++it) {
          const uint32_t fb = smem_u32(&full[it % S]);
          const uint64_t t0 = global_ns();
          while (!mbar_try_wait(fb, (it / S) & 1) && global_ns() - t0 < 200000000ull) {}
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kSkBM, args.Qn, A_MN, B_MN);
      for (int it = 0; it < nch; ++it) {
        const int s = it % S;
        if (!mbar_wait(smem_u32(&full[s]), (it / S) & 1, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(base + s * stage_bytes);
        const uint32_t b_base = a_base + kSkABytes;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t ad = A_MN ? sw128_desc(a_base + k * 2048, 8192, 1024) : sw128_desc(a_base + k * 32, 16, 1024);
          const uint64_t bd = B_MN ? sw128_desc(b_base + k * 2048, 8192, 1024) : sw128_desc(b_base + k * 32, 16, 1024);
          umma_bf16(tmem_d, ad, bd, idesc, (it > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(smem_u32(&empty[s]));
      }
      umma_commit(smem_u32(acc_full));
    }
  } else {
    {
      const uint32_t bar = smem_u32(acc_full);
      const uint64_t t0 = global_ns();
      bool ok = true;
      while (!mbar_try_wait(bar, 0)) {
        if (global_ns() - t0 > QLORA_WAIT_NS) { ok = false; break; }
      }
      if (!ok) {
        *abort_flag = 1;
        if (args.status) atomicOr(args.status, QLORA_DEV_TIMEOUT);
      }
    }
    tc_fence_after();
    if (!*abort_flag && nch > 0) {
      const int q = warp & 3;
      const int64_t row = p0 + q * 32 + lane;
      const uint32_t taddr = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
      float* dst = args.partial + (static_cast<int64_t>(split) * args.P + row) * args.Qtot + q0;
#pragma unroll 1
      for (int c = 0; c < qv / 16; ++c) {
        uint32_t r[16];
        tmem_ld16(taddr + c * 16, r);
        tmem_ld_wait();
        if (row < args.P) {
          float4* d4 = reinterpret_cast<float4*>(dst + c * 16);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            d4[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
        }
      }
    }
  }

  // Single-lane roles (producer, MMA issuer) leave their warps diverged;
  // the CTA/cluster barrier below is warp-aligned, so every warp first
  // reconverges here -- otherwise the barrier can complete while a lane is
  // still working and TMEM could be released under it.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, tcols);
  }
}

// ---------------------------------------------------------------- finishing

// Token-indexed results (T or G): v[m, i] = sum over splits of src.
// Writes (each optional): f32 [M, r]; s_bf16 [2M, r8]: rows 0..M-1 hold
// bf16(s*v), rows M..2M-1 the remainder bf16(s*v - bf16(s*v)), zero padded;
// hl [M, Qh] = [bf16(v) | bf16(v - bf16(v))] at columns [0, r) and
// [r16, r16 + r), zeros elsewhere.
__global__ void k_finish_rows(const float* __restrict__ src, int64_t src_ld, int splits,
                              int64_t split_stride, int64_t M, int r, int r8, int r16, int Qh,
                              float s, float* __restrict__ f32, __nv_bfloat16* __restrict__ s_bf16,
                              __nv_bfloat16* __restrict__ hl) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int width = max(r16, Qh - 2 * r16);
  const int64_t m = idx / width;
  const int i = static_cast<int>(idx % width);
  if (m >= M) return;
  if (i < r16) {
    float v = 0.0f;
    if (i < r) {
      for (int sp = 0; sp < splits; ++sp) v += src[sp * split_stride + m * src_ld + i];
    }
    if (f32 && i < r) f32[m * r + i] = v;
    if (s_bf16 && i < r8) {
      const float sv = s * v;
      const __nv_bfloat16 h = __float2bfloat16_rn(sv);
      s_bf16[m * r8 + i] = h;
      s_bf16[(M + m) * r8 + i] = __float2bfloat16_rn(sv - __bfloat162float(h));
    }
    if (hl) {
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      hl[m * Qh + i] = h;
      hl[m * Qh + r16 + i] = __float2bfloat16_rn(v - __bfloat162float(h));
    }
  }
  if (hl && i < Qh - 2 * r16) hl[m * Qh + 2 * r16 + i] = __float2bfloat16_rn(0.0f);
}

// Gradient results: for row p of C (p = k for dA, p = n for dB),
// g[p, i] = s * sum over splits (C[p, i] + C[p, r16 + i]).  dA is stored
// transposed ([r, K]), dB as is ([N, r]).  Shared-memory transpose tile of
// 32 rows x 32 ranks.
__global__ void k_finish_grad(const float* __restrict__ partial, int64_t Qtot, int splits, int64_t P,
                              int r, int r16, float s, int transpose, int out_bf16, void* out) {
  __shared__ float tile[32][33];
  const int64_t p0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int i0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8 threads
  for (int yy = ty; yy < 32; yy += 8) {
    const int64_t p = p0 + yy;
    const int i = i0 + tx;
    float v = 0.0f;
    if (p < P && i < r) {
      for (int sp = 0; sp < splits; ++sp) {
        const float* row = partial + (static_cast<int64_t>(sp) * P + p) * Qtot;
        v += row[i] + row[r16 + i];
      }
      v *= s;
    }
    tile[yy][tx] = v;
  }
  __syncthreads();
  for (int yy = ty; yy < 32; yy += 8) {
    if (transpose) {
      const int i = i0 + yy;
      const int64_t p = p0 + tx;
      if (i < r && p < P) {
        const float v = tile[tx][yy];
        if (out_bf16) static_cast<__nv_bfloat16*>(out)[i * P + p] = __float2bfloat16_rn(v);
        else static_cast<float*>(out)[i * P + p] = v;
      }
    } else {
      const int64_t p = p0 + yy;
      const int i = i0 + tx;
      if (i < r && p < P) {
        const float v = tile[yy][tx];
        if (out_bf16) static_cast<__nv_bfloat16*>(out)[p * r + i] = __float2bfloat16_rn(v);
        else static_cast<float*>(out)[p * r + i] = v;
      }
    }
  }
}

// Copy B [N, r] into a zero-padded [N, r8] buffer (only when r % 8 != 0, so
// that its rows are 16-byte multiples for the tensor maps).
__global__ void k_pad_cols(const __nv_bfloat16* __restrict__ src, int64_t rows, int r, int r8,
                           __nv_bfloat16* __restrict__ dst) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= rows * r8) return;
  const int64_t n = idx / r8;
  const int i = static_cast<int>(idx % r8);
  dst[idx] = (i < r) ? src[n * r + i] : __float2bfloat16_rn(0.0f);
}

}  // namespace qlora
