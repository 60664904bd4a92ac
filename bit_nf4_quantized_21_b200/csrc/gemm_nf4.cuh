// gemm_nf4.cuh -- the fused NF4 GEMM on tcgen05 tensor cores (K3 forward,
// K4 backward-dX), with the LoRA product folded into the same accumulator.
//
//   forward : Y [M, N]  = X [M, K] . W^[N, K]^T  + (s T) [M, r] . B [N, r]^T
//   dX      : dX [M, K] = dY [M, N] . W^[N, K]   + (s G) [M, r] . A [r, K]
//
// W^ never exists in global memory: each 64-wide slice of the contraction is
// dequantised from the packed codes straight into the swizzled shared-memory
// layout the tensor core reads, used for one pipeline stage and overwritten.
// The adapter product is extra contraction steps of the same tcgen05
// accumulator, with s*T carried as two bf16 terms (hi = bf16(sT),
// lo = bf16(sT - hi)):  [X | sT_hi | sT_lo] . [W^ | B | B]^T.  Every output
// is one fp32 sum rounded once to bf16, and the adapter term keeps ~16
// mantissa bits of s*T.
//
// CTA tile: 128 activation rows x 256 output columns, contraction stage 64.
// Warp roles (320 threads):
//   warp 0      TMA producer: activation tile + packed-code tile per stage
//               (or the adapter tiles in the trailing LoRA stages)
//   warp 1      TMEM allocator and single-thread MMA issuer
//   warps 2..9  dequantisers during the main loop (one 64-weight block per
//               thread per stage), then the epilogue (TMEM -> bf16 -> global)
//
// Shared-memory tiles are 1024-byte aligned and use the 128-byte swizzle.
// The dequantised tile is written the same way in both modes -- one 128-byte
// row per (weight row n, 64-column block) -- and is read as a K-major B
// operand in the forward (rows = output n) and as an MN-major B operand in
// dX (rows = contraction n, 64-element MN atoms = output k).
#pragma once
#include "nf4_decode.cuh"

namespace qlora {

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 64;
constexpr int kGemmStages = 4;
constexpr int kGemmThreads = 320;
constexpr int kGemmDeqThreads = 256;
constexpr uint32_t kGemmABytes = kGemmBM * kGemmBK * 2;   // 16 KB activations
constexpr uint32_t kGemmWBytes = kGemmBN * kGemmBK * 2;   // 32 KB dequantised bf16
constexpr uint32_t kGemmCBytes = kGemmBN * kGemmBK / 2;   //  8 KB packed codes
constexpr uint32_t kGemmStageBytes = kGemmABytes + kGemmWBytes + kGemmCBytes;
constexpr uint32_t kGemmSmemBytes = kGemmStages * kGemmStageBytes + 1024 /*align*/ + 256 /*bars*/;
constexpr uint32_t kGemmTmemCols = 256;

enum GemmMode : int { kModeFwd = 0, kModeDx = 1 };

struct GemmArgs {
  // weight format
  const uint8_t* q8;
  const float* s2;
  const float* absmax_f32;
  int dq;
  int64_t wN, wK;        // weight rows (N) and columns (K)
  // problem
  int64_t M;             // activation rows
  int64_t out_cols;      // N (fwd) or K (dX)
  int64_t ldo;           // leading dimension of out
  __nv_bfloat16* out;
  float* out_f32;        // when non-null, the output goes here in fp32 instead (unrounded)
  int num_kt;            // contraction stages over the weight
  int lora_r16;          // adapter rank rounded up to 16 (0: no adapter)
  int64_t lora_lo_row;   // row of the adapter operand where the lo plane starts (= M)
  int* status;
  int tma_out;           // 2-SM kernel: 1 when its tm_out maps `out` (bf16, 64 x 32 boxes, 128-byte swizzle)
};

// Output columns [gc, gc + 16) of row `row` (fp32 accumulator words r):
// rounded once to bf16 into args.out, or kept fp32 in args.out_f32.
__device__ __forceinline__ void gemm_store16(const GemmArgs& args, int64_t row, int64_t gc, const uint32_t (&r)[16]) {
  const bool whole = gc + 16 <= args.out_cols;
  if (args.out_f32) {
    float* dst = args.out_f32 + row * args.ldo + gc;
    if (whole && (args.ldo & 3) == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) reinterpret_cast<uint4*>(dst)[i] = make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
    } else {
      for (int i = 0; i < 16 && gc + i < args.out_cols; ++i) dst[i] = __uint_as_float(r[i]);
    }
    return;
  }
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
  __nv_bfloat16* dst = args.out + row * args.ldo + gc;
  if (whole && (args.ldo & 7) == 0) {
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  } else {
    const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(pk);
    for (int i = 0; i < 16 && gc + i < args.out_cols; ++i) dst[i] = hv[i];
  }
}

struct GemmSmem {
  uint8_t* base;  // 1024-aligned
  __device__ __forceinline__ uint8_t* a(int s) const { return base + s * kGemmStageBytes; }
  __device__ __forceinline__ uint8_t* w(int s) const { return a(s) + kGemmABytes; }
  __device__ __forceinline__ uint8_t* c(int s) const { return w(s) + kGemmWBytes; }
};

template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm_nf4(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_codes,
               const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_lb,
               const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  GemmSmem sm;
  sm.base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm.base + kGemmStages * kGemmStageBytes);
  uint64_t* full_a = bars;                       // [S] TMA landed (activations + codes / adapters)
  uint64_t* full_b = bars + kGemmStages;         // [S] dequantised tile written
  uint64_t* empty = bars + 2 * kGemmStages;      // [S] MMA finished reading the stage
  uint64_t* acc_full = bars + 3 * kGemmStages;   // accumulator complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * kGemmStages + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kGemmBM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kGemmBN;   // output-column tile origin
  const int nl1 = (args.lora_r16 + 63) / 64;   // adapter stages per plane
  const int num_lt = 2 * nl1;                  // hi plane, then lo plane
  const int total = args.num_kt + num_lt;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(smem_u32(&full_a[s]), 1);
      mbar_init(smem_u32(&full_b[s]), kGemmDeqThreads);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(acc_full), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_act);
    tma_prefetch_desc(&tm_codes);
    if (num_lt) { tma_prefetch_desc(&tm_la); tma_prefetch_desc(&tm_lb); }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kGemmTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < total; ++it) {
        const int s = it % kGemmStages;
        if (it >= kGemmStages &&
            !mbar_wait(smem_u32(&empty[s]), ((it / kGemmStages) + 1) & 1, abort_flag, args.status))
          break;
        const uint32_t fa = smem_u32(&full_a[s]);
        if (it < args.num_kt) {
          mbar_arrive_expect_tx(fa, kGemmABytes + kGemmCBytes);
          if (MODE == kModeFwd) {
            tma_load_2d(smem_u32(sm.a(s)), &tm_act, fa, it * kGemmBK, static_cast<int32_t>(m0));
            tma_load_2d(smem_u32(sm.c(s)), &tm_codes, fa, it * (kGemmBK / 2), static_cast<int32_t>(n0));
          } else {
            tma_load_2d(smem_u32(sm.a(s)), &tm_act, fa, it * kGemmBK, static_cast<int32_t>(m0));
            tma_load_2d(smem_u32(sm.c(s)), &tm_codes, fa, static_cast<int32_t>(n0 / 2), it * kGemmBK);
          }
        } else {
          const int lt = it - args.num_kt;
          const int li = lt % nl1;
          const int64_t arow = (lt / nl1) * args.lora_lo_row + m0;
          mbar_arrive_expect_tx(fa, kGemmABytes + kGemmWBytes);
          tma_load_2d(smem_u32(sm.a(s)), &tm_la, fa, li * 64, static_cast<int32_t>(arow));
          if (MODE == kModeFwd) {
            tma_load_2d(smem_u32(sm.w(s)), &tm_lb, fa, li * 64, static_cast<int32_t>(n0));
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tma_load_2d(smem_u32(sm.w(s)) + j * 8192, &tm_lb, fa, static_cast<int32_t>(n0) + 64 * j, li * 64);
          }
        }
        ++issued;
      }
      if (*abort_flag) {
        // drain loads still in flight before the CTA may exit
        for (int it = max(0, issued - kGemmStages); it < issued; ++it) {
          const uint32_t fa = smem_u32(&full_a[it % kGemmStages]);
          const uint64_t t0 = global_ns();
          while (!mbar_try_wait(fa, (it / kGemmStages) & 1) && global_ns() - t0 < qlora_drain_limit()) {}
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kGemmBM, kGemmBN, 0, MODE == kModeDx ? 1 : 0);
      for (int it = 0; it < total; ++it) {
        const int s = it % kGemmStages;
        const uint32_t par = (it / kGemmStages) & 1;
        if (!mbar_wait(smem_u32(&full_a[s]), par, abort_flag, args.status)) break;
        if (!mbar_wait(smem_u32(&full_b[s]), par, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(sm.a(s));
        const uint32_t w_base = smem_u32(sm.w(s));
        const int nk = (it < args.num_kt) ? 4 : min(4, (args.lora_r16 - ((it - args.num_kt) % nl1) * 64) / 16);
        for (int k = 0; k < nk; ++k) {
          const uint64_t adesc = sw128_desc(a_base + k * 32, 16, 1024);
          const uint64_t bdesc = (MODE == kModeFwd) ? sw128_desc(w_base + k * 32, 16, 1024)
                                                    : sw128_desc(w_base + k * 2048, 8192, 1024);
          umma_bf16(tmem_d, adesc, bdesc, idesc, (it > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(smem_u32(&empty[s]));
      }
      // always signal the epilogue: it must not free TMEM under running MMAs
      umma_commit(smem_u32(acc_full));
    }
  } else {
    // ------------------------------------------------------- dequantisers
    const int t = threadIdx.x - 64;  // 0..255
    int64_t wn;                      // weight row of this thread's block
    int64_t kb;                      // 64-column block index within the weight row
    int64_t kb_step, wn_step;
    uint32_t crow_off, wrow_off, cswz, wswz;
    const int64_t KB = args.wK / 64;
    if (MODE == kModeFwd) {
      wn = n0 + t; kb = 0; kb_step = 1; wn_step = 0;
      crow_off = t * 32; cswz = (t >> 2) & 1;          // codes: 32-byte rows, 32-byte swizzle
      wrow_off = t * 128; wswz = t & 7;
    } else {
      const int nl = t & 63, j = t >> 6;
      wn = nl; kb = n0 / 64 + j; kb_step = 0; wn_step = 64;
      crow_off = nl * 128 + j * 32; cswz = nl & 7;      // codes: 128-byte rows, 128-byte swizzle
      wrow_off = j * 8192 + nl * 128; wswz = nl & 7;
    }
    // block scale of the first stage, then one stage ahead
    auto scale_of = [&](int64_t n, int64_t k) -> float {
      if (n >= args.wN || k >= KB) return 0.0f;
      return nf4_block_scale(args.q8, args.s2, args.absmax_f32, args.dq, n * KB + k);
    };
    float scale_next = (args.num_kt > 0) ? scale_of(wn, kb) : 0.0f;
    for (int it = 0; it < total; ++it) {
      const int s = it % kGemmStages;
      const float scale = scale_next;
      const bool valid = (wn < args.wN) && (kb < KB);
      if (!mbar_wait(smem_u32(&full_a[s]), (it / kGemmStages) & 1, abort_flag, args.status)) break;
      if (it < args.num_kt) {
        uint8_t* wdst = sm.w(s) + wrow_off;
        if (valid) {
          const uint8_t* csrc = sm.c(s) + crow_off;
          uint4 c0, c1;
          if (MODE == kModeFwd) {
            c0 = *reinterpret_cast<const uint4*>(csrc + ((0u ^ cswz) << 4));
            c1 = *reinterpret_cast<const uint4*>(csrc + ((1u ^ cswz) << 4));
          } else {
            // logical 16-byte chunks 2j, 2j+1 of a 128-byte swizzled row
            const uint32_t row_base = crow_off & ~127u;
            const uint32_t ch = (crow_off & 127u) >> 4;
            c0 = *reinterpret_cast<const uint4*>(sm.c(s) + row_base + (((ch + 0) ^ cswz) << 4));
            c1 = *reinterpret_cast<const uint4*>(sm.c(s) + row_base + (((ch + 1) ^ cswz) << 4));
          }
          const NF4Table tab = nf4_table(scale);
          const NF4Shr sh = nf4_shr();
          const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t o[4];
            nf4_decode8(cw[c], tab, o, sh);
            *reinterpret_cast<uint4*>(wdst + ((static_cast<uint32_t>(c) ^ wswz) << 4)) =
                make_uint4(o[0], o[1], o[2], o[3]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(wdst + (c << 4)) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      mbar_arrive(smem_u32(&full_b[s]));
      // next stage's scale, loaded after the arrive so its release does not wait on it
      if (it + 1 < args.num_kt) scale_next = scale_of(wn + wn_step, kb + kb_step);
      wn += wn_step;
      kb += kb_step;
    }

    // ------------------------------------------------------------ epilogue
    {
      // bounded wait that ignores the abort flag: MMAs may still be running
      const uint32_t bar = smem_u32(acc_full);
      const uint64_t t0 = global_ns(), limit = qlora_wait_limit();
      bool ok = true;
      while (!mbar_try_wait(bar, 0)) {
        if (global_ns() - t0 > limit) { ok = false; break; }
      }
      if (!ok) {
        *abort_flag = 1;
        if (args.status) atomicOr(args.status, QLORA_DEV_TIMEOUT);
      }
    }
    tc_fence_after();
    if (!*abort_flag) {
      const int q = warp & 3;              // TMEM lane quarter this warp may read
      const int half = (warp - 2) >> 2;    // column half
      const int64_t row = m0 + q * 32 + lane;
      const uint32_t taddr = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        const int col = half * 128 + c * 16;
        uint32_t r[16];
        tmem_ld16(taddr + col, r);
        tmem_ld_wait();
        const int64_t gc = n0 + col;
        if (row < args.M && gc < args.out_cols) gemm_store16(args, row, gc, r);
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
    tmem_dealloc(tmem_d, kGemmTmemCols);
  }
}

}  // namespace qlora
