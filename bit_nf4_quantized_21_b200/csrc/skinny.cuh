// skinny.cuh -- the rank-r adapter products on tcgen05 tensor cores.
//
// One kernel computes C[p, q] = sum_j Aop(p, j) * Bop(q, j) for a tall
// operand (P rows) against a narrow one (Q <= 256 columns per CTA), split
// over the contraction j across CTAs, and finishes the result itself: when
// a tile is split, each CTA writes its fp32 partial, counts itself in on the
// tile's counter, and the last CTA to arrive adds the partials in split
// order (deterministic, no float atomics) and applies the final transform.
// One launch may carry two independent problems (dA and dB).  The four uses
// (s = alpha/r):
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
// Final transforms:
//   rows (T, G), row m:  v[i] (i < r; 0 above) ->  f32 [M, r] = v;
//     s_bf16 [2M, r8]: row m = bf16(s v), row M + m = bf16(s v - bf16(s v));
//     hl [M, Qh] = [bf16(v) | bf16(v - bf16(v))] at [0, r16) and [r16, 2 r16),
//     zeros in [2 r16, Qh).  (Each output optional.)
//   grad (dA, dB), row p:  g[p, i] = s * sum over splits (C[p, i] + C[p, r16 + i]),
//     stored transposed ([r, P], dA) or not ([P, r], dB), fp32 or bf16.
// A rows launch can also carry a side task: T [rows, r] fp32 -> hl planes,
// for the backward's dB operand, shared out over the launch's CTAs.
//
// Tile: 128 rows of P, one 64-deep contraction chunk per pipeline stage.
// Warps: 0 = TMA producer, 1 = TMEM allocator + MMA issuer, 2..5 = epilogue.
#pragma once
#include "ptx.cuh"

namespace qlora {

constexpr int kSkBM = 128;
constexpr int kSkThreads = 192;
constexpr uint32_t kSkABytes = kSkBM * 64 * 2;   // 16 KB

enum SkFinish : int { kFinRows = 0, kFinGrad = 1 };

struct SkinnyArgs {
  // the product
  int64_t P;          // rows of C
  int Qn;             // columns of C handled by one CTA (multiple of 16; of 64 for MN-major B)
  int64_t Qtot;       // columns of C (leading dimension of the partial buffer)
  int num_chunks;     // 64-deep contraction chunks in total
  int chunks_per_split;
  int stages;
  int ptiles, splits, qchunks;   // CTA grid of this problem: ptiles x splits x qchunks
  float* partial;     // [splits][P][Qtot], used when splits * qchunks > 1
  int64_t partial_elems;   // floats the partial buffer holds (range checks of the debug build)
  unsigned int* cnt;  // [ptiles] arrival counters, zero on entry (when splits * qchunks > 1)
  int* status;
  // the final transform
  int finish;         // kFinRows or kFinGrad
  float s;
  float vscale;       // rows: every value is multiplied by this first (1 / (1 - p) under dropout, else 1)
  int r, r8, r16, Qh;
  float* f32;                      // rows
  __nv_bfloat16* s_bf16;           // rows
  __nv_bfloat16* hl;               // rows
  int transpose, out_bf16;         // grad
  void* out;                       // grad
  const float* side_src;           // rows side task (nullable): [side_rows, r] fp32
  int64_t side_rows;
  __nv_bfloat16* side_hl;          // [side_rows, Qh]
};

__device__ __forceinline__ void sk_bar(uint32_t threads) {
  asm volatile("bar.sync 1, %0;" ::"r"(threads) : "memory");
}
// Named barrier 1 that also ANDs a predicate over the participating threads.
__device__ __forceinline__ bool sk_bar_and(uint32_t threads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(threads)
      : "memory");
  return r != 0;
}

// bf16 hi / lo terms of 16 values, packed 2 per word (hi = bf16(x),
// lo = bf16(x - hi)).
__device__ __forceinline__ void sk_hilo16(const float (&x)[16], uint32_t (&hi)[8], uint32_t (&lo)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    hi[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
    const float h0 = __uint_as_float(hi[i] << 16), h1 = __uint_as_float(hi[i] & 0xFFFF0000u);
    lo[i] = pack_bf16x2(x[2 * i] - h0, x[2 * i + 1] - h1);
  }
}
// 8 bf16 (one 16-byte store); `n` < 8 stores only the first n.
__device__ __forceinline__ void sk_st8(__nv_bfloat16* dst, const uint32_t* w, int n) {
  if (n >= 8) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(w);
    for (int i = 0; i < n; ++i) dst[i] = h[i];
  }
}

// Rows transform of 16 columns [c0, c0 + 16) of row m.  Each thread owns a
// row, so the outputs go out as 16-byte stores (row offsets are multiples of
// 16 bytes: r8 and r16 are multiples of 8 and 16, Qh of 64; fp32 T takes
// the vector path when r % 4 == 0).  Values of columns >= r are zero.
__device__ __forceinline__ void sk_rows_out(const SkinnyArgs& a, int64_t m, int c0, const float (&v0)[16]) {
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = v0[i] * a.vscale;
  if (a.f32) {
    float* d = a.f32 + m * a.r + c0;
    if ((a.r & 3) == 0 && c0 + 16 <= a.r) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        reinterpret_cast<float4*>(d)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
      for (int i = 0; i < 16 && c0 + i < a.r; ++i) d[i] = v[i];
    }
  }
  if (a.s_bf16 && c0 < a.r8) {
    float sv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) sv[i] = a.s * v[i];
    uint32_t hi[8], lo[8];
    sk_hilo16(sv, hi, lo);
    const int n = min(16, a.r8 - c0);
    __nv_bfloat16* dh = a.s_bf16 + m * a.r8 + c0;
    __nv_bfloat16* dl = a.s_bf16 + (a.P + m) * a.r8 + c0;
    sk_st8(dh, hi, n);
    sk_st8(dl, lo, n);
    if (n > 8) { sk_st8(dh + 8, hi + 4, n - 8); sk_st8(dl + 8, lo + 4, n - 8); }
  }
  if (a.hl) {
    uint32_t hi[8], lo[8];
    sk_hilo16(v, hi, lo);
    __nv_bfloat16* dh = a.hl + m * a.Qh + c0;
    __nv_bfloat16* dl = dh + a.r16;
    sk_st8(dh, hi, 8); sk_st8(dh + 8, hi + 4, 8);
    sk_st8(dl, lo, 8); sk_st8(dl + 8, lo + 4, 8);
  }
}
// Zero columns [2 r16, Qh) of an hl row (a multiple of 32 bf16).
__device__ __forceinline__ void sk_hl_zero(__nv_bfloat16* row, int r16, int Qh) {
  for (int i = 2 * r16; i < Qh; i += 8) *reinterpret_cast<uint4*>(row + i) = make_uint4(0, 0, 0, 0);
}

// Grad transform of ranks [c0, c0 + 16) of row p from the hi and lo sums.
// Transposed (dA [r, P]): consecutive threads own consecutive p, so each
// store instruction of a warp is contiguous.  Not transposed (dB [P, r]):
// the row's ranks are contiguous, 16-byte stores when r allows.
__device__ __forceinline__ void sk_grad_out(const SkinnyArgs& a, int64_t p, int c0, const float (&g)[16]) {
  if (!a.transpose && c0 + 16 <= a.r && (a.r & 7) == 0) {
    if (a.out_bf16) {
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(g[2 * i], g[2 * i + 1]);
      __nv_bfloat16* d = static_cast<__nv_bfloat16*>(a.out) + p * a.r + c0;
      sk_st8(d, w, 8);
      sk_st8(d + 8, w + 4, 8);
    } else {
      float4* d = reinterpret_cast<float4*>(static_cast<float*>(a.out) + p * a.r + c0);
#pragma unroll
      for (int i = 0; i < 4; ++i) d[i] = make_float4(g[4 * i], g[4 * i + 1], g[4 * i + 2], g[4 * i + 3]);
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int gi = c0 + i;
    if (gi >= a.r) break;
    const int64_t o = a.transpose ? static_cast<int64_t>(gi) * a.P + p : p * a.r + gi;
    if (a.out_bf16) static_cast<__nv_bfloat16*>(a.out)[o] = __float2bfloat16_rn(g[i]);
    else static_cast<float*>(a.out)[o] = g[i];
  }
}

// Test hook (qlora_debug_inject_stall): when set, CTA 0 of the first problem
// of every adapter-product launch withholds the loads of its first stage, so
// that its MMA thread's bounded wait runs out and the launch takes its
// timeout path (status bit, early exit, TMEM released).
__device__ int g_qlora_inject_stall = 0;

template <int A_MN, int B_MN>
__global__ void __launch_bounds__(kSkThreads, 1)
    k_skinny(const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_b0,
             const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_b1,
             const __grid_constant__ SkinnyArgs a0, const __grid_constant__ SkinnyArgs a1, const int n0) {
  extern __shared__ uint8_t smem_raw[];
  const bool second = static_cast<int>(blockIdx.x) >= n0;
  const SkinnyArgs& args = second ? a1 : a0;
  const CUtensorMap* tm_a = second ? &tm_a1 : &tm_a0;
  const CUtensorMap* tm_b = second ? &tm_b1 : &tm_b0;
  const int bid = second ? static_cast<int>(blockIdx.x) - n0 : static_cast<int>(blockIdx.x);
  const int nctas = args.ptiles * args.splits * args.qchunks;
  const int ptile = bid % args.ptiles;
  const int split = (bid / args.ptiles) % args.splits;
  const int qchunk = bid / (args.ptiles * args.splits);

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
  volatile int* s_last = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // a fused GEMM launched behind this kernel may start its own work now
  // (it waits for this kernel's results only where it reads them)
  if (threadIdx.x == 0) griddep_launch_dependents();
  const int64_t p0 = static_cast<int64_t>(ptile) * kSkBM;
  const int q0 = qchunk * 256;
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
    tma_prefetch_desc(tm_a);
    tma_prefetch_desc(tm_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  if (threadIdx.x == 0)
    QLORA_CHECK_ONLY(static_cast<uint32_t>(S) * stage_bytes + (2 * S + 1) * 8 + 16 + 1023 <= dyn_smem_bytes(), 200);

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      const bool stall = bid == 0 && !second && *reinterpret_cast<volatile int*>(&g_qlora_inject_stall) != 0;
      for (int it = 0; it < nch; ++it) {
        const int s = it % S;
        if (it >= S && !mbar_wait(smem_u32(&empty[s]), ((it / S) + 1) & 1, abort_flag, args.status)) break;
        if (stall && it == 0) {   // test hook: this stage's loads are withheld
          ++issued;
          continue;
        }
        const uint32_t fb = smem_u32(&full[s]);
        const uint32_t a_dst = smem_u32(base + s * stage_bytes);
        const uint32_t b_dst = a_dst + kSkABytes;
        const int j0 = (c_begin + it) * 64;
        mbar_arrive_expect_tx(fb, stage_bytes);
        if (A_MN) {
          tma_load_2d(a_dst, tm_a, fb, static_cast<int32_t>(p0), j0);
          tma_load_2d(a_dst + 8192, tm_a, fb, static_cast<int32_t>(p0) + 64, j0);
        } else {
          tma_load_2d(a_dst, tm_a, fb, j0, static_cast<int32_t>(p0));
        }
        if (B_MN) {
          for (int h = 0; h < args.Qn / 64; ++h) tma_load_2d(b_dst + h * 8192, tm_b, fb, q0 + 64 * h, j0);
        } else {
          tma_load_2d(b_dst, tm_b, fb, j0, q0);
        }
        ++issued;
      }
      if (*abort_flag) {
        for (int it = max(0, issued - S); it < issued; ++it) {
          const uint32_t fb = smem_u32(&full[it % S]);
          const uint64_t t0 = global_ns();
          while (!mbar_try_wait(fb, (it / S) & 1) && global_ns() - t0 < qlora_drain_limit()) {}
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
    const int q = warp & 3;
    const int et = threadIdx.x - 64;                  // 0..127
    const int64_t row = p0 + q * 32 + lane;
    const uint32_t taddr = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
    const bool rows_mode = args.finish == kFinRows;
    const int nred = args.splits * args.qchunks;
    // one decision for all 128 epilogue threads (the flag may be raised by a
    // timed-out role at any moment, and the named barriers below need all)
    const bool go = sk_bar_and(128, !*abort_flag) && nch > 0;
    if (go) {
      if (nred == 1) {
        // the whole sum is in TMEM: transform straight from it
        if (rows_mode) {
#pragma unroll 1
          for (int c = 0; c < args.r16 / 16; ++c) {
            if (!QLORA_CHECK(static_cast<uint32_t>(c * 16 + 16) <= tcols, 202)) break;
            uint32_t t[16];
            tmem_ld16(taddr + c * 16, t);
            tmem_ld_wait();
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = 0.0f + __uint_as_float(t[i]);
            if (row < args.P) sk_rows_out(args, row, c * 16, v);
          }
        } else {
#pragma unroll 1
          for (int c = 0; c < args.r16 / 16; ++c) {
            if (!QLORA_CHECK(static_cast<uint32_t>(args.r16 + c * 16 + 16) <= tcols, 202)) break;
            uint32_t th[16], tl[16];
            tmem_ld16(taddr + c * 16, th);
            tmem_ld16(taddr + args.r16 + c * 16, tl);
            tmem_ld_wait();
            float g[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              g[i] = (0.0f + (__uint_as_float(th[i]) + __uint_as_float(tl[i]))) * args.s;
            if (row < args.P) sk_grad_out(args, row, c * 16, g);
          }
        }
      } else {
        // publish this CTA's partial tile, count in, the last arrival finishes;
        // only the columns the finish reads (r16 of T or G; the hi and lo
        // halves, 2 r16, of dA or dB) -- Qn is rounded up to a whole box
        float* dst = args.partial + (static_cast<int64_t>(split) * args.P + row) * args.Qtot + q0;
        const int used = min(qv, max(0, (rows_mode ? args.r16 : 2 * args.r16) - q0));
#pragma unroll 1
        for (int c = 0; c < used / 16; ++c) {
          uint32_t t[16];
          tmem_ld16(taddr + c * 16, t);
          tmem_ld_wait();
          if (row < args.P &&
              QLORA_CHECK(static_cast<uint32_t>(c * 16 + 16) <= tcols &&
                              (static_cast<int64_t>(split) * args.P + row) * args.Qtot + q0 + c * 16 + 16 <= args.partial_elems,
                          201)) {
            float4* d4 = reinterpret_cast<float4*>(dst + c * 16);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              d4[i] = make_float4(__uint_as_float(t[4 * i]), __uint_as_float(t[4 * i + 1]),
                                  __uint_as_float(t[4 * i + 2]), __uint_as_float(t[4 * i + 3]));
          }
        }
        sk_bar(128);   // every partial write of the CTA before the release below
        if (et == 0) {
          const unsigned int old = atom_add_acq_rel_gpu(args.cnt + ptile, 1u);
          *s_last = (old == static_cast<unsigned int>(nred - 1)) ? 1 : 0;
        }
        sk_bar(128);   // the acquire above before any partial read of the CTA
        if (*s_last) {
          const float* src = args.partial + row * args.Qtot;
          const int64_t sstride = args.P * args.Qtot;
          [[maybe_unused]] const int need = rows_mode ? args.r16 : 2 * args.r16;
          if (row < args.P &&
              QLORA_CHECK((args.splits - 1) * sstride + row * args.Qtot + need <= args.partial_elems, 203)) {
#pragma unroll 1
            for (int c = 0; c < args.r16 / 16; ++c) {
              // The partials come from L2: loads of several splits are put in
              // flight together (one round trip per batch instead of per
              // split); the sum keeps split order.
              float v[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] = 0.0f;
              if (rows_mode) {
                constexpr int kB = 4;
                for (int sp0 = 0; sp0 < args.splits; sp0 += kB) {
                  float4 x[kB][4];
#pragma unroll
                  for (int u = 0; u < kB; ++u) {
                    if (sp0 + u < args.splits) {
                      const float4* s4 = reinterpret_cast<const float4*>(src + (sp0 + u) * sstride + c * 16);
#pragma unroll
                      for (int i = 0; i < 4; ++i) x[u][i] = __ldcg(s4 + i);
                    }
                  }
#pragma unroll
                  for (int u = 0; u < kB; ++u) {
                    if (sp0 + u < args.splits) {
#pragma unroll
                      for (int i = 0; i < 4; ++i) {
                        v[4 * i] += x[u][i].x; v[4 * i + 1] += x[u][i].y;
                        v[4 * i + 2] += x[u][i].z; v[4 * i + 3] += x[u][i].w;
                      }
                    }
                  }
                }
                sk_rows_out(args, row, c * 16, v);
              } else {
                constexpr int kB = 2;
                for (int sp0 = 0; sp0 < args.splits; sp0 += kB) {
                  float4 h[kB][4], l[kB][4];
#pragma unroll
                  for (int u = 0; u < kB; ++u) {
                    if (sp0 + u < args.splits) {
                      const float4* sh = reinterpret_cast<const float4*>(src + (sp0 + u) * sstride + c * 16);
                      const float4* sl =
                          reinterpret_cast<const float4*>(src + (sp0 + u) * sstride + args.r16 + c * 16);
#pragma unroll
                      for (int i = 0; i < 4; ++i) { h[u][i] = __ldcg(sh + i); l[u][i] = __ldcg(sl + i); }
                    }
                  }
#pragma unroll
                  for (int u = 0; u < kB; ++u) {
                    if (sp0 + u < args.splits) {
#pragma unroll
                      for (int i = 0; i < 4; ++i) {
                        v[4 * i] += h[u][i].x + l[u][i].x; v[4 * i + 1] += h[u][i].y + l[u][i].y;
                        v[4 * i + 2] += h[u][i].z + l[u][i].z; v[4 * i + 3] += h[u][i].w + l[u][i].w;
                      }
                    }
                  }
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] *= args.s;
                sk_grad_out(args, row, c * 16, v);
              }
            }
          }
          if (et == 0) args.cnt[ptile] = 0u;   // leave the counter as found
        }
      }
      // hl planes: zero columns [2 r16, Qh)
      if (rows_mode && args.hl && row < args.P && qchunk == 0 && (nred == 1 || *s_last))
        sk_hl_zero(args.hl + row * args.Qh, args.r16, args.Qh);
    }
    // side task: T rows -> hl planes, shared out over this problem's CTAs
    if (rows_mode && args.side_src) {
      const int64_t per = (args.side_rows + nctas - 1) / nctas;
      const int64_t m_end = min(args.side_rows, (bid + 1) * per);
      for (int64_t m = bid * per + et; m < m_end; m += 128) {
        __nv_bfloat16* hrow = args.side_hl + m * args.Qh;
        for (int c0 = 0; c0 < args.r16; c0 += 16) {
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = (c0 + i < args.r) ? args.side_src[m * args.r + c0 + i] : 0.0f;
          uint32_t hi[8], lo[8];
          sk_hilo16(v, hi, lo);
          sk_st8(hrow + c0, hi, 8); sk_st8(hrow + c0 + 8, hi + 4, 8);
          sk_st8(hrow + args.r16 + c0, lo, 8); sk_st8(hrow + args.r16 + c0 + 8, lo + 4, 8);
        }
        sk_hl_zero(hrow, args.r16, args.Qh);
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
