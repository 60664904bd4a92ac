// gemm_nf4_pair.cuh -- the fused NF4 GEMM on a 2-SM pair (tcgen05.mma
// cta_group::2), forward and backward-dX.  Same mathematics as
// gemm_nf4.cuh (dequantise into shared memory, adapter folded into the
// accumulator as hi/lo bf16 planes); the pair works on a 256 x 256 output
// tile, so every dequantised weight feeds 256 tokens instead of 128 and each
// SM dequantises and stores only its 128-row half of the weight tile.
//
//   CTA rank r of a pair holds: activation rows m0 + 128r .. +127 (MMA A
//   half), weight rows (forward) or output columns (dX) n0 + 128r .. +127
//   (MMA B half), and TMEM rows for its 128 activation rows x 256 columns.
//
// Pipeline per 64-deep stage (6-stage ring):
//   - each CTA's producer loads its packed codes with a local TMA (local
//     barrier full_c) and its activation tile with a pair TMA whose bytes
//     complete on the leader's barrier full_a (the leader sets expect-tx for
//     both CTAs);
//   - one of two dequant warp groups (stages alternate between them) turns
//     the codes into the bf16 B half, fences it for the async proxy and
//     arrives (one arrive per warp) on the leader's barrier full_b;
//   - the leader's MMA thread waits full_a and full_b, issues 4
//     tcgen05.mma.cta_group::2 (M 256, N 256, K 16) and commits to `empty`
//     in both CTAs (multicast commit).
// Epilogue: every CTA reads its own TMEM half (tcgen05.ld) and writes bf16.
#pragma once
#include "nf4_decode.cuh"
#include "gemm_nf4.cuh"

namespace qlora {

constexpr int kPairStages = 6;
constexpr int kPairThreads = 320;
constexpr uint32_t kPairABytes = 128 * 64 * 2;   // 16 KB activations (this CTA's half)
constexpr uint32_t kPairWBytes = 128 * 64 * 2;   // 16 KB dequantised weight half
constexpr uint32_t kPairCBytes = 128 * 64 / 2;   //  4 KB packed codes
constexpr uint32_t kPairStageBytes = kPairABytes + kPairWBytes + kPairCBytes;
constexpr uint32_t kPairSmemBytes = kPairStages * kPairStageBytes + 1024 + 512;
constexpr uint32_t kPairTmemCols = 256;
constexpr int kPairDeqWarps = 4;                 // per stage, per CTA

template <int MODE>
__global__ void __launch_bounds__(kPairThreads, 1)
    k_gemm_nf4_pair(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_codes,
                    const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_lb,
                    const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  auto slot_a = [&](int s) { return base + s * kPairStageBytes; };
  auto slot_w = [&](int s) { return base + s * kPairStageBytes + kPairABytes; };
  auto slot_c = [&](int s) { return base + s * kPairStageBytes + kPairABytes + kPairWBytes; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kPairStages * kPairStageBytes);
  uint64_t* full_a = bars;                          // leader: both activation halves (+ adapter tiles)
  uint64_t* full_c = bars + kPairStages;            // local: this CTA's codes
  uint64_t* full_b = bars + 2 * kPairStages;        // leader: both dequantised halves
  uint64_t* empty = bars + 3 * kPairStages;         // local: MMA done with the stage (multicast commit)
  uint64_t* acc_full = bars + 4 * kPairStages;      // local: accumulator complete (multicast commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 * kPairStages + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * 256 + rank * 128;   // this CTA's activation rows
  const int64_t np0 = static_cast<int64_t>(blockIdx.x >> 1) * 256;           // pair's output columns
  const int64_t nc0 = np0 + rank * 128;                                      // this CTA's B half
  const int nl1 = (args.lora_r16 + 63) / 64;
  const int num_lt = 2 * nl1;
  const int total = args.num_kt + num_lt;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(smem_u32(&full_a[s]), 1);
      mbar_init(smem_u32(&full_c[s]), 1);
      mbar_init(smem_u32(&full_b[s]), 2 * kPairDeqWarps);
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
    tmem_alloc_pair(smem_u32(tmem_slot), kPairTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();   // barriers of both CTAs initialised before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  auto leader_bar = [&](uint64_t* b) { return mapa_shared(smem_u32(b), 0); };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < total; ++it) {
        const int s = it % kPairStages;
        if (it >= kPairStages &&
            !mbar_wait_cluster(smem_u32(&empty[s]), ((it / kPairStages) + 1) & 1, abort_flag, args.status))
          break;
        const uint32_t fa = leader_bar(&full_a[s]);
        const uint32_t fc = smem_u32(&full_c[s]);
        if (it < args.num_kt) {
          mbar_arrive_expect_tx(fc, kPairCBytes);
          if (MODE == kModeFwd)
            tma_load_2d(smem_u32(slot_c(s)), &tm_codes, fc, it * 32, static_cast<int32_t>(nc0));
          else
            tma_load_2d(smem_u32(slot_c(s)), &tm_codes, fc, static_cast<int32_t>(nc0 / 2), it * 64);
          if (leader) mbar_arrive_expect_tx(smem_u32(&full_a[s]), 2 * kPairABytes);
          tma_load_2d_pair(smem_u32(slot_a(s)), &tm_act, fa, it * 64, static_cast<int32_t>(m0));
        } else {
          const int lt = it - args.num_kt;
          const int li = lt % nl1;
          const int64_t arow = (lt / nl1) * args.lora_lo_row + m0;
          mbar_arrive(fc);   // no codes: keeps the dequant warps' phases in step
          if (leader) mbar_arrive_expect_tx(smem_u32(&full_a[s]), 2 * (kPairABytes + kPairWBytes));
          tma_load_2d_pair(smem_u32(slot_a(s)), &tm_la, fa, li * 64, static_cast<int32_t>(arow));
          if (MODE == kModeFwd) {
            tma_load_2d_pair(smem_u32(slot_w(s)), &tm_lb, fa, li * 64, static_cast<int32_t>(nc0));
          } else {
            tma_load_2d_pair(smem_u32(slot_w(s)), &tm_lb, fa, static_cast<int32_t>(nc0), li * 64);
            tma_load_2d_pair(smem_u32(slot_w(s)) + 8192, &tm_lb, fa, static_cast<int32_t>(nc0) + 64, li * 64);
          }
        }
        ++issued;
      }
      if (*abort_flag) {
        for (int it = max(0, issued - kPairStages); it < issued; ++it) {
          const uint32_t fc = smem_u32(&full_c[it % kPairStages]);
          const uint64_t t0 = global_ns();
          while (!mbar_try_wait(fc, (it / kPairStages) & 1) && global_ns() - t0 < 200000000ull) {}
          if (leader) {
            const uint32_t fa = smem_u32(&full_a[it % kPairStages]);
            const uint64_t t1 = global_ns();
            while (!mbar_try_wait_cluster(fa, (it / kPairStages) & 1) && global_ns() - t1 < 200000000ull) {}
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer (leader)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(256, 256, 0, MODE == kModeDx ? 1 : 0);
      for (int it = 0; it < total; ++it) {
        const int s = it % kPairStages;
        const uint32_t par = (it / kPairStages) & 1;
        if (!mbar_wait_cluster(smem_u32(&full_a[s]), par, abort_flag, args.status)) break;
        if (!mbar_wait_cluster(smem_u32(&full_b[s]), par, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(slot_a(s));
        const uint32_t w_base = smem_u32(slot_w(s));
        const int nk = (it < args.num_kt) ? 4 : min(4, (args.lora_r16 - ((it - args.num_kt) % nl1) * 64) / 16);
        for (int k = 0; k < nk; ++k) {
          const uint64_t adesc = sw128_desc(a_base + k * 32, 16, 1024);
          const uint64_t bdesc = (MODE == kModeFwd) ? sw128_desc(w_base + k * 32, 16, 1024)
                                                    : sw128_desc(w_base + k * 2048, 8192, 1024);
          umma_bf16_pair(tmem_d, adesc, bdesc, idesc, (it > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit_pair(smem_u32(&empty[s]), 0x3);
      }
      umma_commit_pair(smem_u32(acc_full), 0x3);
    }
  } else {
    // ---------------------------------------------------------- dequant
    const int g = (warp - 2) >> 2;                 // stage parity this warp group handles
    const int t = ((warp - 2) & 3) * 32 + lane;    // 0..127
    const int64_t KB = args.wK / 64;
    int64_t wn0, kb0, wn_step, kb_step;
    uint32_t c_off, c_swz, w_off, w_swz, c_ch0;
    if (MODE == kModeFwd) {
      wn0 = nc0 + t; kb0 = 0; wn_step = 0; kb_step = 1;
      c_off = t * 32; c_swz = (t >> 2) & 1; c_ch0 = 0;          // 32-byte rows, 32-byte swizzle
      w_off = t * 128; w_swz = t & 7;
    } else {
      const int nl = t & 63, j = t >> 6;
      wn0 = nl; kb0 = nc0 / 64 + j; wn_step = 64; kb_step = 0;
      c_off = nl * 64; c_swz = (nl >> 1) & 3; c_ch0 = 2 * j;    // 64-byte rows, 64-byte swizzle
      w_off = j * 8192 + nl * 128; w_swz = nl & 7;
    }
    // raw block-scale inputs of this thread's stage `it`, loaded 3 own stages ahead
    auto load_raw = [&](int it, uint32_t& rq, float& rs) {
      rq = 0; rs = 0.0f;
      if (it >= args.num_kt) return;
      const int64_t n = wn0 + wn_step * it, k = kb0 + kb_step * it;
      if (n >= args.wN || k >= KB) return;
      const int64_t f = n * KB + k;
      if (args.dq) { rq = __ldg(args.q8 + f); rs = __ldg(args.s2 + (f >> 8)); }
      else rs = __ldg(args.absmax_f32 + f);
    };
    uint32_t q0, q1, q2;
    float s0, s1, s2;
    load_raw(g, q0, s0);
    load_raw(g + 2, q1, s1);
    load_raw(g + 4, q2, s2);
    for (int it = g; it < total; it += 2) {
      const int s = it % kPairStages;
      const float scale = args.dq ? __fmul_rn(static_cast<float>(q0), s0) : s0;
      q0 = q1; s0 = s1; q1 = q2; s1 = s2;
      load_raw(it + 6, q2, s2);
      if (!mbar_wait(smem_u32(&full_c[s]), (it / kPairStages) & 1, abort_flag, args.status)) break;
      if (it < args.num_kt) {
        const int64_t n = wn0 + wn_step * it, k = kb0 + kb_step * it;
        uint8_t* wdst = slot_w(s) + w_off;
        if (n < args.wN && k < KB) {
          const uint8_t* cs = slot_c(s) + c_off;
          const uint4 c0 = *reinterpret_cast<const uint4*>(cs + (((c_ch0 + 0) ^ c_swz) << 4));
          const uint4 c1 = *reinterpret_cast<const uint4*>(cs + (((c_ch0 + 1) ^ c_swz) << 4));
          const NF4Table tab = nf4_table(scale);
          const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t o[4];
            nf4_decode8(cw[c], tab, o);
            *reinterpret_cast<uint4*>(wdst + ((static_cast<uint32_t>(c) ^ w_swz) << 4)) =
                make_uint4(o[0], o[1], o[2], o[3]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(wdst + (c << 4)) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_bar(&full_b[s]));
    }

    // ------------------------------------------------------------ epilogue
    {
      const uint32_t bar = smem_u32(acc_full);
      const uint64_t t0 = global_ns();
      bool ok = true;
      while (!mbar_try_wait_cluster(bar, 0)) {
        if (global_ns() - t0 > QLORA_WAIT_NS) { ok = false; break; }
      }
      if (!ok) {
        *abort_flag = 1;
        if (args.status) atomicOr(args.status, QLORA_DEV_TIMEOUT);
      }
    }
    tc_fence_after();
    if (!*abort_flag) {
      const int q = warp & 3;
      const int half = (warp - 2) >> 2;
      const int64_t row = m0 + q * 32 + lane;
      const uint32_t taddr = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        const int col = half * 128 + c * 16;
        uint32_t r[16];
        tmem_ld16(taddr + col, r);
        tmem_ld_wait();
        const int64_t gc = np0 + col;
        if (row < args.M && gc < args.out_cols) {
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
          __nv_bfloat16* dst = args.out + row * args.ldo + gc;
          if (gc + 16 <= args.out_cols && (args.ldo & 7) == 0) {
            reinterpret_cast<uint4*>(dst)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            reinterpret_cast<uint4*>(dst)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          } else {
            const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(pk);
            for (int i = 0; i < 16 && gc + i < args.out_cols; ++i) dst[i] = hv[i];
          }
        }
      }
    }
  }

  tc_fence_before();
  cluster_sync();   // the peer may still read this CTA's shared memory / arrive on its barriers until here
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_d, kPairTmemCols);
  }
}

}  // namespace qlora
