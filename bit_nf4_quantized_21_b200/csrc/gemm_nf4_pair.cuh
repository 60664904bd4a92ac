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
// Three shared-memory rings per CTA; stage `it` (64 deep) uses slot
// it % depth of each (depths for one M tile per pair; with two, 4
// activation slots hold both tiles' halves and there are 3 weight slots,
// PairRing below):
//   activations  6 x 16 KB  pair TMA by the producer warp (0), completing on
//                           the leader's full_a; freed by the MMA (empty_a)
//   codes        6 x  4 KB  local TMA by the code warp (15) (full_c); a
//                           dequant warp loads stage it + 3's codes into
//                           registers right after decoding stage it, and
//                           frees a stage's slot (empty_c) once its decode
//                           has consumed them
//   bf16 weight  6 x 16 KB  written by dequant group it % 3 after the MMA
//                           freed the slot (empty_w); one arrive per warp
//                           on the leader's full_w
// Two MMA-issuing threads in the leader (warps 1 and 14) take alternate
// stages: issuer i waits full_a and full_w of stage it = i (mod 2), issues
// its 4 tcgen05.mma.cta_group::2 (M 256, N 256, K 16) into its own
// accumulator D_i (TMEM columns 256 i .. 256 i + 255: the two use all 512)
// and commits to empty_a and empty_w in both CTAs (multicast commits).  A
// thread that waits on a barrier right after issuing MMAs stalls until they
// drain (~250 cycles of bubble per stage, measured), which one issuer
// cannot hide; with two, one issues while the other waits.  The epilogue
// adds D_0 + D_1 (fixed order: deterministic).  Adapter stages load their
// B operand by TMA into the weight slot, issued by the dequant group that
// owns the slot, with the bytes counted on that slot's full_w.
// Every waiter waits for each phase of its slots in order: a waiter that
// takes every G-th stage (issuers G = 2, dequant groups G = 3) owns whole
// slots because each ring depth is a multiple of its waiters' G, so no
// waiter can be two phases behind and the 1-bit phase parity is safe.
// Epilogue: all 16 warps of every CTA read its own TMEM half (tcgen05.ld)
// and write bf16.
//
// WDENSE = true is the same GEMM over a dense bf16 weight (plain LoRA, the
// baseline the QLoRA pages compare against): the weight tile of every
// stage arrives by TMA straight into the weight slot, the way the adapter
// stages' B tiles do (tm_codes then maps the bf16 weight), and nothing is
// dequantised.
#pragma once
#include "nf4_decode.cuh"
#include "gemm_nf4.cuh"

namespace qlora {

// MSUB = 1: one 256-row M tile per pair; MSUB = 2: two (a 512 x 256 output
// tile), so every dequantised weight stage feeds 512 tokens.  Ring depths
// per MSUB (activation slots hold MSUB x 16 KB per CTA).
template <int MSUB> struct PairRing;
template <> struct PairRing<1> { static constexpr int A = 6, W = 6; };
template <> struct PairRing<2> { static constexpr int A = 4, W = 3; };
constexpr int kPairRingC = 6;                    // packed-code ring depth
constexpr int kPairDeqGroups = 3;                // group it % 3 decodes stage it (owns W slots it % depth)
// A waiter that takes every G-th stage must own whole slots: with a ring
// depth that is not a multiple of G it could come to a slot whose previous
// phase (another waiter's stage) is still pending, and a parity wait would
// then take the phase before that for the one it wants.
static_assert(PairRing<1>::W % kPairDeqGroups == 0 && PairRing<2>::W % kPairDeqGroups == 0,
              "each weight slot must belong to one dequant group");
static_assert(kPairRingC % kPairDeqGroups == 0, "each code slot must belong to one dequant group");
constexpr int kPairDeqWarps = 4;                 // warps per group (128 weight rows)
constexpr int kPairIssuers = 2;
// with MSUB = 1 the issuers alternate stages (G = 2); with MSUB = 2 each
// takes every stage (G = 1)
static_assert(PairRing<1>::A % kPairIssuers == 0 && PairRing<1>::W % kPairIssuers == 0,
              "each operand slot must belong to one issuer");
constexpr int kPairIssuerWarp1 = 2 + kPairDeqGroups * kPairDeqWarps;   // second MMA issuer
// The code producer has a warp of its own: as a second lane of the
// activation producer's warp it was starved while lane 0 spun on its ring
// (a diverged warp runs one path at a time) and issued codes only ~half a
// stage ahead instead of a whole ring ahead.
constexpr int kPairCodesWarp = kPairIssuerWarp1 + 1;
constexpr int kPairThreads = 32 * (kPairCodesWarp + 1);
constexpr uint32_t kPairABytes = 128 * 64 * 2;   // 16 KB activations (this CTA's half of one M tile)
constexpr uint32_t kPairWBytes = 128 * 64 * 2;   // 16 KB dequantised weight half
constexpr uint32_t kPairCBytes = 128 * 64 / 2;   //  4 KB packed codes
template <int MSUB> struct PairLayout {
  static constexpr uint32_t OffW = PairRing<MSUB>::A * MSUB * kPairABytes;
  static constexpr uint32_t OffC = OffW + PairRing<MSUB>::W * kPairWBytes;
  static constexpr uint32_t OffBar = OffC + kPairRingC * kPairCBytes;
  static constexpr uint32_t Bytes = OffBar + 1024 /*align*/ + 512 /*bars*/;
};
constexpr uint32_t kPairSmemBytes = PairLayout<1>::Bytes > PairLayout<2>::Bytes ? PairLayout<1>::Bytes : PairLayout<2>::Bytes;
constexpr uint32_t kPairTmemCols = 512;   // two 256-column accumulators
static_assert(kPairSmemBytes <= 227 * 1024, "pair kernel shared memory");

template <int MODE, bool WDENSE = false, int MSUB = 1>
__global__ void __launch_bounds__(kPairThreads, 1)
    k_gemm_nf4_pair(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_codes,
                    const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_lb,
                    const __grid_constant__ CUtensorMap tm_out, const GemmArgs args) {
  static_assert(MSUB == 1 || MSUB == 2, "one or two M tiles per pair");
  constexpr int kPairRingA = PairRing<MSUB>::A;
  constexpr int kPairRingW = PairRing<MSUB>::W;
  constexpr uint32_t kSlotA = MSUB * kPairABytes;
  using Lay = PairLayout<MSUB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  auto slot_a = [&](int it) { return base + (it % kPairRingA) * kSlotA; };
  auto slot_w = [&](int it) { return base + Lay::OffW + (it % kPairRingW) * kPairWBytes; };
  auto slot_c = [&](int it) { return base + Lay::OffC + (it % kPairRingC) * kPairCBytes; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + Lay::OffBar);
  uint64_t* full_a = bars;                                  // [A] leader: activation halves (+ adapter tiles)
  uint64_t* empty_a = full_a + kPairRingA;                  // [A] local: MMA done with the activations
  uint64_t* full_c = empty_a + kPairRingA;                  // [C] local: codes landed
  uint64_t* empty_c = full_c + kPairRingC;                  // [C] local: codes copied to registers
  uint64_t* full_w = empty_c + kPairRingC;                  // [W] leader: both weight halves written
  uint64_t* empty_w = full_w + kPairRingW;                  // [W] local: MMA done with the weights
  uint64_t* acc_full = empty_w + kPairRingW;                // local: accumulator complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto par = [](int it, int depth) { return static_cast<uint32_t>((it / depth) & 1); };
  auto prev_par = [](int it, int depth) { return static_cast<uint32_t>(((it / depth) + 1) & 1); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  // this CTA's activation rows: m0 + 256 s .. + 127 for M tile s < MSUB
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * 256 * MSUB + rank * 128;
  const int64_t np0 = static_cast<int64_t>(blockIdx.x >> 1) * 256;           // pair's output columns
  const int64_t nc0 = np0 + rank * 128;                                      // this CTA's B half
  const int nl1 = (args.lora_r16 + 63) / 64;
  const int num_lt = 2 * nl1;
  const int total = args.num_kt + num_lt;

  if (threadIdx.x == 0) {
    // MSUB = 2: both issuers read every stage, so each slot is freed by two commits
    for (int i = 0; i < kPairRingA; ++i) { mbar_init(smem_u32(&full_a[i]), 1); mbar_init(smem_u32(&empty_a[i]), MSUB); }
    for (int i = 0; i < kPairRingC; ++i) {
      mbar_init(smem_u32(&full_c[i]), 1);
      mbar_init(smem_u32(&empty_c[i]), kPairDeqWarps);
    }
    for (int i = 0; i < kPairRingW; ++i) {
      mbar_init(smem_u32(&full_w[i]), 2 * kPairDeqWarps);
      mbar_init(smem_u32(&empty_w[i]), MSUB);
    }
    mbar_init(smem_u32(acc_full), kPairIssuers);
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
  if (threadIdx.x == 0) QLORA_CHECK_ONLY(Lay::Bytes <= dyn_smem_bytes(), 100);
  auto leader_bar = [&](uint64_t* b) { return mapa_shared(smem_u32(b), 0); };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // activation tiles (and, in the adapter stages, the adapter B tiles)
      int issued = 0;
      for (int it = 0; it < total; ++it) {
        const int ia = it % kPairRingA;
        if (it >= kPairRingA &&
            !mbar_wait(smem_u32(&empty_a[ia]), prev_par(it, kPairRingA), abort_flag, args.status))
          break;
        const uint32_t fa = leader_bar(&full_a[ia]);
        if (it < args.num_kt) {
          if (leader) mbar_arrive_expect_tx(smem_u32(&full_a[ia]), 2 * kSlotA);
#pragma unroll
          for (int t = 0; t < MSUB; ++t)
            if (QLORA_CHECK((it % kPairRingA) * kSlotA + (t + 1) * kPairABytes <= Lay::OffW && m0 >= 0, 101))
              tma_load_2d_pair(smem_u32(slot_a(it)) + t * kPairABytes, &tm_act, fa, it * 64, static_cast<int32_t>(m0 + 256 * t));
        } else {
          // adapter stage: the A tile here; the adapter B tile is loaded into
          // the weight slot, and its bytes counted on that slot's full_w, by
          // the dequant group that owns the slot (it has seen every earlier
          // phase of full_w; this thread may be a whole activation ring
          // ahead, and full_a of this slot may still be in an earlier stage's
          // phase, so neither may carry the B tile's bytes)
          // s*T (s*G) comes from the kernel ahead in the stream
          if (it == args.num_kt) griddep_wait();
          const int lt = it - args.num_kt;
          const int li = lt % nl1;
          const int64_t arow = (lt / nl1) * args.lora_lo_row + m0;
          if (leader) mbar_arrive_expect_tx(smem_u32(&full_a[ia]), 2 * kSlotA);
#pragma unroll
          for (int t = 0; t < MSUB; ++t)
            if (QLORA_CHECK((it % kPairRingA) * kSlotA + (t + 1) * kPairABytes <= Lay::OffW && arow >= 0 && li >= 0, 101))
              tma_load_2d_pair(smem_u32(slot_a(it)) + t * kPairABytes, &tm_la, fa, li * 64, static_cast<int32_t>(arow + 256 * t));
        }
        ++issued;
      }
      if (*abort_flag && leader) {
        for (int it = max(0, issued - kPairRingA); it < issued; ++it) {
          const uint32_t fa = smem_u32(&full_a[it % kPairRingA]);
          const uint64_t t1 = global_ns();
          while (!mbar_try_wait_cluster(fa, par(it, kPairRingA)) && global_ns() - t1 < qlora_drain_limit()) {}
        }
      }
    }
  } else if (warp == kPairCodesWarp) {
    if (lane == 0) {
      // packed codes, freed by the dequant warps (runs ahead of the MMA)
      int issued = 0;
      for (int it = 0; it < total; ++it) {
        const int ic = it % kPairRingC;
        if (it >= kPairRingC &&
            !mbar_wait(smem_u32(&empty_c[ic]), prev_par(it, kPairRingC), abort_flag, args.status))
          break;
        const uint32_t fc = smem_u32(&full_c[ic]);
        if (it < args.num_kt && !WDENSE) {
          mbar_arrive_expect_tx(fc, kPairCBytes);
          if (!QLORA_CHECK(Lay::OffC + (it % kPairRingC + 1) * kPairCBytes <= Lay::OffBar, 102)) {
            ++issued;   // no load: the wait on this slot runs out (bounded) and the launch aborts
            continue;
          }
          if (MODE == kModeFwd)
            tma_load_2d(smem_u32(slot_c(it)), &tm_codes, fc, it * 32, static_cast<int32_t>(nc0));
          else
            tma_load_2d(smem_u32(slot_c(it)), &tm_codes, fc, static_cast<int32_t>(nc0 / 2), it * 64);
        } else {
          mbar_arrive(fc);   // no codes (adapter stage, dense weight): keeps the dequant warps' phases in step
        }
        ++issued;
      }
      if (*abort_flag) {
        for (int it = max(0, issued - kPairRingC); it < issued; ++it) {
          const uint32_t fc = smem_u32(&full_c[it % kPairRingC]);
          const uint64_t t0 = global_ns();
          while (!mbar_try_wait(fc, par(it, kPairRingC)) && global_ns() - t0 < qlora_drain_limit()) {}
        }
      }
    }
  } else if (warp == 1 || warp == kPairIssuerWarp1) {
    // ------------------------------------------------- MMA issuers (leader)
    if (leader && lane == 0) {
      // MSUB = 1: issuer i takes the stages it = i (mod 2) into D_i (summed
      // in the epilogue); MSUB = 2: issuer i takes every stage for M tile i
      // into D_i
      const int me = (warp == 1) ? 0 : 1;
      const uint32_t dcol = tmem_d + 256u * me;
      const int first = (MSUB == 1) ? me : 0;
      constexpr int step = (MSUB == 1) ? kPairIssuers : 1;
      constexpr uint32_t idesc = idesc_bf16(256, 256, 0, MODE == kModeDx ? 1 : 0);
      const bool cols_ok = QLORA_CHECK(256u * me + 256u <= kPairTmemCols, 104);
      for (int it = first; cols_ok && it < total; it += step) {
        const int ia = it % kPairRingA, iw = it % kPairRingW;
        if (!mbar_wait(smem_u32(&full_a[ia]), par(it, kPairRingA), abort_flag, args.status)) break;
        if (!mbar_wait(smem_u32(&full_w[iw]), par(it, kPairRingW), abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(slot_a(it)) + (MSUB == 1 ? 0u : me * kPairABytes);
        const uint32_t w_base = smem_u32(slot_w(it));
        const int nk = (it < args.num_kt) ? 4 : min(4, (args.lora_r16 - ((it - args.num_kt) % nl1) * 64) / 16);
        for (int k = 0; k < nk; ++k) {
          const uint64_t adesc = sw128_desc(a_base + k * 32, 16, 1024);
          const uint64_t bdesc = (MODE == kModeFwd) ? sw128_desc(w_base + k * 32, 16, 1024)
                                                    : sw128_desc(w_base + k * 2048, 8192, 1024);
          umma_bf16_pair(dcol, adesc, bdesc, idesc, (it > first || k > 0) ? 1u : 0u);
        }
        umma_commit_pair(smem_u32(&empty_a[ia]), 0x3);
        umma_commit_pair(smem_u32(&empty_w[iw]), 0x3);
      }
      umma_commit_pair(smem_u32(acc_full), 0x3);
    }
  } else {
    // ---------------------------------------------------------- dequant
    const int g = (warp - 2) >> 2;                 // handles stages it with it % kPairDeqGroups == g
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
    // raw block-scale inputs of this thread's stages, loaded 3 own stages ahead
    auto load_raw = [&](int it, uint32_t& rq, float& rs) {
      rq = 0; rs = 0.0f;
      if (it >= args.num_kt || WDENSE) return;
      const int64_t n = wn0 + wn_step * it, k = kb0 + kb_step * it;
      if (n >= args.wN || k >= KB) return;
      const int64_t f = n * KB + k;
      if (args.dq) { rq = __ldg(args.q8 + f); rs = __ldg(args.s2 + (f >> 8)); }
      else rs = __ldg(args.absmax_f32 + f);
    };
    uint32_t q0, q1, q2;
    float s0, s1, s2;
    constexpr int G = kPairDeqGroups;
    load_raw(g, q0, s0);
    load_raw(g + G, q1, s1);
    load_raw(g + 2 * G, q2, s2);
    // codes of stage `it` into registers (after its full_c phase)
    auto fetch = [&](int it, uint4& a0, uint4& a1) -> bool {
      if (!mbar_wait(smem_u32(&full_c[it % kPairRingC]), par(it, kPairRingC), abort_flag, args.status)) return false;
      const int64_t n = wn0 + wn_step * it, k = kb0 + kb_step * it;
      if (it < args.num_kt && n < args.wN && k < KB && !WDENSE) {
        const uint8_t* cs = slot_c(it) + c_off;
        a0 = *reinterpret_cast<const uint4*>(cs + (((c_ch0 + 0) ^ c_swz) << 4));
        a1 = *reinterpret_cast<const uint4*>(cs + (((c_ch0 + 1) ^ c_swz) << 4));
      } else {
        a0 = make_uint4(0, 0, 0, 0); a1 = a0;
      }
      return true;
    };
    uint4 n0, n1;
    bool live = g >= total || fetch(g, n0, n1);
    for (int it = g; it < total && live; it += G) {
      const int ic = it % kPairRingC, iw = it % kPairRingW;
      const float scale = args.dq ? __fmul_rn(dq_value(q0, args.dq), s0) : s0;
      const uint4 c0 = n0, c1 = n1;
      const int64_t n = wn0 + wn_step * it, k = kb0 + kb_step * it;
      const bool valid = it < args.num_kt && n < args.wN && k < KB;
      // the bf16 slot is free once the MMA of its previous use has completed
      if (it >= kPairRingW &&
          !mbar_wait(smem_u32(&empty_w[iw]), prev_par(it, kPairRingW), abort_flag, args.status))
        break;
      if (it >= args.num_kt || WDENSE) {
        // the stage's B operand by TMA: the adapter tile, or the dense weight
        // tile (rows/columns past the weight's edge arrive as zeros)
        if (((warp - 2) & 3) == 0 && lane == 0) {
          const bool lora = it >= args.num_kt;
          // the adapter B tile may come from the kernel ahead (the padded B)
          if (lora && it < args.num_kt + G) griddep_wait();
          const CUtensorMap* map = lora ? &tm_lb : &tm_codes;
          const int32_t kk = lora ? ((it - args.num_kt) % nl1) * 64 : it * 64;
          const uint32_t fw = leader_bar(&full_w[iw]);
          mbar_expect_tx_cluster(fw, kPairWBytes);
          // (a skipped load leaves this slot's wait to run out: bounded, the launch aborts)
          if (!QLORA_CHECK(Lay::OffW + (iw + 1) * kPairWBytes <= Lay::OffC && kk >= 0, 103)) {
          } else if (MODE == kModeFwd) {
            tma_load_2d_pair(smem_u32(slot_w(it)), map, fw, kk, static_cast<int32_t>(nc0));
          } else {
            tma_load_2d_pair(smem_u32(slot_w(it)), map, fw, static_cast<int32_t>(nc0), kk);
            tma_load_2d_pair(smem_u32(slot_w(it)) + 8192, map, fw, static_cast<int32_t>(nc0) + 64, kk);
          }
        }
      } else {
        uint8_t* wdst = slot_w(it) + w_off;
        if (valid && QLORA_CHECK(Lay::OffW + iw * kPairWBytes + w_off + 128 <= Lay::OffC, 103)) {
          const NF4Table tab = nf4_table(scale);
          const NF4Shr sh = nf4_shr();
          const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t o[4];
            nf4_decode8(cw[c], tab, o, sh);
            *reinterpret_cast<uint4*>(wdst + ((static_cast<uint32_t>(c) ^ w_swz) << 4)) =
                make_uint4(o[0], o[1], o[2], o[3]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(wdst + (c << 4)) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      // next own stage's codes: their loads run while this stage is handed over
      if (it + G < total && !fetch(it + G, n0, n1)) live = false;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_cluster(leader_bar(&full_w[iw]));
        mbar_arrive(smem_u32(&empty_c[ic]));   // this stage's codes were consumed by the stores above
      }
      q0 = q1; s0 = s1; q1 = q2; s1 = s2;
      load_raw(it + 3 * G, q2, s2);
    }
    // After an abort, adapter-tile loads this lane issued may still be in
    // flight into shared memory, and nobody else waits for them: give them
    // time to land before the CTA can exit (error path only; a tile load
    // takes microseconds).
    if (*abort_flag && ((warp - 2) & 3) == 0 && lane == 0 && (WDENSE || total > args.num_kt)) {
      const uint64_t t0 = global_ns();
      while (global_ns() - t0 < 1000000ull) {}
    }
  }

  // ------------------------------------------------------------ epilogue
  // Every warp, the role warps included: warp w reads TMEM lanes 32 (w % 4)
  // .. + 31 (its quarter of the accumulator rows) and takes a quarter of
  // the 16-column chunks, contiguous; four (one M tile: two pairs of) TMEM
  // loads go out before each wait.  With a bf16 output the warp stages its
  // 32 rows x 64 columns per box in shared memory (128-byte swizzle: the
  // lanes' 16-byte pieces of one column range fall in different banks) and
  // one lane writes the box with a TMA store, so the global writes are whole
  // rows of the box instead of 32 scattered 16-byte pieces per instruction.
  // After the last MMA every ring is free: warp w stages at base + 8 KB w.
  // Single-lane roles leave their warps diverged, and tcgen05.ld is
  // warp-collective: reconverge first.
  __syncwarp();
  {
    const uint32_t bar = smem_u32(acc_full);
    const uint64_t t0 = global_ns(), limit = qlora_wait_limit();
    bool ok = true;
    while (!mbar_try_wait_cluster(bar, 0)) {
      if (global_ns() - t0 > limit) { ok = false; break; }
    }
    if (!ok) {
      *abort_flag = 1;
      if (args.status) atomicOr(args.status, QLORA_DEV_TIMEOUT);
    }
  }
  __syncwarp();
  tc_fence_after();
  if (!*abort_flag) {
    const int q = warp & 3, j = warp >> 2;
    const uint32_t taddr = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
    uint8_t* stg = base + warp * 8192;
    const bool stg_ok = QLORA_CHECK(static_cast<uint32_t>(warp + 1) * 8192u <= Lay::OffBar, 106);
    // columns 16 c .. 16 c + 15 (c < 4) of this lane's row of a 64-column box, as bf16
    auto stage16 = [&](uint8_t* box, int c, const uint32_t (&r)[16]) {
      uint32_t pk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
      uint8_t* row = box + lane * 128;
      *reinterpret_cast<uint4*>(row + (((2 * c) ^ (lane & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      *reinterpret_cast<uint4*>(row + (((2 * c + 1) ^ (lane & 7)) << 4)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    };
    // the box at output column x, row y (boxes that start past the edge are skipped; TMA clips the rest)
    auto store_box = [&](const uint8_t* box, int64_t x, int64_t y) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && x < args.out_cols && y < args.M && stg_ok && QLORA_CHECK(x >= 0 && y >= 0 && (x & 7) == 0, 107)) {
        tma_store_2d(&tm_out, smem_u32(box), static_cast<int32_t>(x), static_cast<int32_t>(y));
        bulk_commit();
      }
    };
    if (MSUB == 1) {
      // D_0 + D_1 (fixed order); with a single stage the second issuer had
      // none and D_1 was never written.  Chunks 4j .. 4j + 3 (one box).
      const int64_t row = m0 + q * 32 + lane;
      const bool two = total > 1;
#pragma unroll 1
      for (int i = 0; i < 4; i += 2) {
        const int col = (4 * j + i) * 16;
        QLORA_CHECK_ONLY(256 + col + 32 <= static_cast<int>(kPairTmemCols), 105);
        uint32_t r[2][16], r1[2][16];
        tmem_ld16(taddr + col, r[0]);
        tmem_ld16(taddr + 256 + col, r1[0]);
        tmem_ld16(taddr + col + 16, r[1]);
        tmem_ld16(taddr + 256 + col + 16, r1[1]);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (two) {
#pragma unroll
            for (int e = 0; e < 16; ++e) r[h][e] = __float_as_uint(__uint_as_float(r[h][e]) + __uint_as_float(r1[h][e]));
          }
          if (args.tma_out) {
            stage16(stg, i + h, r[h]);
          } else {
            const int64_t gc = np0 + col + 16 * h;
            if (row < args.M && gc < args.out_cols) gemm_store16(args, row, gc, r[h]);
          }
        }
      }
      if (args.tma_out) store_box(stg, np0 + 64 * j, m0 + q * 32);
    } else {
      // D_t holds M tile t.  Chunks 8j .. 8j + 7 (two boxes): warps 0-7
      // M tile 0, warps 8-15 M tile 1.
      const int t = j >> 1;
      const int64_t row = m0 + 256 * t + q * 32 + lane;
#pragma unroll 1
      for (int bx = 0; bx < 2; ++bx) {
        const int col = (j & 1) * 128 + bx * 64;
        QLORA_CHECK_ONLY(256 * t + col + 64 <= static_cast<int>(kPairTmemCols), 105);
        uint32_t r[4][16];
#pragma unroll
        for (int h = 0; h < 4; ++h) tmem_ld16(taddr + 256 * t + col + 16 * h, r[h]);
        tmem_ld_wait();
        if (args.tma_out) {
          uint8_t* box = stg + bx * 4096;
#pragma unroll
          for (int h = 0; h < 4; ++h) stage16(box, h, r[h]);
          store_box(box, np0 + col, m0 + 256 * t + q * 32);
        } else {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int64_t gc = np0 + col + 16 * h;
            if (row < args.M && gc < args.out_cols) gemm_store16(args, row, gc, r[h]);
          }
        }
      }
    }
  }
  // the TMA stores have read their shared-memory boxes before the CTA can exit
  if (args.tma_out && lane == 0) bulk_wait_read();

  // this grid does not complete before the kernel ahead of it (when no
  // adapter stage waited for it above)
  if (threadIdx.x == 0) griddep_wait();
  // The CTA/cluster barrier below is warp-aligned: every warp reconverges
  // first, so that it cannot complete while a lane is still working and
  // TMEM be released under it.
  __syncwarp();
  tc_fence_before();
  cluster_sync();   // the peer may still read this CTA's shared memory / arrive on its barriers until here
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_d, kPairTmemCols);
  }
}

}  // namespace qlora
