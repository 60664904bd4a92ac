// gemv_nf4.cuh -- the decode-shaped forward (M <= 16 tokens): a
// weight-streaming NF4 GEMV on tcgen05 tensor cores.
//
//   Y [M, N] = X [M, K] . W^[N, K]^T + s T [M, r] . B [N, r]^T,   M <= 16
//
// (the same layer forward as the fused GEMM; the pages' h = W^x + (alpha/r)
// B(Ax), with the frozen base stored as blockwise NF4 and dequantised just
// in time.)  At these M the work is a stream of the packed weights:
// 0.516 B per weight from HBM against 2 M flops, so the design goal is to
// keep the weight stream moving and to spend as little as possible per
// weight on the chip.
//
// Roles per CTA (608 threads, one CTA per SM, persistent):
//   warp 0       TMA producer: per 128-deep slice, the packed codes of 128
//                weight rows (8 KB, 64 bytes per row) and the matching
//                16 x 128 activation slice (4 KB) into a shared-memory ring
//   warps 1, 18  MMA issuers (warp 1 also allocates TMEM): issuer i takes
//                the slices with it = i (mod 2) into its own accumulator
//   warps 2..13  three dequant groups of 4 warps; group g decodes slices
//                it = g (mod 3).  Thread = one weight row: its 128 codes of
//                the slice are exactly two quantisation blocks, each decoded
//                with the block's 16-entry bf16 table (nf4_decode.cuh) and
//                stored with tcgen05.st straight into tensor memory, where
//                they are the MMA's A operand (row = TMEM lane, 2 bf16 per
//                column).  The weights never touch shared memory.
//   warps 14..17 epilogue: accumulator (128 rows x 16 tokens, fp32) out of
//                TMEM, plus the adapter term s T B^T in fp32, rounded once
//                to bf16.  Before its first tile these warps also compute
//                the adapter's down-projection T = X A^T for the whole grid
//                (below), while the other roles are already streaming.
// MMA per slice: 8 x tcgen05.mma.cta_group::1.kind::f16, M 128 (weight
// rows, A from TMEM), N 16 (tokens, B = activation slice, K-major, 128-byte
// swizzle), K 16; each issuer's accumulator is double-buffered in TMEM so
// the epilogue of one tile overlaps the next tile's stream.  At N = 16 the
// limit is the issuing thread, not the math (measured on B200): a
// tcgen05.mma occupies the tensor pipe ~45-50 cycles at any N <= 64, but
// one thread that waits on a barrier, issues a slice's 8 MMAs and commits
// needs ~720 cycles per slice; two issuers on different SMSPs need ~350
// between them.  Hence 128-deep slices (fewer waits and commits per
// weight) and two issuers.
//
// Work split (stream-K): the weight is cut into units of 128 rows x 128
// columns, ordered tile-major (tile = 128 rows); CTA c of G streams units
// [U c / G, U (c+1) / G), so every CTA streams the same number of bytes
// whatever the shape.  A tile whose units span several CTAs is finished by
// the last of them to arrive: each writes its fp32 partial tile to the
// workspace, bumps the tile's counter, and the CTA that sees the final count
// adds the partials in CTA order (fixed order: deterministic), then applies
// the epilogue.  No CTA waits for another over a weight tile.
//
// Adapter down-projection T = X A^T [M, r] (fp32), folded into the same
// launch: every CTA's epilogue threads (1) compute the partial of T over the
// CTA's share of the contraction (K / G columns, CUDA cores, fp32, columns in
// order) into partial slot c, (2) once every CTA has published its partial,
// add up, in CTA order, the partials of the CTA's share of T's entries and
// write them to T, and (3) once every CTA has done that, load s T into
// shared memory for the epilogue.  The two grid-wide waits need every CTA
// resident at once, which the launch guarantees (cooperative launch, one
// CTA per SM); both are bounded like every other wait.  T is ready within a
// few microseconds of the start, before the first tile's epilogue needs it.
#pragma once
#include "nf4_decode.cuh"

namespace qlora {

constexpr int kGvRows = 128;                  // weight rows per tile (MMA M)
constexpr int kGvNT = 16;                     // token columns (MMA N); M <= 16
constexpr int kGvKS = 128;                    // contraction depth of one slice (two 64-weight blocks)
constexpr int kGvStages = 6;                  // ring depth: slot i = codes + activations (smem) + dequantised slice (TMEM)
constexpr int kGvIssuers = 2;                 // MMA-issuing threads (warps 1 and kGvIssuerWarp1)
constexpr int kGvGroups = 3;                  // dequant warp groups
constexpr int kGvDeqWarps = 4 * kGvGroups;
// Waiters that take every G-th slice (dequant groups, issuers) must own
// whole ring slots, or a parity wait could take an older phase for the
// pending one.
static_assert(kGvStages % kGvGroups == 0 && kGvStages % kGvIssuers == 0, "ring slots per waiter");
constexpr int kGvEpiWarp0 = 2 + kGvDeqWarps;  // first epilogue warp
constexpr int kGvIssuerWarp1 = kGvEpiWarp0 + 4;  // second MMA issuer (its own warp, another SMSP)
constexpr int kGvThreads = 32 * (kGvIssuerWarp1 + 1);
constexpr int kGvMaxCtas = 256;               // partial-tile slots in the workspace
constexpr int kGvMaxRank = 256;
constexpr uint32_t kGvCBytes = kGvRows * kGvKS / 2;  // 8 KB packed codes per slice
constexpr uint32_t kGvXBytes = kGvNT * kGvKS * 2;     // 4 KB activations per slice (two 128-byte-swizzled boxes)
constexpr uint32_t kGvOffX = kGvStages * kGvCBytes;
constexpr uint32_t kGvOffST = kGvOffX + kGvStages * kGvXBytes;
constexpr uint32_t kGvOffBar = kGvOffST + kGvNT * kGvMaxRank * 4;
constexpr uint32_t kGvSmemUsed = kGvOffBar + 1024 /*align*/ + 512 /*barriers*/;
constexpr uint32_t kGvSmemBytes = kGvSmemUsed > 118 * 1024 ? kGvSmemUsed : 118 * 1024;   // one CTA per SM
constexpr uint32_t kGvTmemCols = 512;         // D[issuer][buffer] at columns 32 (2 issuer + buffer), A slots at 128 + 64 i
constexpr uint32_t kGvTmemA0 = 32 * 2 * kGvIssuers;
constexpr uint32_t kGvASlotCols = kGvKS / 2;  // 2 bf16 per 32-bit column
static_assert(kGvTmemA0 + kGvASlotCols * kGvStages <= kGvTmemCols, "TMEM budget");
static_assert(kGvSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(2 * (kGvSmemBytes + 1024) > 228 * 1024, "one CTA per SM (the kernel is persistent)");

struct GvArgs {
  const uint8_t* q8;
  const float* s2;
  const float* absmax_f32;
  int dq;
  int64_t N, K;              // weight rows, columns
  int M;                     // tokens (1..16)
  int r;                     // adapter rank
  float s;                   // alpha / r
  float tscale;              // T = (X A^T) * tscale (1 / (1 - p) under dropout, else 1)
  const __nv_bfloat16* X;    // [M, K] the adapter's input for T (the activations, or their dropout)
  const __nv_bfloat16* A;    // [r, K] adapter down-projection
  float* T;                  // [M, r] fp32 out: X A^T (unscaled)
  float* tpart;              // [G][M][r] partials of T
  int* tcnt;                 // [2] grid arrival counters of the two T phases, zero on entry
  const __nv_bfloat16* B;    // [N, r]
  __nv_bfloat16* Y;          // [M, N]
  float* part;               // [kGvMaxCtas][2][128][16] partial tiles
  int* cnt;                  // [tiles] arrival counters, zero on entry
  int64_t KU;                // slices per weight row: ceil(K / 128)
  int64_t units;             // tiles * KU
  int* status;
};

// tcgen05.mma with the A operand in tensor memory (the "TS" form).
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 bits, 32 consecutive columns per thread.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// Named barrier that also ANDs a predicate over the participating threads.
__device__ __forceinline__ bool named_bar_and(uint32_t id, uint32_t threads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}
// Bounded wait whose outcome is the same in every lane of the warp, so that
// the warp-collective tcgen05 instructions after it never diverge (a lane
// that saw the abort flag a moment before the phase completed would
// otherwise leave the others alone in a .sync.aligned instruction).
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                               int* status) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status);
  return __all_sync(0xFFFFFFFFu, ok);
}

// CTA that streams unit u when U units are split over G CTAs as
// [U c / G, U (c + 1) / G).
__host__ __device__ __forceinline__ int64_t gv_cta_of(int64_t u, int64_t U, int64_t G) {
  return ((u + 1) * G - 1) / U;
}
__host__ __device__ __forceinline__ int64_t gv_begin(int64_t c, int64_t U, int64_t G) { return U * c / G; }

// acc + sum over the 8 bf16 pairs of x and a, in element order (bf16 -> fp32
// is exact: the 16 bits are the top half of the fp32 word)
__device__ __forceinline__ float gv_dot8(uint4 x, uint4 a, float acc) {
  const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, as[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc = fmaf(__uint_as_float(xs[i] << 16), __uint_as_float(as[i] << 16), acc);
    acc = fmaf(__uint_as_float(xs[i] & 0xFFFF0000u), __uint_as_float(as[i] & 0xFFFF0000u), acc);
  }
  return acc;
}

// The 128 epilogue threads of this CTA publish their writes (a barrier, then
// one releasing arrival on the grid counter) and wait until all G CTAs have
// arrived (an acquiring poll, then a barrier).  Bounded: on timeout the
// CTA's abort flag and the timeout status are set.  Returns the same
// outcome in every one of the 128 threads.
__device__ __forceinline__ bool gv_grid_arrive_wait(int* ctr, int64_t G, int et, volatile int* abort_flag,
                                                    int* status) {
  named_bar_sync(1, 128);
  bool ok = true;
  if (et == 0) {
    red_add_release_gpu(ctr, 1);
    const uint64_t t0 = global_ns();
    while (true) {
      int v;
      asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
      if (v >= G) break;
      if (*abort_flag) { ok = false; break; }
      if (global_ns() - t0 > qlora_wait_limit()) {
        *abort_flag = 1;
        if (status) atomicOr(status, QLORA_DEV_TIMEOUT);
        ok = false;
        break;
      }
      __nanosleep(128);
    }
  }
  ok = named_bar_and(1, 128, ok);
  return ok;
}

// T = X A^T for the whole grid, then s T into shared memory (see the header).
__device__ __forceinline__ bool gv_adapter_T(const GvArgs& args, int64_t c, int64_t G, int et, float* sT,
                                             volatile int* abort_flag) {
  const int MR = args.M * args.r;
  const int64_t K8 = args.K / 8;
  const int64_t v0 = K8 * c / G, v1 = K8 * (c + 1) / G;
  float* mine = args.tpart + c * MR;
  for (int o = et; o < MR; o += 128) {
    const int m = o / args.r, j = o - m * args.r;
    const uint4* xp = reinterpret_cast<const uint4*>(args.X + static_cast<int64_t>(m) * args.K);
    const uint4* ap = reinterpret_cast<const uint4*>(args.A + static_cast<int64_t>(j) * args.K);
    float acc = 0.0f;
    for (int64_t v = v0; v < v1; ++v) acc = gv_dot8(__ldg(xp + v), __ldg(ap + v), acc);
    mine[o] = acc;
  }
  if (!gv_grid_arrive_wait(args.tcnt, G, et, abort_flag, args.status)) return false;
  const int64_t o0 = MR * c / G, o1 = MR * (c + 1) / G;
  for (int64_t o = o0 + et; o < o1; o += 128) {
    float t = 0.0f;
    for (int64_t cc = 0; cc < G; ++cc) t += __ldcg(args.tpart + cc * MR + o);
    args.T[o] = t * args.tscale;
  }
  if (!gv_grid_arrive_wait(args.tcnt + 1, G, et, abort_flag, args.status)) return false;
  for (int i = et; i < MR; i += 128) sT[i] = args.s * __ldcg(args.T + i);
  named_bar_sync(1, 128);
  return true;
}

__global__ void __launch_bounds__(kGvThreads, 1)
    k_gemv_nf4(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_codes,
               const GvArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* sT = reinterpret_cast<float*>(base + kGvOffST);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kGvOffBar);
  // The MMA thread waits on one barrier per slice (ready) and commits to one
  // (empty): every wait or commit it issues between MMAs costs ~50-150
  // cycles of its issue time (measured), which at N = 16 is the budget.
  uint64_t* fullc = bars;                              // [S] packed codes landed (TMA)
  uint64_t* ready = fullc + kGvStages;                 // [S] activations landed (TMA) + slice in TMEM (4 warps)
  uint64_t* empty = ready + kGvStages;                 // [S] codes read (4 warps) + MMA done with the slot (commit)
  uint64_t* d_full = empty + kGvStages;                // [issuer][2] accumulator complete
  uint64_t* d_empty = d_full + 2 * kGvIssuers;         // [issuer][2] accumulator read out (4 warps)
  uint64_t* mma_done = d_empty + 2 * kGvIssuers;       // every MMA of this CTA retired (one commit per issuer)
  uint64_t* epi_done = mma_done + 1;                   // every epilogue TMEM read retired (4 warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_last = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t KB = args.K / 64;        // 64-weight blocks per row
  const int64_t KU = args.KU;            // 128-deep slices per row (the last may hold one block)
  const int64_t G = gridDim.x;
  const int64_t c = blockIdx.x;
  const int64_t u0 = gv_begin(c, args.units, G), u1 = gv_begin(c + 1, args.units, G);
  const int n_it = static_cast<int>(u1 - u0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGvStages; ++i) {
      mbar_init(smem_u32(&fullc[i]), 1);
      mbar_init(smem_u32(&ready[i]), 1 + 4);
      mbar_init(smem_u32(&empty[i]), 4 + 1);
    }
    for (int i = 0; i < 2 * kGvIssuers; ++i) {
      mbar_init(smem_u32(&d_full[i]), 1);
      mbar_init(smem_u32(&d_empty[i]), 4);
    }
    mbar_init(smem_u32(mma_done), kGvIssuers);
    mbar_init(smem_u32(epi_done), 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_codes);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kGvTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      int64_t t = u0 / KU, ku = u0 - t * KU;
      for (int it = 0; it < n_it; ++it) {
        const int s = it % kGvStages;
        if (it >= kGvStages &&
            !mbar_wait_sleep(smem_u32(&empty[s]), ((it / kGvStages) + 1) & 1, abort_flag, args.status, 64))
          break;
        const uint32_t fc = smem_u32(&fullc[s]), rb = smem_u32(&ready[s]);
        mbar_arrive_expect_tx(fc, kGvCBytes);
        tma_load_2d(smem_u32(base + s * kGvCBytes), &tm_codes, fc, static_cast<int32_t>(ku * (kGvKS / 2)),
                    static_cast<int32_t>(t * kGvRows));
        mbar_arrive_expect_tx(rb, kGvXBytes);
        const uint32_t xs = smem_u32(base + kGvOffX + s * kGvXBytes);
        tma_load_2d(xs, &tm_x, rb, static_cast<int32_t>(ku * kGvKS), 0);
        tma_load_2d(xs + kGvXBytes / 2, &tm_x, rb, static_cast<int32_t>(ku * kGvKS + 64), 0);
        ++issued;
        if (++ku == KU) { ku = 0; ++t; }
      }
      if (*abort_flag) {
        // codes and activations still in flight must land before the CTA exits
        // (the ready barrier also waits for decoder arrivals that may never
        // come, so its wait is bounded and only the TMA bytes matter here)
        for (int it = max(0, issued - kGvStages); it < issued; ++it) {
          const uint32_t fc = smem_u32(&fullc[it % kGvStages]);
          const uint64_t t0 = global_ns();
          while (!mbar_try_wait(fc, (it / kGvStages) & 1) && global_ns() - t0 < qlora_drain_limit()) {}
          const uint32_t rb = smem_u32(&ready[it % kGvStages]);
          const uint64_t t1 = global_ns();
          while (!mbar_try_wait(rb, (it / kGvStages) & 1) && global_ns() - t1 < qlora_drain_limit()) {}
        }
      }
    }
  } else if (warp == 1 || warp == kGvIssuerWarp1) {
    // ---------------------------------------------------------- MMA issuers
    // Issuer i takes the CTA's slices it = i (mod 2) and accumulates them
    // into D[i][segment parity]; for every tile piece (segment) it commits
    // d_full[i][.] once -- also when it had no slice in that piece, which
    // the epilogue knows from the same slice numbering.  Per slice: one
    // barrier wait, 8 MMAs, one commit.  The activation descriptor's address
    // field (bits 0..13, address >> 4) is advanced by plain adds: every slot
    // lies below 256 KB, so the add never carries out of the field.
    if (lane == 0) {
      const int me = (warp == 1) ? 0 : 1;
      constexpr uint32_t idesc = idesc_bf16(kGvRows, kGvNT, 0, 0);
      const uint64_t xdesc0 = sw128_desc(smem_u32(base + kGvOffX), 16, 1024);
      int64_t u = u0;
      int j = 0;
      bool ok = true;
      while (u < u1 && ok) {
        const int64_t t = u / KU;
        const int64_t seg_end = min(u1, (t + 1) * KU);
        const int it_a = static_cast<int>(u - u0), it_b = static_cast<int>(seg_end - u0);
        const uint32_t d_col = tmem + 32u * (2 * me + (j & 1));
        if (j >= 2 && !mbar_wait(smem_u32(&d_empty[2 * me + (j & 1)]), ((j >> 1) + 1) & 1, abort_flag, args.status))
          break;
        bool first = true;
        for (int it = it_a + (((it_a & 1) != me) ? 1 : 0); it < it_b; it += kGvIssuers) {
          const int s = it % kGvStages;
          if (!mbar_wait(smem_u32(&ready[s]), (it / kGvStages) & 1, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t xdesc = xdesc0 + static_cast<uint64_t>((s * kGvXBytes) >> 4);
          const uint32_t a_col = tmem + kGvTmemA0 + kGvASlotCols * s;
#pragma unroll
          for (int k = 0; k < kGvKS / 16; ++k)
            umma_bf16_ts(d_col, a_col + 8u * k,
                         xdesc + static_cast<uint64_t>(((k >> 2) * (kGvXBytes / 2) + 32 * (k & 3)) >> 4), idesc,
                         (first && k == 0) ? 0u : 1u);
          umma_commit(smem_u32(&empty[s]));
          first = false;
        }
        if (!ok) break;
        umma_commit(smem_u32(&d_full[2 * me + (j & 1)]));
        u = seg_end;
        ++j;
      }
      umma_commit(smem_u32(mma_done));
    }
  } else if (warp < kGvEpiWarp0) {
    // ------------------------------------------------------------- dequant
    const int g = (warp - 2) >> 2;
    const int q = warp & 3;                          // TMEM lane quarter of this warp
    const int row = q * 32 + lane;                   // weight row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t c_off = row * (kGvKS / 2), c_swz = (row >> 1) & 3;   // 64-byte rows, 64-byte swizzle
    constexpr int GG = kGvGroups;
    const NF4Shr sh = nf4_shr();
    // raw block-scale inputs (two blocks) of this thread's stages, loaded one
    // own stage ahead; the cursor (pit, pt, pku) walks stages g, g + 3, ...
    int pit = g;
    int64_t pt = (u0 + g) / KU, pku = (u0 + g) - pt * KU;
    auto load_next = [&](uint32_t (&rq)[2], float (&rs)[2]) {
#pragma unroll
      for (int h = 0; h < 2; ++h) { rq[h] = 0; rs[h] = 0.0f; }
      if (pit < n_it) {
        const int64_t n = pt * kGvRows + row;
        if (n < args.N) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int64_t kb = 2 * pku + h;
            if (kb < KB) {
              const int64_t b = n * KB + kb;
              if (args.dq) { rq[h] = __ldg(args.q8 + b); rs[h] = __ldg(args.s2 + (b >> 8)); }
              else rs[h] = __ldg(args.absmax_f32 + b);
            }
          }
        }
      }
      pit += GG;
      pku += GG;
      while (pku >= KU) { pku -= KU; ++pt; }
    };
    uint32_t qa[2], qb[2];
    float sa[2], sb[2];
    load_next(qa, sa);
    load_next(qb, sb);
    for (int it = g; it < n_it; it += GG) {
      const int s = it % kGvStages;
      float scale[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) scale[h] = args.dq ? __fmul_rn(dq_value(qa[h], args.dq), sa[h]) : sa[h];
#pragma unroll
      for (int h = 0; h < 2; ++h) { qa[h] = qb[h]; sa[h] = sb[h]; }
      load_next(qb, sb);
      if (!mbar_wait_warp(smem_u32(&fullc[s]), (it / kGvStages) & 1, abort_flag, args.status)) break;
      const uint8_t* cs = base + s * kGvCBytes + c_off;
      uint4 cc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) cc[i] = *reinterpret_cast<const uint4*>(cs + ((static_cast<uint32_t>(i) ^ c_swz) << 4));
      // the slot's previous slice is out of the MMA (normally long done: the
      // producer waited for the same phase before loading these codes)
      if (it >= kGvStages &&
          !mbar_wait_warp(smem_u32(&empty[s]), ((it / kGvStages) + 1) & 1, abort_flag, args.status))
        break;
      tc_fence_after();
      const uint32_t tcol = tmem + lane_base + kGvTmemA0 + kGvASlotCols * s;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const NF4Table tab = nf4_table(scale[h]);
        const uint32_t cw[8] = {cc[2 * h].x, cc[2 * h].y, cc[2 * h].z, cc[2 * h].w,
                                cc[2 * h + 1].x, cc[2 * h + 1].y, cc[2 * h + 1].z, cc[2 * h + 1].w};
        uint32_t o[32];
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          uint32_t d[4];
          nf4_decode8(cw[w], tab, d, sh);
          o[4 * w + 0] = d[0]; o[4 * w + 1] = d[1]; o[4 * w + 2] = d[2]; o[4 * w + 3] = d[3];
        }
        tmem_st32(tcol + 32u * h, o);
      }
      // the codes are consumed (every stored word depends on them): free the slot
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ready[s]));
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int et = threadIdx.x - kGvEpiWarp0 * 32;   // 0..127
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const int64_t U = args.units;
    int64_t u = u0;
    int j = 0;
    const bool t_ok = gv_adapter_T(args, c, G, et, sT, abort_flag);
    while (u < u1 && t_ok) {
      const int64_t t = u / KU;
      const int64_t seg_end = min(u1, (t + 1) * KU);
      const bool whole = (u == t * KU) && (seg_end == (t + 1) * KU);
      const int64_t n = t * kGvRows + row;
      // adapter term z[m] = sum_j (s T)[m, j] B[n, j] in fp32, computed while
      // the tile is still streaming (it does not depend on the accumulator)
      float z[16];
#pragma unroll
      for (int m = 0; m < 16; ++m) z[m] = 0.0f;
      if (n < args.N) {
        const __nv_bfloat16* brow = args.B + n * args.r;
        for (int j0 = 0; j0 < args.r; j0 += 8) {
          float bv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) bv[i] = (j0 + i < args.r) ? __bfloat162float(brow[j0 + i]) : 0.0f;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (j0 + i < args.r) {
#pragma unroll
              for (int m = 0; m < 16; ++m)
                if (m < args.M) z[m] = fmaf(sT[m * args.r + j0 + i], bv[i], z[m]);
            }
          }
        }
      }
      // every epilogue thread reaches this barrier, and all leave the loop
      // together if any of them gave up waiting
      bool got = mbar_wait_sleep(smem_u32(&d_full[0 + (j & 1)]), (j >> 1) & 1, abort_flag, args.status, 256);
      got = got && mbar_wait_sleep(smem_u32(&d_full[2 + (j & 1)]), (j >> 1) & 1, abort_flag, args.status, 256);
      if (!named_bar_and(1, 128, got)) break;
      tc_fence_after();
      // issuer i holds part of this piece iff it had a slice in it
      const int it_a = static_cast<int>(u - u0), it_b = static_cast<int>(seg_end - u0);
      float y[16];
#pragma unroll
      for (int m = 0; m < 16; ++m) y[m] = 0.0f;
#pragma unroll
      for (int i = 0; i < kGvIssuers; ++i) {
        if (it_b - it_a >= 2 || (it_a & 1) == i) {
          uint32_t v[16];
          tmem_ld16(tmem + lane_base + 32u * (2 * i + (j & 1)), v);
          tmem_ld_wait();
#pragma unroll
          for (int m = 0; m < 16; ++m) y[m] += __uint_as_float(v[m]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&d_empty[0 + (j & 1)]));
        mbar_arrive(smem_u32(&d_empty[2 + (j & 1)]));
      }
      bool finish = whole;
      if (!whole) {
        // partial tile: publish, count, and the last arrival adds them up
        const int slot = (u == u0) ? 0 : 1;
        float4* dst = reinterpret_cast<float4*>(args.part + ((c * 2 + slot) * kGvRows + row) * 16);
        if (QLORA_CHECK(c < kGvMaxCtas && row < kGvRows && t < args.units / KU, 301)) {
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_float4(y[4 * i], y[4 * i + 1], y[4 * i + 2], y[4 * i + 3]);
        }
        named_bar_sync(1, 128);   // every partial write of the CTA before the release below
        const int64_t cf = gv_cta_of(t * KU, U, G), cl = gv_cta_of((t + 1) * KU - 1, U, G);
        if (et == 0) {
          const int old = static_cast<int>(atom_add_acq_rel_gpu(reinterpret_cast<unsigned int*>(args.cnt + t), 1u));
          *s_last = (old == static_cast<int>(cl - cf)) ? 1 : 0;
        }
        named_bar_sync(1, 128);   // the acquire above before any partial read of the CTA
        finish = *s_last != 0;
        if (finish) {
#pragma unroll
          for (int m = 0; m < 16; ++m) y[m] = 0.0f;
          for (int64_t cc = cf; cc <= cl; ++cc) {
            const int sl = (t == gv_begin(cc, U, G) / KU) ? 0 : 1;
            if (!QLORA_CHECK(cc >= 0 && cc < kGvMaxCtas, 302)) break;
            const float4* src = reinterpret_cast<const float4*>(args.part + ((cc * 2 + sl) * kGvRows + row) * 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float4 p = __ldcg(src + i);
              y[4 * i] += p.x; y[4 * i + 1] += p.y; y[4 * i + 2] += p.z; y[4 * i + 3] += p.w;
            }
          }
          if (et == 0) args.cnt[t] = 0;   // leave the counter as found
        }
      }
      if (finish && n < args.N) {
        // frozen-base sum plus adapter term, one rounding to bf16
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m < args.M) args.Y[static_cast<int64_t>(m) * args.N + n] = __float2bfloat16_rn(y[m] + z[m]);
      }
      u = seg_end;
      ++j;
    }
    // this warp's TMEM reads are complete (tcgen05.wait::ld above)
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(epi_done));
  }

  // every MMA (both issuers) and every epilogue TMEM read must have retired
  // before TMEM is released; the owner's lane 0 waits for both explicitly
  // (bounded, ignoring abort) once its own issuing is over -- the other 31
  // lanes wait at the __syncwarp below instead of polling all kernel long
  if (warp == 1 && lane == 0) {
    const uint32_t bars2[2] = {smem_u32(mma_done), smem_u32(epi_done)};
    for (int i = 0; i < 2; ++i) {
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(bars2[i], 0)) {
        __nanosleep(64);
        if (global_ns() - t0 > qlora_wait_limit()) {
          *abort_flag = 1;
          if (args.status) atomicOr(args.status, QLORA_DEV_TIMEOUT);
          break;
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
    tmem_dealloc(tmem, kGvTmemCols);
  }
}

}  // namespace qlora
