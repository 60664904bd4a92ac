// qlora.cu -- libqlora: the C ABI declared in include/qlora.h.
//
// Host side of every entry point: argument validation (before anything is
// enqueued), tensor-map construction for the TMA loads, workspace carving,
// and the kernel sequence on the caller's stream.  The only process state is
// the cached driver entry point for tensor-map encoding and a per-device
// note that the large-shared-memory kernel attributes are set.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "qlora.h"
#ifndef QLORA_NO_NVTX
#include <nvtx3/nvToolsExt.h>
#endif
#include "ptx.cuh"
#include "nf4_constants.cuh"
#include "nf4_decode.cuh"
#include "codec.cuh"
#include "gemm_nf4.cuh"
#include "skinny.cuh"
#include "gemm_nf4_pair.cuh"
#include "gemv_nf4.cuh"
#include "adam.cuh"
#include "merge.cuh"
#include "dropout.cuh"

using namespace qlora;

namespace {

// ------------------------------------------------------------ small helpers
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t rup(int64_t a, int64_t b) { return cdiv(a, b) * b; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D tensor map: `inner` elements per row (contiguous), `outer` rows,
// `row_bytes` between rows.  Out-of-bounds boxes are zero-filled.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  std::memset(m, 0, sizeof(*m));
  return fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool bf16_map(CUtensorMap* m, const void* p, uint64_t cols, uint64_t rows, uint64_t ld_elems,
              uint32_t box_c, uint32_t box_r) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p, cols, rows, ld_elems * 2, box_c, box_r,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

// A named NVTX range around each enqueueing entry point of the C ABI, so
// that a timeline tool shows which call enqueued which kernels (header-only
// NVTX 3: without a tool attached a push or pop checks one pointer).  The
// no-allocation forward has none.  -DQLORA_NO_NVTX compiles them out.
struct NvtxRange {
#ifndef QLORA_NO_NVTX
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
#else
  explicit NvtxRange(const char*) {}
#endif
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// kernels with > 48 KB of dynamic shared memory need the opt-in once per device
bool ensure_smem_attrs() {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load() & bit) return true;
  const int max_smem = 227 * 1024;
  bool ok = cudaFuncSetAttribute(k_gemm_nf4<kModeFwd>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_gemm_nf4<kModeDx>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes) == cudaSuccess;
  const void* pair_kernels[] = {
      reinterpret_cast<const void*>(k_gemm_nf4_pair<kModeFwd, false, 1>), reinterpret_cast<const void*>(k_gemm_nf4_pair<kModeDx, false, 1>),
      reinterpret_cast<const void*>(k_gemm_nf4_pair<kModeFwd, true, 1>), reinterpret_cast<const void*>(k_gemm_nf4_pair<kModeDx, true, 1>),
      reinterpret_cast<const void*>(k_gemm_nf4_pair<kModeFwd, false, 2>), reinterpret_cast<const void*>(k_gemm_nf4_pair<kModeDx, false, 2>),
      reinterpret_cast<const void*>(k_gemm_nf4_pair<kModeFwd, true, 2>), reinterpret_cast<const void*>(k_gemm_nf4_pair<kModeDx, true, 2>)};
  for (const void* k : pair_kernels)
    ok = ok && cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmemBytes) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_skinny<0, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_skinny<0, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_skinny<1, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(k_gemv_nf4, cudaFuncAttributeMaxDynamicSharedMemorySize, kGvSmemBytes) == cudaSuccess;
  if (ok) done.fetch_or(bit);
  return ok;
}

// streaming multiprocessors of the current device (cached per device)
int sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int v = cache[dev].load();
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev].store(v);
  }
  return v;
}

// M tiles per pair launch of the fused GEMM: 1 (256 rows) or 2 (512 rows).
// Two tiles feed every dequantised weight stage to 512 tokens, which halves
// the decode work per flop; one tile gives twice as many pair tiles, which
// packs better into the pairs of SMs when the grid is a few waves.  The
// estimate takes a 512-row tile at kPair2Cost / 10 of a 256-row tile's
// time (both decode the same weights; the larger does twice the MMAs):
// 1.5-1.6 measured on B200 over the LLaMA-7B and 65B projection shapes.
// qlora_debug_set_pair_mtiles can force either (0 = this choice).
std::atomic<int> g_force_mtiles{0};
constexpr int64_t kPair2Cost = 16;
int pair_mtiles(int64_t M, int64_t out_cols) {
  const int f = g_force_mtiles.load();
  if (f == 1 || f == 2) return f;
  if (M <= 256) return 1;
  const int64_t pairs = std::max<int64_t>(1, sm_count() / 2);
  const int64_t nt = cdiv(out_cols, 256);
  const int64_t w1 = cdiv(nt * cdiv(M, 256), pairs), w2 = cdiv(nt * cdiv(M, 512), pairs);
  return (w2 * kPair2Cost < w1 * 10) ? 2 : 1;
}

// Record a caller's timing event on the stream.  Under stream capture the
// record becomes an event node of the graph (an ordinary cudaEventRecord
// would only add an ordering dependency), so that every replay records it.
cudaError_t record_event(cudaEvent_t e, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    return cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
  return cudaEventRecord(e, st);
}

qlora_status check_launch() {
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// ------------------------------------------------------------- validation
qlora_status check_weight(const qlora_nf4_weight* w, bool need_arrays) {
  if (!w) return QLORA_ERR_INVALID_ARG;
  if (w->rows < 1 || w->cols < 64 || (w->cols % 64) != 0) return QLORA_ERR_INVALID_ARG;
  if (w->rows > (int64_t(1) << 31) || w->cols > (int64_t(1) << 31)) return QLORA_ERR_UNSUPPORTED;
  if (w->blocksize != 64 || w->group != 256) return QLORA_ERR_UNSUPPORTED;
  if (w->reserved != 0 || w->double_quant < kDqNone || w->double_quant > kDqE4M3) return QLORA_ERR_INVALID_ARG;
  if (!need_arrays) return QLORA_OK;
  if (!w->codes || !aligned16(w->codes)) return QLORA_ERR_INVALID_ARG;
  if (w->double_quant) {
    if (!w->absmax_q8 || !w->group_scale) return QLORA_ERR_INVALID_ARG;
  } else {
    if (!w->absmax_f32 || !aligned16(w->absmax_f32)) return QLORA_ERR_INVALID_ARG;
  }
  return QLORA_OK;
}

// ------------------------------------------------------ skinny planning
struct SkPlan {
  int64_t P;
  int64_t Qtot;
  int Qn;
  int ptiles;
  int qchunks;
  int num_chunks;
  int splits;
  int per_split;
  int stages;
  size_t partial_bytes;
  int ctas() const { return ptiles * splits * qchunks; }
};

// Split the contraction so that the launch has at most `target` CTAs (one
// wave: a CTA's fixed cost -- TMEM, pipeline fill, epilogue -- is a large
// part of its time, so a second, partly filled round of CTAs nearly doubles
// the kernel), or exactly `force_splits` splits when given.  Fewer splits
// also mean less fp32 partial traffic (written, then re-read by the CTA that
// finishes the tile).
SkPlan plan_skinny(int64_t P, int64_t J, int64_t Qtot, int64_t target = 148, int64_t force_splits = 0) {
  SkPlan pl{};
  pl.P = P;
  pl.Qtot = Qtot;
  pl.Qn = static_cast<int>(std::min<int64_t>(Qtot, 256));
  pl.qchunks = static_cast<int>(cdiv(Qtot, 256));
  pl.num_chunks = static_cast<int>(cdiv(J, 64));
  const int64_t ptiles = cdiv(P, kSkBM);
  pl.ptiles = static_cast<int>(ptiles);
  int64_t splits = force_splits > 0 ? force_splits : target / (ptiles * pl.qchunks);
  splits = std::max<int64_t>(1, std::min<int64_t>(splits, std::max(1, pl.num_chunks / 2)));
  pl.per_split = static_cast<int>(cdiv(pl.num_chunks, splits));
  pl.splits = static_cast<int>(cdiv(pl.num_chunks, pl.per_split));
  const uint32_t stage_bytes = kSkABytes + static_cast<uint32_t>(pl.Qn) * 128u;
  pl.stages = static_cast<int>(std::max<uint32_t>(2, std::min<uint32_t>(6, (200u * 1024u) / stage_bytes)));
  pl.partial_bytes = (pl.splits * pl.qchunks > 1) ? static_cast<size_t>(pl.splits) * P * Qtot * 4 : 0;
  return pl;
}

size_t skinny_smem(const SkPlan& pl) {
  return static_cast<size_t>(pl.stages) * (kSkABytes + pl.Qn * 128u) + 1024 + 256;
}

// One adapter product: its plan, operand tensor maps and arguments.
struct SkJob {
  SkPlan pl;
  CUtensorMap ta, tb;
  SkinnyArgs a;
};

SkinnyArgs sk_args(const SkPlan& pl, float* partial, unsigned int* cnt, int* status) {
  SkinnyArgs a{};
  a.vscale = 1.0f;
  a.partial_elems = static_cast<int64_t>(pl.partial_bytes / 4);
  a.P = pl.P;
  a.Qn = pl.Qn;
  a.Qtot = pl.Qtot;
  a.num_chunks = pl.num_chunks;
  a.chunks_per_split = pl.per_split;
  a.stages = pl.stages;
  a.ptiles = pl.ptiles;
  a.splits = pl.splits;
  a.qchunks = pl.qchunks;
  a.partial = partial;
  a.cnt = cnt;
  a.status = status;
  return a;
}

// One launch for one job, or for two independent jobs of the same operand
// majorness (CTAs [0, n0) run j0, the rest j1).
template <int A_MN, int B_MN>
qlora_status launch_skinny(const SkJob& j0, const SkJob* j1, cudaStream_t st) {
  const int n0 = j0.pl.ctas();
  const int n1 = j1 ? j1->pl.ctas() : 0;
  const size_t smem = std::max(skinny_smem(j0.pl), j1 ? skinny_smem(j1->pl) : size_t(0));
  const SkJob& o = j1 ? *j1 : j0;
  k_skinny<A_MN, B_MN><<<static_cast<unsigned>(n0 + n1), kSkThreads, smem, st>>>(j0.ta, j0.tb, o.ta, o.tb, j0.a,
                                                                                 o.a, n0);
  return check_launch();
}

// -------------------------------------------------------- workspace layout
struct Ws {
  size_t partial, partial2, cnt, t32, sx, ghl, thl, bpad, gv_part, gv_cnt, gv_tpart, total;
};

// Token counts up to this take the weight-streaming decode kernel.
constexpr int64_t kDecodeMaxM = kGvNT;

struct Dims {
  int64_t M, N, K;
  int r, r8, r16, r64, Qh;
};

Dims dims_of(int64_t M, int64_t N, int64_t K, int r) {
  Dims d;
  d.M = M; d.N = N; d.K = K; d.r = r;
  d.r8 = static_cast<int>(rup(r, 8));
  d.r16 = static_cast<int>(rup(r, 16));
  d.r64 = static_cast<int>(rup(r, 64));
  d.Qh = static_cast<int>(rup(2 * d.r16, 64));
  return d;
}

// Skinny plans of one layer call (dA and dB share one launch).
struct SkPlans {
  SkPlan T, G, dA, dB;
};
SkPlans plans_of(const Dims& d) {
  SkPlans p;
  // T and dA + dB are planned to about half the SMs: the fused GEMM behind
  // each of them (a programmatic dependent launch) needs their results only
  // at its end and starts on the SMs they leave free (measured on the
  // LLaMA-7B layer step: +0.7 %; G, which gates the dA + dB launch, keeps
  // the whole GPU)
  p.T = plan_skinny(d.M, d.K, d.r16, 64);
  p.G = plan_skinny(d.M, d.N, d.r64);
  // dA and dB share one launch: one split count for both, so that together
  // they fill (at most) half the SMs
  const int64_t qc = cdiv(d.Qh, 256);
  const int64_t pt = (cdiv(d.K, kSkBM) + cdiv(d.N, kSkBM)) * qc;
  const int64_t sp = std::max<int64_t>(1, 74 / pt);
  p.dA = plan_skinny(d.K, d.M, d.Qh, 0, sp);
  p.dB = plan_skinny(d.N, d.M, d.Qh, 0, sp);
  return p;
}
// Arrival counters: T, G, dA, dB tiles, one 32-bit word each.
size_t cnt_words(const SkPlans& p) { return p.T.ptiles + p.G.ptiles + p.dA.ptiles + p.dB.ptiles; }

// The decode kernel's scratch (M <= 16): partial tiles, per-tile counters
// followed by the two T-phase counters, and the partials of T.
void gv_layout(const Dims& d, Ws& w, size_t& off) {
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  w.gv_part = w.gv_cnt = w.gv_tpart = off;
  if (d.M <= kDecodeMaxM) {
    w.gv_part = off; off += a256(static_cast<size_t>(kGvMaxCtas) * 2 * kGvRows * kGvNT * 4);
    w.gv_cnt = off; off += a256(static_cast<size_t>(cdiv(d.N, kGvRows) + 2) * 4);
    w.gv_tpart = off; off += a256(static_cast<size_t>(kGvMaxCtas) * d.M * d.r * 4);
  }
}

Ws ws_layout(const Dims& d) {
  const SkPlans pl = plans_of(d);
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  Ws w{};
  size_t off = 0;
  // T and G run alone; dA and dB run side by side in one launch
  w.partial = off;
  w.partial2 = off + a256(pl.dA.partial_bytes);
  off += a256(std::max({pl.T.partial_bytes, pl.G.partial_bytes, a256(pl.dA.partial_bytes) + pl.dB.partial_bytes}));
  w.cnt = off; off += a256(cnt_words(pl) * 4);
  w.t32 = off; off += a256(static_cast<size_t>(d.M) * d.r * 4);
  w.sx = off; off += a256(static_cast<size_t>(2 * d.M) * d.r8 * 2);
  w.ghl = off; off += a256(static_cast<size_t>(d.M) * d.Qh * 2);
  w.thl = off; off += a256(static_cast<size_t>(d.M) * d.Qh * 2);
  w.bpad = off; off += a256(static_cast<size_t>(d.N) * d.r8 * 2);
  gv_layout(d, w, off);
  w.total = off;
  return w;
}

// LoRA dropout of one call: Philox key, the integer cut ceil(p 2^32) and
// fp32(1 / (1 - p)).
struct DropCfg {
  uint64_t seed, thr;
  float inv_q;
};
bool dropout_cfg(double p, uint64_t seed, DropCfg* c) {
  if (!std::isfinite(p) || p < 0.0 || p >= 1.0) return false;
  c->seed = seed;
  c->thr = static_cast<uint64_t>(std::ceil(p * 4294967296.0));
  c->inv_q = static_cast<float>(1.0 / (1.0 - p));
  return true;
}
// Workspace of the dropout entries: the plain layout, then X * keep (bf16
// [M, K]), the frozen-path dX in fp32 ([M, K]) and G in fp32 ([M, r]).
struct WsDrop {
  size_t xd, dxf, g32, total;
};
WsDrop ws_drop_layout(const Dims& d) {
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  WsDrop w{};
  size_t off = ws_layout(d).total;
  w.xd = off; off += a256(static_cast<size_t>(d.M) * d.K * 2);
  w.dxf = off; off += a256(static_cast<size_t>(d.M) * d.K * 4);
  w.g32 = off; off += a256(static_cast<size_t>(d.M) * d.r * 4);
  w.total = off;
  return w;
}
unsigned dropout_grid(int64_t items) {
  const int sms = std::max(1, sm_count());
  return static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(cdiv(items, kDropThreads), 16LL * sms)));
}
// Xd = X * keep over the M x K activations.
qlora_status run_dropout_x(const void* X, void* Xd, const Dims& d, const DropCfg& c, cudaStream_t cs) {
  const int64_t n = d.M * d.K;
  k_dropout_x<<<dropout_grid(n / 8), kDropThreads, 0, cs>>>(static_cast<const __nv_bfloat16*>(X),
                                                              static_cast<__nv_bfloat16*>(Xd), n, c.seed, c.thr);
  return check_launch();
}

qlora_status check_linear(int64_t M, const qlora_nf4_weight* Wq, int r, float alpha, const void* workspace,
                          size_t ws_bytes, bool dropout = false) {
  qlora_status st = check_weight(Wq, true);
  if (st != QLORA_OK) return st;
  if (M < 1 || M > (int64_t(1) << 31)) return QLORA_ERR_INVALID_ARG;
  if (r < 1 || r > 256) return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
  if (Wq->rows % 8 != 0) return QLORA_ERR_UNSUPPORTED;
  if (!workspace || !aligned16(workspace)) return QLORA_ERR_WORKSPACE;
  const Dims d = dims_of(M, Wq->rows, Wq->cols, r);
  if (ws_bytes < (dropout ? ws_drop_layout(d).total : ws_layout(d).total)) return QLORA_ERR_WORKSPACE;
  return QLORA_OK;
}

// The final transform of a token-indexed product (T or G) into `a`.
void sk_rows(SkinnyArgs& a, const Dims& d, float s, float* f32, __nv_bfloat16* s_bf16, __nv_bfloat16* hl) {
  a.finish = kFinRows;
  a.s = s; a.r = d.r; a.r8 = d.r8; a.r16 = d.r16; a.Qh = d.Qh;
  a.f32 = f32; a.s_bf16 = s_bf16; a.hl = hl;
}
// Counter words of T, G, dA, dB inside the workspace's counter region.
unsigned int* cnt_T(uint8_t* ws, const Ws& L) { return reinterpret_cast<unsigned int*>(ws + L.cnt); }
unsigned int* cnt_G(uint8_t* ws, const Ws& L, const SkPlans& p) { return cnt_T(ws, L) + p.T.ptiles; }
unsigned int* cnt_dA(uint8_t* ws, const Ws& L, const SkPlans& p) { return cnt_G(ws, L, p) + p.G.ptiles; }
unsigned int* cnt_dB(uint8_t* ws, const Ws& L, const SkPlans& p) { return cnt_dA(ws, L, p) + p.dA.ptiles; }

// Clear the arrival counters of one call (they must start at zero).
qlora_status clear_counters(uint8_t* ws, const Ws& L, const SkPlans& p, cudaStream_t st) {
  return cudaMemsetAsync(ws + L.cnt, 0, cnt_words(p) * 4, st) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// T = X A^T  (fp32 into t32, and optionally s*T in bf16 planes into sx), one
// launch.  The caller has cleared the counters.
qlora_status run_T(const void* X, const void* A, const Dims& d, float s, uint8_t* ws, const Ws& L, float* t32,
                   __nv_bfloat16* sx, int* status, cudaStream_t st, float vscale = 1.0f) {
  const SkPlans P = plans_of(d);
  SkJob j;
  j.pl = P.T;
  if (!bf16_map(&j.ta, X, d.K, d.M, d.K, 64, kSkBM)) return QLORA_ERR_CUDA;
  if (!bf16_map(&j.tb, A, d.K, d.r, d.K, 64, static_cast<uint32_t>(j.pl.Qn))) return QLORA_ERR_CUDA;
  j.a = sk_args(j.pl, reinterpret_cast<float*>(ws + L.partial), cnt_T(ws, L), status);
  sk_rows(j.a, d, s, t32, sx, nullptr);
  j.a.vscale = vscale;
  return launch_skinny<0, 0>(j, nullptr, st);
}

const void* padded_B(const void* B, const Dims& d, uint8_t* ws, const Ws& L, cudaStream_t st, qlora_status* rc) {
  *rc = QLORA_OK;
  if (d.r % 8 == 0) return B;
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(ws + L.bpad);
  const int64_t n = d.N * d.r8;
  k_pad_cols<<<static_cast<unsigned>(cdiv(n, 256)), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(B), d.N, d.r,
                                                                  d.r8, dst);
  *rc = check_launch();
  return dst;
}

qlora_status launch_gemm(int mode, const CUtensorMap& tact, const CUtensorMap& tcodes, const CUtensorMap& tla,
                         const CUtensorMap& tlb, const GemmArgs& a, const qlora_gemm_events* ev,
                         cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(cdiv(a.out_cols, kGemmBN)), static_cast<unsigned>(cdiv(a.M, kGemmBM)));
  if (ev && ev->gemm_start && record_event(static_cast<cudaEvent_t>(ev->gemm_start), st) != cudaSuccess)
    return QLORA_ERR_CUDA;
  if (mode == kModeFwd)
    k_gemm_nf4<kModeFwd><<<grid, kGemmThreads, kGemmSmemBytes, st>>>(tact, tcodes, tla, tlb, a);
  else
    k_gemm_nf4<kModeDx><<<grid, kGemmThreads, kGemmSmemBytes, st>>>(tact, tcodes, tla, tlb, a);
  qlora_status rc = check_launch();
  if (rc == QLORA_OK && ev && ev->gemm_end &&
      record_event(static_cast<cudaEvent_t>(ev->gemm_end), st) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return rc;
}


// Fused NF4 GEMM of one call: tensor maps + dispatch.  M > 128 takes the
// 2-SM pair kernel (256 x 256 or 512 x 256 tiles per pair, pair_mtiles),
// smaller M the 1-CTA kernel.
//   fwd: act = X [M, K], la = s*T planes [2M, r8], lb = B [N, r8], out Y [M, N]
//   dX : act = dY [M, N], la = s*G planes [2M, r8], lb = A [r, K], out dX [M, K]
// The fused GEMM of the forward (mode kModeFwd) or of dX (kModeDx), over
// the NF4 weight Wq or, when Wdense is given, over a dense bf16 weight
// [N, K] (plain LoRA; always the 2-SM pair kernel).
qlora_status run_fused(int mode, const void* act, const qlora_nf4_weight* Wq, const void* Wdense, const Dims& d,
                       const void* la, const void* lb, void* out, const qlora_gemm_events* ev, int* status,
                       cudaStream_t cs, float* out_f32 = nullptr, bool fold = true) {
  const bool dense = Wdense != nullptr;
  const bool pair = d.M > 128 || dense;
  const bool fwd = mode == kModeFwd;
  CUtensorMap tact, tcodes, tla, tlb;
  if (fwd) {
    if (!bf16_map(&tact, act, d.K, d.M, d.K, 64, 128)) return QLORA_ERR_CUDA;
    if (dense) {
      if (!bf16_map(&tcodes, Wdense, d.K, d.N, d.K, 64, 128)) return QLORA_ERR_CUDA;
    } else if (!make_map(&tcodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq->codes, d.K / 2, d.N, d.K / 2, 32,
                         pair ? 128 : kGemmBN, CU_TENSOR_MAP_SWIZZLE_32B)) {
      return QLORA_ERR_CUDA;
    }
    if (!bf16_map(&tlb, lb, d.r8, d.N, d.r8, 64, pair ? 128 : kGemmBN)) return QLORA_ERR_CUDA;
  } else {
    if (!bf16_map(&tact, act, d.N, d.M, d.N, 64, 128)) return QLORA_ERR_CUDA;
    if (dense) {
      if (!bf16_map(&tcodes, Wdense, d.K, d.N, d.K, 64, 64)) return QLORA_ERR_CUDA;
    } else if (pair) {
      if (!make_map(&tcodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq->codes, d.K / 2, d.N, d.K / 2, 64, 64,
                    CU_TENSOR_MAP_SWIZZLE_64B))
        return QLORA_ERR_CUDA;
    } else {
      if (!make_map(&tcodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq->codes, d.K / 2, d.N, d.K / 2, 128, 64,
                    CU_TENSOR_MAP_SWIZZLE_128B))
        return QLORA_ERR_CUDA;
    }
    if (!bf16_map(&tlb, lb, d.K, d.r, d.K, 64, 64)) return QLORA_ERR_CUDA;
  }
  if (!bf16_map(&tla, la, d.r8, 2 * d.M, d.r8, 64, 128)) return QLORA_ERR_CUDA;
  GemmArgs a{};
  if (!dense) {
    a.q8 = Wq->absmax_q8; a.s2 = Wq->group_scale; a.absmax_f32 = Wq->absmax_f32; a.dq = Wq->double_quant;
  }
  a.wN = d.N; a.wK = d.K; a.M = d.M;
  a.out_cols = fwd ? d.N : d.K;
  a.ldo = a.out_cols;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.out_f32 = out_f32;
  a.num_kt = static_cast<int>(fwd ? d.K / 64 : cdiv(d.N, 64));
  a.lora_r16 = fold ? d.r16 : 0;
  a.lora_lo_row = d.M;
  a.status = status;
  if (!pair) return launch_gemm(mode, tact, tcodes, tla, tlb, a, ev, cs);
  // the 2-SM kernel writes a bf16 output with TMA stores (64 x 32 boxes)
  // when its rows are 16-byte aligned; fp32 output goes out directly
  CUtensorMap tout = tla;
  if (!out_f32 && (a.ldo % 8) == 0) {
    if (bf16_map(&tout, out, a.out_cols, d.M, a.ldo, 64, 32)) a.tma_out = 1;
    else tout = tla;   // not encodable: direct stores
  }

  if (ev && ev->gemm_start && record_event(static_cast<cudaEvent_t>(ev->gemm_start), cs) != cudaSuccess)
    return QLORA_ERR_CUDA;
  const int mt = pair_mtiles(d.M, a.out_cols);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * cdiv(a.out_cols, 256)), static_cast<unsigned>(cdiv(d.M, 256 * mt)));
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = kPairSmemBytes;
  cfg.stream = cs;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: the GEMM may start while the adapter
  // kernel ahead of it (T, or dA + dB in the backward) is still running;
  // it waits for that kernel only where it reads its results
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e;
  if (mt == 2) {
    if (dense)
      e = fwd ? cudaLaunchKernelEx(&cfg, k_gemm_nf4_pair<kModeFwd, true, 2>, tact, tcodes, tla, tlb, tout, a)
              : cudaLaunchKernelEx(&cfg, k_gemm_nf4_pair<kModeDx, true, 2>, tact, tcodes, tla, tlb, tout, a);
    else
      e = fwd ? cudaLaunchKernelEx(&cfg, k_gemm_nf4_pair<kModeFwd, false, 2>, tact, tcodes, tla, tlb, tout, a)
              : cudaLaunchKernelEx(&cfg, k_gemm_nf4_pair<kModeDx, false, 2>, tact, tcodes, tla, tlb, tout, a);
  } else {
    if (dense)
      e = fwd ? cudaLaunchKernelEx(&cfg, k_gemm_nf4_pair<kModeFwd, true, 1>, tact, tcodes, tla, tlb, tout, a)
              : cudaLaunchKernelEx(&cfg, k_gemm_nf4_pair<kModeDx, true, 1>, tact, tcodes, tla, tlb, tout, a);
    else
      e = fwd ? cudaLaunchKernelEx(&cfg, k_gemm_nf4_pair<kModeFwd, false, 1>, tact, tcodes, tla, tlb, tout, a)
              : cudaLaunchKernelEx(&cfg, k_gemm_nf4_pair<kModeDx, false, 1>, tact, tcodes, tla, tlb, tout, a);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  if (ev && ev->gemm_end && record_event(static_cast<cudaEvent_t>(ev->gemm_end), cs) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return QLORA_OK;
}

// Decode-shaped forward (M <= 16): Y = X W^T + s T B^T, with T = X A^T
// computed in the same launch and written (fp32) to t32.  Persistent
// stream-K launch, one CTA per SM, cooperative (every CTA resident at once:
// the T phases wait across CTAs).  One memset clears the counters first.
qlora_status run_gemv(const void* X, const void* A, const qlora_nf4_weight* Wq, const Dims& d, float* t32,
                      const void* B, void* Y, float alpha_over_r, uint8_t* ws, const Ws& L,
                      const qlora_gemm_events* ev, int* status, cudaStream_t cs, const void* Xt = nullptr,
                      float tscale = 1.0f) {
  if (d.r > kGvMaxRank) return QLORA_ERR_UNSUPPORTED;
  const int64_t tiles = cdiv(d.N, kGvRows);
  const int64_t KU = cdiv(d.K, kGvKS);
  const int64_t units = tiles * KU;
  const int sms = sm_count();
  if (sms <= 0) return QLORA_ERR_CUDA;
  const int64_t grid = std::min<int64_t>(std::min<int64_t>(sms, kGvMaxCtas), units);
  CUtensorMap tx, tc;
  if (!bf16_map(&tx, X, d.K, d.M, d.K, 64, kGvNT)) return QLORA_ERR_CUDA;
  if (!make_map(&tc, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq->codes, d.K / 2, d.N, d.K / 2, kGvKS / 2, kGvRows,
                CU_TENSOR_MAP_SWIZZLE_64B))
    return QLORA_ERR_CUDA;
  GvArgs a{};
  a.q8 = Wq->absmax_q8; a.s2 = Wq->group_scale; a.absmax_f32 = Wq->absmax_f32; a.dq = Wq->double_quant;
  a.N = d.N; a.K = d.K; a.M = static_cast<int>(d.M); a.r = d.r; a.s = alpha_over_r; a.tscale = tscale;
  a.X = static_cast<const __nv_bfloat16*>(Xt ? Xt : X);
  a.A = static_cast<const __nv_bfloat16*>(A);
  a.T = t32;
  a.tpart = reinterpret_cast<float*>(ws + L.gv_tpart);
  a.B = static_cast<const __nv_bfloat16*>(B);
  a.Y = static_cast<__nv_bfloat16*>(Y);
  a.part = reinterpret_cast<float*>(ws + L.gv_part);
  a.cnt = reinterpret_cast<int*>(ws + L.gv_cnt);
  a.tcnt = a.cnt + tiles;
  a.KU = KU;
  a.units = units;
  a.status = status;
  if (cudaMemsetAsync(a.cnt, 0, static_cast<size_t>(tiles + 2) * 4, cs) != cudaSuccess) return QLORA_ERR_CUDA;
  if (ev && ev->gemm_start && record_event(static_cast<cudaEvent_t>(ev->gemm_start), cs) != cudaSuccess)
    return QLORA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kGvThreads);
  cfg.dynamicSmemBytes = kGvSmemBytes;
  cfg.stream = cs;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k_gemv_nf4, tx, tc, a) != cudaSuccess) return QLORA_ERR_CUDA;
  qlora_status rc = check_launch();
  if (rc == QLORA_OK && ev && ev->gemm_end &&
      record_event(static_cast<cudaEvent_t>(ev->gemm_end), cs) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return rc;
}

// Backward body shared by the NF4 entry (Wq) and the dense-bf16 one (Wdense):
// arguments already validated.
qlora_status linear_bwd_core(const void* dY, const void* X, const Dims& d, const qlora_nf4_weight* Wq,
                             const void* Wdense, const void* A, const void* B, float alpha, const float* T_saved,
                             void* dX, void* dA, void* dB, qlora_dtype grad_dtype, void* workspace, int* d_status,
                             const qlora_gemm_events* events, cudaStream_t cs, const DropCfg* drop = nullptr) {
  qlora_status st = QLORA_OK;
  const Ws L = ws_layout(d);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const float s = alpha / static_cast<float>(d.r);
  const SkPlans P = plans_of(d);
  __nv_bfloat16* sG = reinterpret_cast<__nv_bfloat16*>(ws + L.sx);
  __nv_bfloat16* Ghl = reinterpret_cast<__nv_bfloat16*>(ws + L.ghl);
  __nv_bfloat16* Thl = reinterpret_cast<__nv_bfloat16*>(ws + L.thl);

  const void* Bp = padded_B(B, d, ws, L, cs, &st);
  if (st != QLORA_OK) return st;
  st = clear_counters(ws, L, P, cs);
  if (st != QLORA_OK) return st;
  // the adapter's input: X, or X * keep under dropout (regenerated from the
  // call's seed, the same mask as the forward's)
  const WsDrop WD = drop ? ws_drop_layout(d) : WsDrop{};
  const void* Xa = X;
  if (drop) {
    st = run_dropout_x(X, ws + WD.xd, d, *drop, cs);
    if (st != QLORA_OK) return st;
    Xa = ws + WD.xd;
  }
  const float inv_q = drop ? drop->inv_q : 1.0f;
  // 0. T recomputed when the forward's was not kept
  const float* t = T_saved;
  if (!t) {
    float* t32 = reinterpret_cast<float*>(ws + L.t32);
    st = run_T(Xa, A, d, s, ws, L, t32, nullptr, d_status, cs, inv_q);
    if (st != QLORA_OK) return st;
    t = t32;
  }
  // 1. G = dY B -> s*G (bf16 planes, for the dX fold) and [G_hi | G_lo] (for
  //    dA); the same launch turns T into [T_hi | T_lo] (for dB)
  {
    SkJob j;
    j.pl = P.G;
    if (!bf16_map(&j.ta, dY, d.N, d.M, d.N, 64, kSkBM)) return QLORA_ERR_CUDA;
    if (!bf16_map(&j.tb, Bp, d.r8, d.N, d.r8, 64, 64)) return QLORA_ERR_CUDA;
    j.a = sk_args(j.pl, reinterpret_cast<float*>(ws + L.partial), cnt_G(ws, L, P), d_status);
    // under dropout the adapter term of dX is masked per element, so it is
    // added after the GEMM from fp32 G instead of folded into it
    if (drop)
      sk_rows(j.a, d, s, reinterpret_cast<float*>(ws + WD.g32), nullptr, Ghl);
    else
      sk_rows(j.a, d, s, nullptr, sG, Ghl);
    j.a.side_src = t;
    j.a.side_rows = d.M;
    j.a.side_hl = Thl;
    st = launch_skinny<0, 1>(j, nullptr, cs);
    if (st != QLORA_OK) return st;
  }
  // 2. dA = s G^T X (C[k, q] = sum_m X[m, k] Ghl[m, q]) and dB = s dY^T T
  //    (C[n, q] = sum_m dY[m, n] Thl[m, q]) in one launch; ahead of the dX
  //    GEMM, which needs only G as well and overlaps this launch
  {
    const int out_bf16 = grad_dtype == QLORA_BF16 ? 1 : 0;
    SkJob ja, jb;
    ja.pl = P.dA;
    jb.pl = P.dB;
    if (!bf16_map(&ja.ta, Xa, d.K, d.M, d.K, 64, 64)) return QLORA_ERR_CUDA;
    if (!bf16_map(&ja.tb, Ghl, d.Qh, d.M, d.Qh, 64, 64)) return QLORA_ERR_CUDA;
    if (!bf16_map(&jb.ta, dY, d.N, d.M, d.N, 64, 64)) return QLORA_ERR_CUDA;
    if (!bf16_map(&jb.tb, Thl, d.Qh, d.M, d.Qh, 64, 64)) return QLORA_ERR_CUDA;
    ja.a = sk_args(ja.pl, reinterpret_cast<float*>(ws + L.partial), cnt_dA(ws, L, P), d_status);
    jb.a = sk_args(jb.pl, reinterpret_cast<float*>(ws + L.partial2), cnt_dB(ws, L, P), d_status);
    for (SkinnyArgs* a : {&ja.a, &jb.a}) {
      a->finish = kFinGrad;
      a->s = s; a->r = d.r; a->r8 = d.r8; a->r16 = d.r16; a->Qh = d.Qh;
      a->out_bf16 = out_bf16;
    }
    ja.a.transpose = 1;
    ja.a.s = s * inv_q;
    ja.a.out = dA;
    jb.a.transpose = 0;
    jb.a.out = dB;
    st = launch_skinny<1, 1>(ja, &jb, cs);
    if (st != QLORA_OK) return st;
  }
  // 3. dX = dY W^ + (sG) A; under dropout dY W^ in fp32, then one pass
  //    adding s ((G A) * keep) / (1 - p) and rounding once
  if (dX && !drop) {
    st = run_fused(kModeDx, dY, Wq, Wdense, d, sG, A, dX, events, d_status, cs);
    if (st != QLORA_OK) return st;
  } else if (dX) {
    float* dxf = reinterpret_cast<float*>(ws + WD.dxf);
    st = run_fused(kModeDx, dY, Wq, Wdense, d, sG, A, dX, events, d_status, cs, dxf, false);
    if (st != QLORA_OK) return st;
    k_dropout_dx<<<dropout_grid(d.M * (d.K / 8)), kDropThreads, 0, cs>>>(
        dxf, reinterpret_cast<const float*>(ws + WD.g32), static_cast<const __nv_bfloat16*>(A), d.M, d.K, d.r,
        s * inv_q, drop->seed, drop->thr, static_cast<__nv_bfloat16*>(dX));
    st = check_launch();
    if (st != QLORA_OK) return st;
  }
  return st;
}

// Records a failed range check at site 0xFFFF without touching memory: the
// path from a kernel's check to qlora_debug_range_check, in either build.
__global__ void k_range_selftest() {
  if (threadIdx.x == 0) qlora::qlora_range_ok(false, 0xFFFFu);
}

// Validation of the dense-bf16 entries: the same shape rules as the NF4
// weight (N % 8 == 0, K % 64 == 0, 1 <= r <= 256).
qlora_status check_dense(int64_t M, const void* W, int64_t N, int64_t K, int r, float alpha, const void* workspace,
                         size_t ws_bytes) {
  if (!W || !aligned16(W)) return QLORA_ERR_INVALID_ARG;
  if (N < 1 || K < 64 || (K % 64) != 0) return QLORA_ERR_INVALID_ARG;
  if (N > (int64_t(1) << 31) || K > (int64_t(1) << 31)) return QLORA_ERR_UNSUPPORTED;
  if (N % 8 != 0) return QLORA_ERR_UNSUPPORTED;
  if (M < 1 || M > (int64_t(1) << 31)) return QLORA_ERR_INVALID_ARG;
  if (r < 1 || r > 256) return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace)) return QLORA_ERR_WORKSPACE;
  if (ws_bytes < ws_layout(dims_of(M, N, K, r)).total) return QLORA_ERR_WORKSPACE;
  return QLORA_OK;
}

}  // namespace

// =================================================================== ABI
extern "C" {

const char* qlora_version(void) { return "0.1.0"; }

const char* qlora_status_string(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument";
    case QLORA_ERR_UNSUPPORTED: return "unsupported configuration";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_NONFINITE: return "non-finite input";
    case QLORA_ERR_TIMEOUT: return "device wait timed out";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_SCRATCH_LIMIT: return "problem exceeds the fixed no-allocation scratch";
  }
  return "unknown status";
}

void qlora_nf4_codebook(float* out16) {
  if (!out16) return;
  for (int i = 0; i < 16; ++i) out16[i] = kNF4Level[i];
}

qlora_status qlora_nf4_sizes(int64_t rows, int64_t cols, int double_quant, size_t* codes_bytes,
                             size_t* absmax_bytes, size_t* group_bytes) {
  if (!codes_bytes || !absmax_bytes || !group_bytes) return QLORA_ERR_INVALID_ARG;
  if (rows < 1 || cols < 64 || cols % 64 != 0) return QLORA_ERR_INVALID_ARG;
  if (double_quant < kDqNone || double_quant > kDqE4M3) return QLORA_ERR_INVALID_ARG;
  const int64_t blocks = rows * cols / 64;
  *codes_bytes = static_cast<size_t>(rows * cols / 2);
  *absmax_bytes = static_cast<size_t>(double_quant ? blocks : 4 * blocks);
  *group_bytes = static_cast<size_t>(double_quant ? 4 * cdiv(blocks, 256) : 0);
  return QLORA_OK;
}

size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
  if (M < 1 || N < 1 || K < 64 || K % 64 != 0 || r < 1 || r > 256) return 0;
  return ws_layout(dims_of(M, N, K, r)).total;
}

qlora_status qlora_quantize_nf4(const void* W, qlora_dtype w_dtype, const qlora_nf4_weight* out, int* d_status,
                                void* stream) {
  NvtxRange nvtx_range("qlora_quantize_nf4");
  qlora_status st = check_weight(out, true);
  if (st != QLORA_OK) return st;
  if (!W || !aligned16(W)) return QLORA_ERR_INVALID_ARG;
  if (w_dtype != QLORA_F32 && w_dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  if (out->absmax_f32 && !aligned16(out->absmax_f32)) return QLORA_ERR_INVALID_ARG;
  const int64_t nblocks = out->rows * out->cols / 64;
  const unsigned groups = static_cast<unsigned>(cdiv(nblocks, 256));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (w_dtype == QLORA_BF16)
    k_quantize_nf4<<<groups, kQuantThreads, 0, s>>>(
        PtrSrc<__nv_bfloat16>{static_cast<const __nv_bfloat16*>(W)}, nblocks, out->double_quant, out->codes,
        out->absmax_q8, out->group_scale, out->absmax_f32, d_status);
  else
    k_quantize_nf4<<<groups, kQuantThreads, 0, s>>>(PtrSrc<float>{static_cast<const float*>(W)}, nblocks,
                                                    out->double_quant, out->codes, out->absmax_q8,
                                                    out->group_scale, out->absmax_f32, d_status);
  return check_launch();
}

qlora_status qlora_dequantize(const qlora_nf4_weight* Wq, void* W_out, void* stream) {
  NvtxRange nvtx_range("qlora_dequantize");
  qlora_status st = check_weight(Wq, true);
  if (st != QLORA_OK) return st;
  if (!W_out || !aligned16(W_out)) return QLORA_ERR_INVALID_ARG;
  const int64_t nblocks = Wq->rows * Wq->cols / 64;
  k_dequantize_nf4<<<static_cast<unsigned>(cdiv(nblocks, kDeqThreads)), kDeqThreads, 0,
                     static_cast<cudaStream_t>(stream)>>>(Wq->codes, Wq->absmax_q8, Wq->group_scale, Wq->absmax_f32,
                                                          Wq->double_quant, nblocks,
                                                          static_cast<__nv_bfloat16*>(W_out));
  return check_launch();
}

qlora_status qlora_linear_fwd(const void* X, int64_t M, const qlora_nf4_weight* Wq, const void* A, const void* B,
                              int r, float alpha, void* Y, float* T_save, void* workspace, size_t ws_bytes,
                              int* d_status, const qlora_gemm_events* events, void* stream) {
  NvtxRange nvtx_range("qlora_linear_fwd");
  qlora_status st = check_linear(M, Wq, r, alpha, workspace, ws_bytes);
  if (st != QLORA_OK) return st;
  if (!X || !A || !B || !Y || !aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(Y))
    return QLORA_ERR_INVALID_ARG;
  if (T_save && !aligned16(T_save)) return QLORA_ERR_INVALID_ARG;
  if (!ensure_smem_attrs()) return QLORA_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const Dims d = dims_of(M, Wq->rows, Wq->cols, r);
  const Ws L = ws_layout(d);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const float s = alpha / static_cast<float>(r);
  float* t32 = T_save ? T_save : reinterpret_cast<float*>(ws + L.t32);
  __nv_bfloat16* sT = reinterpret_cast<__nv_bfloat16*>(ws + L.sx);

  if (M <= kDecodeMaxM)   // decode shape: one weight-streaming launch (T included)
    return run_gemv(X, A, Wq, d, t32, B, Y, s, ws, L, events, d_status, cs);

  // 1. T = X A^T and s*T (bf16) for the fold
  st = clear_counters(ws, L, plans_of(d), cs);
  if (st != QLORA_OK) return st;
  st = run_T(X, A, d, s, ws, L, t32, sT, d_status, cs);
  if (st != QLORA_OK) return st;
  const void* Bp = padded_B(B, d, ws, L, cs, &st);
  if (st != QLORA_OK) return st;

  // 2. Y = X W^T + (sT) B^T
  return run_fused(kModeFwd, X, Wq, nullptr, d, sT, Bp, Y, events, d_status, cs);
}

qlora_status qlora_linear_bwd(const void* dY, const void* X, int64_t M, const qlora_nf4_weight* Wq, const void* A,
                              const void* B, int r, float alpha, const float* T_saved, void* dX, void* dA, void* dB,
                              qlora_dtype grad_dtype, void* workspace, size_t ws_bytes, int* d_status,
                              const qlora_gemm_events* events, void* stream) {
  NvtxRange nvtx_range("qlora_linear_bwd");
  qlora_status st = check_linear(M, Wq, r, alpha, workspace, ws_bytes);
  if (st != QLORA_OK) return st;
  if (!dY || !X || !A || !B || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(dY) || !aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(dA) || !aligned16(dB))
    return QLORA_ERR_INVALID_ARG;
  if ((dX && !aligned16(dX)) || (T_saved && !aligned16(T_saved))) return QLORA_ERR_INVALID_ARG;
  if (grad_dtype != QLORA_F32 && grad_dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  if (!ensure_smem_attrs()) return QLORA_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const Dims d = dims_of(M, Wq->rows, Wq->cols, r);
  return linear_bwd_core(dY, X, d, Wq, nullptr, A, B, alpha, T_saved, dX, dA, dB, grad_dtype, workspace, d_status,
                         events, cs);
}

size_t qlora_workspace_bytes_dropout(int64_t M, int64_t N, int64_t K, int r) {
  if (M < 1 || N < 1 || K < 64 || K % 64 != 0 || r < 1 || r > 256) return 0;
  return ws_drop_layout(dims_of(M, N, K, r)).total;
}

qlora_status qlora_lora_dropout_mask(int64_t M, int64_t K, double p, uint64_t seed, uint8_t* keep, void* stream) {
  NvtxRange nvtx_range("qlora_lora_dropout_mask");
  DropCfg c;
  if (!dropout_cfg(p, seed, &c)) return QLORA_ERR_INVALID_ARG;
  if (M < 1 || K < 64 || K % 64 != 0 || M > (int64_t(1) << 31) || K > (int64_t(1) << 31))
    return QLORA_ERR_INVALID_ARG;
  if (!keep || !aligned16(keep)) return QLORA_ERR_INVALID_ARG;
  const int64_t n = M * K;
  k_dropout_mask<<<dropout_grid(n / 4), kDropThreads, 0, static_cast<cudaStream_t>(stream)>>>(keep, n, c.seed, c.thr);
  return check_launch();
}

qlora_status qlora_linear_fwd_dropout(const void* X, int64_t M, const qlora_nf4_weight* Wq, const void* A,
                                      const void* B, int r, float alpha, double p, uint64_t seed, void* Y,
                                      float* T_save, void* workspace, size_t ws_bytes, int* d_status,
                                      const qlora_gemm_events* events, void* stream) {
  NvtxRange nvtx_range("qlora_linear_fwd_dropout");
  qlora_status st = check_linear(M, Wq, r, alpha, workspace, ws_bytes, true);
  if (st != QLORA_OK) return st;
  DropCfg drop;
  if (!dropout_cfg(p, seed, &drop)) return QLORA_ERR_INVALID_ARG;
  if (!X || !A || !B || !Y || !aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(Y))
    return QLORA_ERR_INVALID_ARG;
  if (T_save && !aligned16(T_save)) return QLORA_ERR_INVALID_ARG;
  if (!ensure_smem_attrs()) return QLORA_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const Dims d = dims_of(M, Wq->rows, Wq->cols, r);
  const Ws L = ws_layout(d);
  const WsDrop WD = ws_drop_layout(d);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const float s = alpha / static_cast<float>(r);
  float* t32 = T_save ? T_save : reinterpret_cast<float*>(ws + L.t32);
  __nv_bfloat16* sT = reinterpret_cast<__nv_bfloat16*>(ws + L.sx);
  void* Xd = ws + WD.xd;
  st = run_dropout_x(X, Xd, d, drop, cs);   // the adapter's input X * keep
  if (st != QLORA_OK) return st;
  if (M <= kDecodeMaxM)
    return run_gemv(X, A, Wq, d, t32, B, Y, s, ws, L, events, d_status, cs, Xd, drop.inv_q);
  st = clear_counters(ws, L, plans_of(d), cs);
  if (st != QLORA_OK) return st;
  st = run_T(Xd, A, d, s, ws, L, t32, sT, d_status, cs, drop.inv_q);
  if (st != QLORA_OK) return st;
  const void* Bp = padded_B(B, d, ws, L, cs, &st);
  if (st != QLORA_OK) return st;
  // the frozen path sees X undropped
  return run_fused(kModeFwd, X, Wq, nullptr, d, sT, Bp, Y, events, d_status, cs);
}

qlora_status qlora_linear_bwd_dropout(const void* dY, const void* X, int64_t M, const qlora_nf4_weight* Wq,
                                      const void* A, const void* B, int r, float alpha, double p, uint64_t seed,
                                      const float* T_saved, void* dX, void* dA, void* dB, qlora_dtype grad_dtype,
                                      void* workspace, size_t ws_bytes, int* d_status,
                                      const qlora_gemm_events* events, void* stream) {
  NvtxRange nvtx_range("qlora_linear_bwd_dropout");
  qlora_status st = check_linear(M, Wq, r, alpha, workspace, ws_bytes, true);
  if (st != QLORA_OK) return st;
  DropCfg drop;
  if (!dropout_cfg(p, seed, &drop)) return QLORA_ERR_INVALID_ARG;
  if (!dY || !X || !A || !B || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(dY) || !aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(dA) || !aligned16(dB))
    return QLORA_ERR_INVALID_ARG;
  if ((dX && !aligned16(dX)) || (T_saved && !aligned16(T_saved))) return QLORA_ERR_INVALID_ARG;
  if (grad_dtype != QLORA_F32 && grad_dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  if (!ensure_smem_attrs()) return QLORA_ERR_CUDA;
  const Dims d = dims_of(M, Wq->rows, Wq->cols, r);
  return linear_bwd_core(dY, X, d, Wq, nullptr, A, B, alpha, T_saved, dX, dA, dB, grad_dtype, workspace, d_status,
                         events, static_cast<cudaStream_t>(stream), &drop);
}

qlora_status qlora_lora_linear_fwd(const void* X, int64_t M, const void* W, int64_t N, int64_t K, const void* A,
                                   const void* B, int r, float alpha, void* Y, float* T_save, void* workspace,
                                   size_t ws_bytes, int* d_status, const qlora_gemm_events* events, void* stream) {
  NvtxRange nvtx_range("qlora_lora_linear_fwd");
  qlora_status st = check_dense(M, W, N, K, r, alpha, workspace, ws_bytes);
  if (st != QLORA_OK) return st;
  if (!X || !A || !B || !Y || !aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(Y))
    return QLORA_ERR_INVALID_ARG;
  if (T_save && !aligned16(T_save)) return QLORA_ERR_INVALID_ARG;
  if (!ensure_smem_attrs()) return QLORA_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const Dims d = dims_of(M, N, K, r);
  const Ws L = ws_layout(d);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const float s = alpha / static_cast<float>(r);
  float* t32 = T_save ? T_save : reinterpret_cast<float*>(ws + L.t32);
  __nv_bfloat16* sT = reinterpret_cast<__nv_bfloat16*>(ws + L.sx);
  st = clear_counters(ws, L, plans_of(d), cs);
  if (st != QLORA_OK) return st;
  st = run_T(X, A, d, s, ws, L, t32, sT, d_status, cs);
  if (st != QLORA_OK) return st;
  const void* Bp = padded_B(B, d, ws, L, cs, &st);
  if (st != QLORA_OK) return st;
  return run_fused(kModeFwd, X, nullptr, W, d, sT, Bp, Y, events, d_status, cs);
}

qlora_status qlora_lora_linear_bwd(const void* dY, const void* X, int64_t M, const void* W, int64_t N, int64_t K,
                                   const void* A, const void* B, int r, float alpha, const float* T_saved, void* dX,
                                   void* dA, void* dB, qlora_dtype grad_dtype, void* workspace, size_t ws_bytes,
                                   int* d_status, const qlora_gemm_events* events, void* stream) {
  NvtxRange nvtx_range("qlora_lora_linear_bwd");
  qlora_status st = check_dense(M, W, N, K, r, alpha, workspace, ws_bytes);
  if (st != QLORA_OK) return st;
  if (!dY || !X || !A || !B || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(dY) || !aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(dA) || !aligned16(dB))
    return QLORA_ERR_INVALID_ARG;
  if ((dX && !aligned16(dX)) || (T_saved && !aligned16(T_saved))) return QLORA_ERR_INVALID_ARG;
  if (grad_dtype != QLORA_F32 && grad_dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  if (!ensure_smem_attrs()) return QLORA_ERR_CUDA;
  return linear_bwd_core(dY, X, dims_of(M, N, K, r), nullptr, W, A, B, alpha, T_saved, dX, dA, dB, grad_dtype,
                         workspace, d_status, events, static_cast<cudaStream_t>(stream));
}

qlora_status qlora_adam_step(float* master, float* m, float* v, void* param_bf16, const void* grad,
                             qlora_dtype grad_dtype, int64_t n, int64_t step, float lr, float beta1, float beta2,
                             float eps, float weight_decay, float grad_scale, int* d_status, void* stream) {
  NvtxRange nvtx_range("qlora_adam_step");
  if (n < 0 || step < 1) return QLORA_ERR_INVALID_ARG;
  if (grad_dtype != QLORA_F32 && grad_dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  for (float x : {lr, beta1, beta2, eps, weight_decay, grad_scale})
    if (!std::isfinite(x)) return QLORA_ERR_INVALID_ARG;
  if (beta1 < 0.0f || beta1 >= 1.0f || beta2 < 0.0f || beta2 >= 1.0f || eps < 0.0f) return QLORA_ERR_INVALID_ARG;
  if (n == 0) return QLORA_OK;
  if (!master || !m || !v || !grad) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(master) || !aligned16(m) || !aligned16(v) || !aligned16(grad)) return QLORA_ERR_INVALID_ARG;
  if (param_bf16 && !aligned16(param_bf16)) return QLORA_ERR_INVALID_ARG;
  const double b1t = std::pow(static_cast<double>(beta1), static_cast<double>(step));
  const double b2t = std::pow(static_cast<double>(beta2), static_cast<double>(step));
  qlora::AdamArgs a{};
  a.master = master; a.m = m; a.v = v;
  a.param = static_cast<__nv_bfloat16*>(param_bf16);
  a.grad = grad;
  a.grad_bf16 = grad_dtype == QLORA_BF16 ? 1 : 0;
  a.n = n;
  a.grad_scale = grad_scale;
  a.decay = static_cast<float>(1.0 - static_cast<double>(lr) * static_cast<double>(weight_decay));
  a.beta1 = beta1;
  a.one_minus_beta1 = static_cast<float>(1.0 - static_cast<double>(beta1));
  a.beta2 = beta2;
  a.one_minus_beta2 = static_cast<float>(1.0 - static_cast<double>(beta2));
  a.eps = eps;
  a.step_size = static_cast<float>(static_cast<double>(lr) / (1.0 - b1t));
  a.rsqrt_bc2 = static_cast<float>(1.0 / std::sqrt(1.0 - b2t));
  a.status = d_status;
  const int sms = sm_count();
  if (sms <= 0) return QLORA_ERR_CUDA;
  const int64_t want = std::max<int64_t>(1, cdiv(n / 4, qlora::kAdamThreads));
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(want, static_cast<int64_t>(sms) * 8));
  qlora::k_adam_step<<<grid, qlora::kAdamThreads, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return check_launch();
}

qlora_status qlora_debug_set_wait_limit(uint64_t ns) {
  const unsigned long long v = ns ? static_cast<unsigned long long>(ns) : QLORA_WAIT_NS;
  return cudaMemcpyToSymbol(g_qlora_wait_ns, &v, sizeof(v)) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_debug_set_pair_mtiles(int n) {
  if (n < 0 || n > 2) return QLORA_ERR_INVALID_ARG;
  g_force_mtiles.store(n);
  return QLORA_OK;
}

int qlora_debug_checks_enabled(void) {
#ifdef QLORA_DEBUG_CHECKS
  return 1;
#else
  return 0;
#endif
}

qlora_status qlora_debug_range_check(unsigned int* site) {
  if (!site) return QLORA_ERR_INVALID_ARG;
  *site = 0;
  const unsigned int zero = 0;
  if (cudaMemcpyFromSymbol(site, g_qlora_range_fail, sizeof(unsigned int)) != cudaSuccess) return QLORA_ERR_CUDA;
  return cudaMemcpyToSymbol(g_qlora_range_fail, &zero, sizeof(zero)) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_debug_range_selftest(void* stream) {
  k_range_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return check_launch();
}

qlora_status qlora_debug_inject_stall(int on) {
  const int v = on ? 1 : 0;
  return cudaMemcpyToSymbol(g_qlora_inject_stall, &v, sizeof(v)) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_paged_alloc(size_t bytes, void** ptr) {
  if (!ptr) return QLORA_ERR_INVALID_ARG;
  *ptr = nullptr;
  if (bytes == 0) return QLORA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  void* p = nullptr;
  if (cudaMallocManaged(&p, bytes, cudaMemAttachGlobal) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  // resident on the GPU by preference: pages the driver evicts to the host
  // under memory pressure, or that the caller prefetches there, migrate back
  // on the GPU's next access
  if (cudaMemAdvise(p, bytes, cudaMemAdviseSetPreferredLocation, dev) != cudaSuccess) {
    cudaGetLastError();
    cudaFree(p);
    return QLORA_ERR_CUDA;
  }
  *ptr = p;
  return QLORA_OK;
}

qlora_status qlora_paged_free(void* ptr) {
  if (!ptr) return QLORA_OK;
  return cudaFree(ptr) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_paged_prefetch(void* ptr, size_t bytes, int to_device, void* stream) {
  NvtxRange nvtx_range("qlora_paged_prefetch");
  if (!ptr || bytes == 0) return QLORA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  const int dst = to_device ? dev : cudaCpuDeviceId;
  if (cudaMemPrefetchAsync(ptr, bytes, dst, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return QLORA_OK;
}

qlora_status qlora_merge_nf4(const qlora_nf4_weight* Wq, const void* A, const void* B, int r, float alpha,
                             float* W_merged, const qlora_nf4_weight* out, int* d_status, void* stream) {
  NvtxRange nvtx_range("qlora_merge_nf4");
  qlora_status st = check_weight(Wq, true);
  if (st != QLORA_OK) return st;
  st = check_weight(out, true);
  if (st != QLORA_OK) return st;
  if (out->rows != Wq->rows || out->cols != Wq->cols) return QLORA_ERR_INVALID_ARG;
  if (out->absmax_f32 && !aligned16(out->absmax_f32)) return QLORA_ERR_INVALID_ARG;
  if (r < 1 || r > 256 || !std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
  if (!A || !B || !aligned16(A) || !aligned16(B) || (W_merged && !aligned16(W_merged))) return QLORA_ERR_INVALID_ARG;
  const int64_t N = Wq->rows, K = Wq->cols;
  const float s = alpha / static_cast<float>(r);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (!W_merged) {
    // one pass: the quantiser kernel forms each merged weight itself
    if (out->codes == Wq->codes) return QLORA_ERR_INVALID_ARG;   // in place needs the two-pass form
    const int64_t nblocks = N * K / 64;
    const qlora::MergeSrc src{Wq->codes, Wq->absmax_q8, Wq->group_scale, Wq->absmax_f32, Wq->double_quant, K,
                              static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B), r, s};
    qlora::k_quantize_nf4<<<static_cast<unsigned>(cdiv(nblocks, 256)), qlora::kQuantThreads, 0, cs>>>(
        src, nblocks, out->double_quant, out->codes, out->absmax_q8, out->group_scale, out->absmax_f32, d_status);
    return check_launch();
  }
  const int64_t threads = N * (K / 8);
  qlora::k_merge_nf4<<<static_cast<unsigned>(cdiv(threads, qlora::kMergeThreads)), qlora::kMergeThreads, 0, cs>>>(
      Wq->codes, Wq->absmax_q8, Wq->group_scale, Wq->absmax_f32, Wq->double_quant, N, K,
      static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B), r, s, W_merged);
  st = check_launch();
  if (st != QLORA_OK) return st;
  return qlora_quantize_nf4(W_merged, QLORA_F32, out, d_status, stream);
}

}  // extern "C"

// ======================================================= no-allocation forward
// The forward of qlora_linear_fwd with its workspace carved from a fixed
// file-scope device array instead of a caller buffer (see qlora.h for who
// needs this).  Host code must not hand `g_noalloc_scratch` to a kernel: in
// host code that name is only a host-side stand-in.  The device address is
// looked up once per device with cudaGetSymbolAddress.
namespace {

__device__ __align__(256) uint8_t g_noalloc_scratch[QLORA_NOALLOC_SCRATCH_BYTES];

// The address is cached per device together with the id of the context it
// was looked up in: after a cudaDeviceReset the device's next primary
// context loads the module afresh and the array may sit elsewhere, so a
// changed context id triggers a new lookup.  Without the driver's context-id
// query the address is looked up on every call.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

bool current_ctx_id(unsigned long long* id) {
  static std::once_flag once;
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_cur || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};
unsigned long long g_noalloc_ctx[64] = {};

qlora_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QLORA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  unsigned long long ctx = 0;
  const bool have_id = current_ctx_id(&ctx);
  if (!have_id || !g_noalloc_ptr[dev] || g_noalloc_ctx[dev] != ctx) {
    // the lookup also makes the device's primary context current when no
    // runtime call has done so yet; the context id is read after it
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return QLORA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = current_ctx_id(&ctx) ? ctx : 0;
  }
  *out = g_noalloc_ptr[dev];
  return QLORA_OK;
}

// Forward-only carve: T partials, arrival counters, fp32 T, s*T planes,
// padded B (and the decode kernel's partial tiles and counters).
Ws noalloc_fwd_layout(const Dims& d) {
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  Ws w{};
  size_t off = 0;
  const SkPlans pl = plans_of(d);
  w.partial = w.partial2 = off; off += a256(pl.T.partial_bytes);
  w.cnt = off; off += a256(cnt_words(pl) * 4);
  w.t32 = off; off += a256(static_cast<size_t>(d.M) * d.r * 4);
  w.sx = off; off += a256(static_cast<size_t>(2 * d.M) * d.r8 * 2);
  w.ghl = w.thl = off;
  w.bpad = off; off += (d.r % 8) ? a256(static_cast<size_t>(d.N) * d.r8 * 2) : 0;
  gv_layout(d, w, off);
  w.total = off;
  return w;
}

}  // namespace

extern "C" qlora_status qlora_linear_fwd_noalloc(const void* X, int64_t M, const qlora_nf4_weight* Wq,
                                                 const void* A, const void* B, int r, float alpha, void* Y,
                                                 float* T_save, int* d_status, void* stream) {
  qlora_status st = check_weight(Wq, true);
  if (st != QLORA_OK) return st;
  if (M < 1 || M > (int64_t(1) << 31) || r < 1 || r > 256 || !std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
  if (Wq->rows % 8 != 0) return QLORA_ERR_UNSUPPORTED;
  if (!X || !A || !B || !Y || !aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(Y))
    return QLORA_ERR_INVALID_ARG;
  if (T_save && !aligned16(T_save)) return QLORA_ERR_INVALID_ARG;
  const Dims d = dims_of(M, Wq->rows, Wq->cols, r);
  const Ws L = noalloc_fwd_layout(d);
  if (L.total > QLORA_NOALLOC_SCRATCH_BYTES) return QLORA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != QLORA_OK) return st;
  if (!ensure_smem_attrs()) return QLORA_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  const float s = alpha / static_cast<float>(r);
  float* t32 = T_save ? T_save : reinterpret_cast<float*>(ws + L.t32);
  __nv_bfloat16* sT = reinterpret_cast<__nv_bfloat16*>(ws + L.sx);

  if (M <= kDecodeMaxM) return run_gemv(X, A, Wq, d, t32, B, Y, s, ws, L, nullptr, d_status, cs);
  st = clear_counters(ws, L, plans_of(d), cs);
  if (st != QLORA_OK) return st;

  st = run_T(X, A, d, s, ws, L, t32, sT, d_status, cs);
  if (st != QLORA_OK) return st;
  const void* Bp = padded_B(B, d, ws, L, cs, &st);
  if (st != QLORA_OK) return st;

  return run_fused(kModeFwd, X, Wq, nullptr, d, sT, Bp, Y, nullptr, d_status, cs);
}
