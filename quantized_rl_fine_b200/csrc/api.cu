// C ABI of libmoeq: argument validation, workspace layout, tensor maps and
// kernel launches. Built as one translation unit together with the kernel
// sources (see moeq_all.cu).
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "dequant.cuh"
#include "gemm.cuh"
#include "launchers.cuh"

// NVTX ranges around every entry point that launches work (header-only NVTX
// v3: a no-op unless a profiler has injected its tool). Compiled out with
// -DMOEQ_NVTX=0.
#ifndef MOEQ_NVTX
#define MOEQ_NVTX 1
#endif
#if MOEQ_NVTX
#include <nvtx3/nvToolsExt.h>
namespace moeq {
struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};
}  // namespace moeq
#define MOEQ_TRACE(name) const ::moeq::TraceRange moeq_trace_range_(name)
#else
#define MOEQ_TRACE(name) ((void)0)
#endif

namespace moeq {


namespace {

// --------------------------------------------------------------- test hook kernel

// One thread per (row, group): 32 elements of a row from its 16 packed bytes
// and its group scale, with the GEMM kernels' dequant functions.
template <int FMT>
__global__ void dequant_rows_kernel(const uint8_t* __restrict__ packed, const void* __restrict__ scales,
                                    int64_t R, int K, uint16_t* __restrict__ out) {
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int G = K / 32;
  if (gid >= R * G) return;
  const int64_t r = gid / G;
  const int g = static_cast<int>(gid % G);
  const uint4 pk = *reinterpret_cast<const uint4*>(packed + r * (K / 2) + g * 16);
  uint32_t sbits;
  if constexpr (FMT == MOE_W_INT4_G32_BF16) {
    sbits = static_cast<const uint16_t*>(scales)[static_cast<int64_t>(g) * R + r];
  } else {
    sbits = static_cast<const uint8_t*>(scales)[static_cast<int64_t>(g) * R + r];
  }
  uint32_t o[16];
  dequant32<FMT>(pk, sbits, o);
  uint4* dst = reinterpret_cast<uint4*>(out + r * K + g * 32);
#pragma unroll
  for (int c = 0; c < 4; ++c) dst[c] = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
}

// One thread per (listed expert, row, group): the 32 elements of one
// quantization group of one weight row, written as 64 contiguous bytes. The
// temporary-buffer scheme of the Orbit article dequantizes whole experts like
// this; the grouped GEMMs of this library never do.
template <int FMT>
__global__ void dequant_experts_kernel(const uint8_t* __restrict__ packed,
                                       const void* __restrict__ scales,
                                       const int32_t* __restrict__ experts, int count, int E, int N,
                                       int K, uint16_t* __restrict__ out) {
  grid_dependency_wait();
  grid_dependents_launch();
  const int G = K / 32;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t per_expert = static_cast<int64_t>(N) * G;
  if (gid >= per_expert * count) return;
  const int i = static_cast<int>(gid / per_expert);
  const int64_t rg = gid - i * per_expert;
  const int n = static_cast<int>(rg / G);
  const int g = static_cast<int>(rg - static_cast<int64_t>(n) * G);
  const int e = experts[i];
  uint4* dst = reinterpret_cast<uint4*>(out + (static_cast<int64_t>(i) * N + n) * K + g * 32);
  if (e < 0 || e >= E) {   // not an expert of the stack: zeros, and the error word
    if (rg == 0) raise_device_error(MOE_DEVERR_BAD_OFFSETS);
#pragma unroll
    for (int c = 0; c < 4; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const uint4 pk = *reinterpret_cast<const uint4*>(
      packed + (static_cast<int64_t>(e) * N + n) * (K / 2) + g * 16);
  const int64_t soff = (static_cast<int64_t>(e) * G + g) * N + n;
  const uint32_t sbits = (FMT == MOE_W_INT4_G32_BF16) ? static_cast<const uint16_t*>(scales)[soff]
                                                      : static_cast<const uint8_t*>(scales)[soff];
  uint32_t o[16];
  dequant32<FMT>(pk, sbits, o);
#pragma unroll
  for (int c = 0; c < 4; ++c) dst[c] = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
}

// --------------------------------------------------------------- host helpers

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D tiled tensor map: extents dims[0..2] (dims[0] contiguous), byte strides
// of dims 1 and 2, box extents box[0..2]. A 2-D map is dims[2] = 1.
bool make_map_3d(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, const uint64_t dims[3],
                 const uint64_t strides[2], const uint32_t box[3], CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  cuuint64_t st[2] = {strides[0], strides[1]};
  cuuint32_t b[3] = {box[0], box[1], box[2]};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(ptr), d, st, b, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}

int max_smem_optin() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 227 * 1024;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return 227 * 1024;
  return n;
}

// Token rows per tile from the mean rows per expert, rounded up to a multiple
// of 16 and capped at max_bn (MOEQ_BN overrides up to 256, tuning only).
int choose_bn(int64_t M, int E, int max_bn) {
  if (const char* env = getenv("MOEQ_BN")) {
    const int v = atoi(env);
    if (v >= 16 && v <= 256 && v % 16 == 0) return v;
  }
  // 1.5x the mean rows per expert, so that most experts fit one token tile
  // (their weights are streamed once); experts with more rows are split by
  // the kernel into tiles of BN rows and a shorter last one.
  const double mean = static_cast<double>(M) / std::max(1, E);
  const double want = std::max(1.0, 1.5 * mean);
  const int bn = static_cast<int>((std::min(want, static_cast<double>(max_bn)) + 15.0) / 16.0) * 16;
  return std::min(max_bn, std::max(16, bn));
}

int next_pow2(int x) {
  int p = 32;
  while (p < x) p <<= 1;
  return p;
}

moe_status check_qweight(const moe_qweight* w) {
  if (!w) return MOE_ERR_INVALID_ARG;
  if (!w->packed || !w->scales) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->packed) || !aligned16(w->scales)) return MOE_ERR_MISALIGNED;
  if (w->fmt != MOE_W_INT4_G32_BF16 && w->fmt != MOE_W_MXFP4_G32_E8M0) return MOE_ERR_INVALID_ARG;
  if (w->E < 1 || w->E > 1024 || w->N < 1 || w->K < 1) return MOE_ERR_INVALID_ARG;
  if (w->K % 64 != 0 || w->N % 64 != 0) return MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(w->E) * w->N >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_groups(const moe_groups* g, int E) {
  if (!g || !g->expert_offsets || !g->active || !g->num_active) return MOE_ERR_INVALID_ARG;
  if (g->E != E) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// Experts with more rows than this run the wide-tile forward when the layer
// is large enough to split by size (moe_grouped_qgemm_fwd).
constexpr int kWideMinRows = 192;

struct GemmPlan {
  int BN, stages, a_stages, grid, n_ftiles, acc_cols, tmem_cols, n_issuers, lanes, dq_warps;
  bool pair;    // forward on CTA pairs (M = 256 MMAs)
  bool pipes;   // two tile pipelines per CTA
  bool halves;  // forward: A stages handed over in 64-wide halves
  uint32_t stage_bytes;
  size_t smem;
};

// F: output features; tile_f: output features per tile (128, or 64 for the
// SwiGLU forward, whose tile holds 64 gate and the 64 matching up rows).
// Tensor memory (512 columns) holds n_issuers partial accumulators of
// acc_cols columns each and, in the forward kernels, the A stages (64
// columns per 128-wide fill). Token tiles are capped at 96 rows: two partials
// and four A stages fit, and the token-row box leaves room for six
// shared-memory stages (wider tiles measured slower, forward and backward).
GemmPlan plan_gemm(int mode, int64_t M, const moe_qweight* w, int F, int tile_f, int fmt) {
  GemmPlan pl;
  pl.n_ftiles = (F + tile_f - 1) / tile_f;
  // CTA pairs (forward, an even number of feature tiles): one M = 256 MMA per
  // K step of two SMs' weight tiles, and each SM loads half of the token
  // rows. Opt-in with MOEQ_PAIR=1.
  pl.pair = false;
  if (const char* env = getenv("MOEQ_PAIR")) pl.pair = (atoi(env) == 1);
  pl.pair = pl.pair && mode == kModeFwd && pl.n_ftiles % 2 == 0;
  // A pair's CTAs hold half of the token rows each, so its tiles may be twice
  // as wide for the same shared memory per stage. The backward kernels take
  // 192-row tiles once the mean expert holds 128 rows or more: an expert's
  // weights are then dequantized for half as many token tiles, which pays for
  // the shallower ring (measured at 341 rows per expert: -12 % and -21 % on
  // the two backward GEMMs; at 85 rows wider tiles only cost stages).
  // Wide tiles: up to 384 rows (MOEQ_WIDE_BN caps them lower, tuning).
  int wide_cap = 2 * kWideHalfRows;
  if (const char* env = getenv("MOEQ_WIDE_BN")) {
    const int v = atoi(env);
    if (v >= 16 && v <= 2 * kWideHalfRows && v % 16 == 0) wide_cap = v;
  }
  pl.BN = choose_bn(M, w->E, pl.pair ? 192 : (mode == kModeFwdW ? wide_cap : 96));
  if (mode == kModeFwdW) pl.BN = std::min(pl.BN, wide_cap);
  if (mode == kModeBwd && !getenv("MOEQ_BN") && M >= 128 * static_cast<int64_t>(w->E))
    pl.BN = 192;
  if (pl.pair) pl.BN = (pl.BN + 31) / 32 * 32;   // pair MMAs take N in steps of 32
  pl.acc_cols = (pl.BN + 31) / 32 * 32;
  pl.stage_bytes = gemm_stage_bytes(mode, pl.BN, fmt, pl.pair);
  // MOEQ_NI caps the number of MMA-issuing warps (tuning only).
  int ni_max = kMaxIssuers;
  if (const char* env = getenv("MOEQ_NI")) {
    const int v = atoi(env);
    if (v >= 1 && v <= kMaxIssuers) ni_max = v;
  }
  // Pipeline lanes: four (one dequant warp per lane quarter, 128 elements per
  // thread and fill) while a token tile of at most 64 rows leaves room for a
  // ring of eight or more stages; two (two warps per quarter) for wider tiles,
  // whose stages would otherwise be too few. MOEQ_LANES overrides (tuning).
  pl.lanes = pl.BN <= 64 ? 4 : 2;
  if (const char* env = getenv("MOEQ_LANES")) {
    const int v = atoi(env);
    if (v == 2 || v == 4) pl.lanes = v;
  }
  // Dequant warps: sixteen; eight (one per lane quarter and lane, a whole
  // 128-wide fill per thread) with two lanes when MOEQ_DQW=8 (tuning).
  pl.dq_warps = 16;
  if (const char* env = getenv("MOEQ_DQW")) {
    if (atoi(env) == 8 && pl.lanes == 2 && !pl.pair) pl.dq_warps = 8;
  }
  const int L = pl.lanes;
  // Every ring has a multiple of L stages, and of n_issuers where the issuers
  // wait on it (the A ring), so that each stage has one waiter per role.
  auto ring_step = [L](int ni) {
    int a = L, b = ni;
    while (b) { const int t = a % b; a = b; b = t; }
    return L / a * ni;
  };
  // As many shared-memory fills as fit (at most 16): a deep ring hides the
  // latency of the weight stream.
  const int avail = max_smem_optin();
  auto fits = [&](int s, int sa) {
    return static_cast<int>(s * pl.stage_bytes + gemm_fixed_smem_bytes(mode, s, sa, w->E)) <= avail;
  };
  if (mode == kModeFwdW) {
    // Wide token tiles: A stages of 32 columns (64-wide fills), a multiple of
    // the two lanes, next to one accumulator of up to 384 columns, or to two
    // (two issuers, two tile pipelines) while two accumulators and four A
    // stages fit (tiles of at most 192 rows).
    pl.lanes = 2;
    pl.dq_warps = 16;
    pl.n_issuers = (2 * pl.acc_cols + 4 * 32 <= 512) ? 2 : 1;
    pl.halves = false;
    pl.a_stages = std::min(8, (512 - pl.n_issuers * pl.acc_cols) / 32 / 2 * 2);
    pl.tmem_cols = 512;
    int stages = 16;
    while (stages > 2 && !fits(stages, pl.a_stages)) stages -= 2;
    pl.stages = stages;
  } else if (mode != kModeBwd) {
    // A stage of a 128-wide fill: 64 tensor-memory columns. The most issuers
    // that still leave four A stages; with two issuers and wide accumulators
    // (more than 128 columns each) two A stages, handed over in halves, so
    // that a pipeline's next fill is dequantized while its previous fill's
    // second half is multiplied (forward only). MOEQ_HALVES=0/1 overrides
    // (tuning).
    int halves_env = -1;
    if (const char* env = getenv("MOEQ_HALVES")) halves_env = atoi(env) != 0 ? 1 : 0;
    bool pipes_allowed = true;
    if (const char* env = getenv("MOEQ_PIPES")) pipes_allowed = (atoi(env) != 0);
    pl.n_issuers = 1;
    pl.a_stages = 4;
    pl.halves = false;
    for (int ni = ni_max; ni >= 1; --ni) {
      const int step = ring_step(ni);
      const int room = (512 - ni * pl.acc_cols) / 64;
      const int sa = std::min(8, room / step * step);
      if (sa >= 4) {
        pl.n_issuers = ni;
        pl.a_stages = sa;
        pl.halves = halves_env == 1 && mode == kModeFwd;
        break;
      }
      if (mode == kModeFwd && ni == 2 && sa >= 2 && halves_env != 0 && pipes_allowed) {
        pl.n_issuers = ni;
        pl.a_stages = sa;
        pl.halves = true;
        break;
      }
    }
    pl.tmem_cols = 512;
    // MOEQ_STAGES caps the shared-memory ring (tuning only).
    int stages = 16;
    if (const char* env = getenv("MOEQ_STAGES")) {
      const int v = atoi(env);
      if (v >= L && v <= 16 && v % L == 0) stages = v;
    }
    while (stages > L && !fits(stages, pl.a_stages)) stages -= L;
    pl.stages = stages;
  } else {
    pl.halves = false;
    int stages = 16;
    while (stages > L && !fits(stages, stages)) stages -= L;
    pl.stages = stages;
    pl.a_stages = stages;
    pl.n_issuers = 1;
    for (int ni = ni_max; ni >= 1; --ni) {
      if (ni * pl.acc_cols <= 512 && stages % ring_step(ni) == 0) { pl.n_issuers = ni; break; }
    }
    pl.tmem_cols = next_pow2(pl.n_issuers * pl.acc_cols);
  }
  // Two tile pipelines (each issuer accumulates whole tiles, so one tile's
  // epilogue overlaps the other's MMAs) need two lanes and two issuers.
  // Measured against every issuer taking every other fill: forward -0.6 %
  // (C2) to -9 % (an MXFP4 shape at 256 rows per expert), backward -5 % to
  // -19 % (the SwiGLU backward epilogue is the heaviest); no shape slower.
  // MOEQ_PIPES=0 turns them off (tuning only).
  pl.pipes = true;
  if (const char* env = getenv("MOEQ_PIPES")) pl.pipes = (atoi(env) != 0);
  pl.pipes = pl.pipes && pl.n_issuers == 2;
  const int stages = pl.stages;
  pl.smem = stages * pl.stage_bytes + gemm_fixed_smem_bytes(mode, stages, pl.a_stages, w->E);
  const int64_t bound = static_cast<int64_t>(pl.pair ? pl.n_ftiles / 2 : pl.n_ftiles) *
                        (std::min<int64_t>(w->E, M) + (M + pl.BN - 1) / pl.BN);
  if (pl.pair)   // CTAs, two per pair tile; the launch clamps to the resident pairs
    pl.grid = 2 * static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(num_sms() / 2, bound)));
  else
    pl.grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(num_sms(), bound)));
  return pl;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Workspace convention: ws == NULL with ws_bytes != NULL is a size query
// (writes *ws_bytes). ws == NULL with ws_bytes == NULL runs without a
// workspace, which is valid only when the call needs none. Otherwise
// *ws_bytes must cover `need` and ws must be 256-byte aligned.
moe_status check_workspace(void* ws, size_t* ws_bytes, size_t need) {
  if (!ws) {
    if (ws_bytes) {
      *ws_bytes = need;
      return MOE_OK;
    }
    return need == 0 ? MOE_OK : MOE_ERR_WORKSPACE;
  }
  if (!ws_bytes || *ws_bytes < need) return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_MISALIGNED;
  return MOE_OK;
}

// Runs one grouped GEMM launch over the rows of `bmat` (a, a' or dout).
moe_status run_gemm(int mode, int epi, const void* bmat, int64_t M, const moe_qweight* w,
                    const moe_groups* g, void* out, int64_t ldo, void* saved, const GemmPlan& pl,
                    cudaStream_t s, const int32_t* b_rows = nullptr, int32_t m_lo = 0,
                    int32_t m_hi = 0x7fffffff) {
  const bool fwd = gemm_is_fwd(mode);
  const int F = fwd ? (epi == MOE_EPI_SWIGLU ? w->N / 2 : w->N) : w->K;
  const int R = fwd ? w->K : w->N;
  const uint32_t fill = (mode == kModeFwd || mode == kModeBwdT) ? 128 : 64;   // reduction per fill
  CUtensorMap tb, tw, ts;
  const bool int4 = w->fmt == MOE_W_INT4_G32_BF16;
  const uint64_t esz = int4 ? 2 : 1;
  const CUtensorMapDataType sdt = int4 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const uint64_t E = w->E, N = w->N, K = w->K;
  const uint32_t chunks = fill / 64;                        // 64-element K chunks per fill
  {  // token rows: [M][R] BF16 viewed as (64, M, R/64) -> smem [chunk][BN rows][64]
     // (wide tiles: two boxes of kWideHalfRows rows)
    const uint64_t dims[3] = {64, static_cast<uint64_t>(M), static_cast<uint64_t>(R) / 64};
    const uint64_t strides[2] = {static_cast<uint64_t>(R) * 2, 128};
    const uint32_t rows = (mode == kModeFwdW) ? kWideHalfRows : (pl.pair ? pl.BN / 2 : pl.BN);
    const uint32_t box[3] = {64, rows, chunks};
    if (!make_map_3d(&tb, bmat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return MOE_ERR_CUDA;
  }
  // Forward packed rows: fill / 2 bytes a row, 64-byte or 32-byte swizzle.
  const CUtensorMapSwizzle wsw = (fill == 128) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  if (fwd && epi == MOE_EPI_SWIGLU) {
    // packed [E][N][K/2] as [2E][N/2][K/2]: one box brings 64 gate and the 64 up rows
    const uint64_t wd[3] = {K / 2, N / 2, 2 * E};
    const uint64_t ws[2] = {K / 2, (N / 2) * (K / 2)};
    const uint32_t wb[3] = {fill / 2, 64, 2};
    // scales [E][K/32][N] as [E*K/32][2][N/2] -> smem [groups][2 halves][64]
    const uint64_t sd[3] = {N / 2, 2, E * (K / 32)};
    const uint64_t ss[2] = {(N / 2) * esz, N * esz};
    const uint32_t sb[3] = {64, 2, fill / 32};
    if (!make_map_3d(&tw, w->packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, wd, ws, wb, wsw) ||
        !make_map_3d(&ts, w->scales, sdt, sd, ss, sb, CU_TENSOR_MAP_SWIZZLE_NONE))
      return MOE_ERR_CUDA;
  } else if (fwd) {
    const uint64_t wd[3] = {K / 2, E * N, 1};
    const uint64_t ws[2] = {K / 2, E * N * (K / 2)};
    const uint32_t wb[3] = {fill / 2, 128, 1};
    const uint64_t sd[3] = {N, E * (K / 32), 1};
    const uint64_t ss[2] = {N * esz, E * (K / 32) * N * esz};
    const uint32_t sb[3] = {128, fill / 32, 1};
    if (!make_map_3d(&tw, w->packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, wd, ws, wb, wsw) ||
        !make_map_3d(&ts, w->scales, sdt, sd, ss, sb, CU_TENSOR_MAP_SWIZZLE_NONE))
      return MOE_ERR_CUDA;
  } else {
    // backward: one box is the fill's reduction rows n (64, or 128 with A in
    // tensor memory) x the tile's 128 features (64 B); scales [4 groups][rows]
    const uint64_t wd[3] = {K / 2, E * N, 1};
    const uint64_t ws[2] = {K / 2, E * N * (K / 2)};
    const uint32_t wb[3] = {64, fill, 1};
    const uint64_t sd[3] = {N, E * (K / 32), 1};
    const uint64_t ss[2] = {N * esz, E * (K / 32) * N * esz};
    const uint32_t sb[3] = {fill, 4, 1};
    if (!make_map_3d(&tw, w->packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, wd, ws, wb,
                     CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map_3d(&ts, w->scales, sdt, sd, ss, sb, CU_TENSOR_MAP_SWIZZLE_NONE))
      return MOE_ERR_CUDA;
  }
  GemmArgs p;
  p.offsets = g->expert_offsets;
  p.active = g->active;
  p.num_active = g->num_active;
  p.E = w->E;
  p.N = w->N;
  p.K = w->K;
  p.M = static_cast<int32_t>(M);
  p.BN = pl.BN;
  p.n_ftiles = pl.pair ? pl.n_ftiles / 2 : pl.n_ftiles;
  p.n_issuers = pl.n_issuers;
  p.acc_cols = pl.acc_cols;
  p.tmem_cols = pl.tmem_cols;
  p.F = F;
  p.R = R;
  p.stages = pl.stages;
  p.a_stages = pl.a_stages;
  p.stage_bytes = pl.stage_bytes;
  p.pipes = pl.pipes ? 1 : 0;
  p.a_halves = pl.halves ? 1 : 0;
  // Token tiles of an expert: equal widths; MOEQ_SPLIT=bn gives BN-row tiles
  // and a shorter last one (fewer padding rows, measured no faster; tuning).
  p.split_even = 1;
  if (const char* env = getenv("MOEQ_SPLIT")) p.split_even = (strcmp(env, "bn") == 0) ? 0 : 1;
  p.m_lo = m_lo;
  p.m_hi = m_hi;
  // Gathered rows: the token-row tensor map above is encoded (over the same
  // base) but not read; the producers copy row b_rows[p] of bmat instead.
  p.b_rows = b_rows;
  p.b_src = static_cast<const __nv_bfloat16*>(bmat);
  if (b_rows && pl.stages < 4) return MOE_ERR_UNSUPPORTED;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.ldo = ldo;
  p.saved = static_cast<__nv_bfloat16*>(saved);
  return cuda_status(launch_grouped_qgemm(mode, w->fmt, epi, pl.lanes, pl.dq_warps, pl.pair, tb, tw,
                                          ts, p, pl.grid, pl.smem, s));
}

}  // namespace
}  // namespace moeq

using namespace moeq;

extern "C" {

int32_t moe_abi_version(void) { return MOEQ_ABI_VERSION; }

int32_t moe_nvtx_enabled(void) { return MOEQ_NVTX ? 1 : 0; }

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_MISALIGNED: return "MOE_ERR_MISALIGNED";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
    default: return "MOE_ERR_UNKNOWN";
  }
}

moe_status moe_route_permute(const float* logits, const void* x, int64_t T, int32_t E, int32_t k,
                             int64_t d, int32_t chunk_size, int32_t* topk_idx, float* gates,
                             int32_t* expert_offsets, int32_t* active, int32_t* num_active,
                             int32_t* chunk_offsets, int32_t* num_chunks, int32_t* perm_token,
                             int32_t* inv_perm, void* x_perm, void* ws, size_t* ws_bytes,
                             void* stream) {
  MOEQ_TRACE("moe_route_permute");
  if (T < 1 || E < 1 || E > 1024 || k < 1 || k > 32 || k > E || chunk_size < 1)
    return MOE_ERR_INVALID_ARG;
  if (T * k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  // Launches that take the single-pass tail need no scratch (size 0); larger
  // ones keep per-block expert histograms in the workspace.
  const size_t need = route_single_pass(T, E)
                          ? 0
                          : align_up(static_cast<size_t>(route_num_blocks(T)) * E * sizeof(int32_t), 256);
  moe_status st = check_workspace(ws, ws_bytes, need);
  if (st != MOE_OK) return st;
  if (!ws && ws_bytes) return MOE_OK;   // size query
  const void* ptrs[] = {logits, topk_idx, gates, expert_offsets, active, num_active,
                        chunk_offsets, num_chunks, perm_token, inv_perm};
  for (const void* p : ptrs) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  }
  if (x) {
    if (!x_perm || d < 8 || d % 8 != 0) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_MISALIGNED;
  }
  return cuda_status(launch_route(logits, x, static_cast<int>(T), E, k, d, chunk_size, topk_idx,
                                  gates, expert_offsets, active, num_active, chunk_offsets,
                                  num_chunks, perm_token, inv_perm, x ? x_perm : nullptr,
                                  static_cast<int32_t*>(ws), static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Routing without a caller-supplied workspace.
//
// Some callers cannot hand this library any scratch memory: a serving runtime
// that reserves all of HBM in one arena at start-up and forbids device
// allocation afterwards, code that enqueues work while a CUDA graph is being
// captured (cudaMalloc is not capturable), or a plain C host that has no
// caching allocator and would otherwise pay a device-wide synchronization for
// each cudaMalloc/cudaFree pair. For them the per-block expert histograms of
// the routing kernels live in the fixed array below, which every GPU that
// loads the library keeps for the life of the process.
// ---------------------------------------------------------------------------

namespace {

constexpr int64_t kRouteStaticScratchInts = int64_t(1) << 20;   // 4 MiB of int32 per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) int32_t g_route_static_scratch[kRouteStaticScratchInts];

std::mutex g_static_scratch_mutex;
int32_t* g_static_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_route_static_scratch on the current device. In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
moe_status static_scratch_on_current_device(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
  if (!g_static_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_static_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    // The routing kernels' own one-time setup on this device, done here too,
    // so that after the first call no later call does any setup.
    if (route_prepare_device(nullptr) != cudaSuccess) return MOE_ERR_CUDA;
    g_static_scratch_addr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_static_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_route_permute_noalloc(const float* logits, const void* x, int64_t T, int32_t E,
                                     int32_t k, int64_t d, int32_t chunk_size, int32_t* topk_idx,
                                     float* gates, int32_t* expert_offsets, int32_t* active,
                                     int32_t* num_active, int32_t* chunk_offsets,
                                     int32_t* num_chunks, int32_t* perm_token, int32_t* inv_perm,
                                     void* x_perm, void* stream) {
  MOEQ_TRACE("moe_route_permute_noalloc");
  if (T < 1 || E < 1 || E > 1024 || k < 1 || k > 32 || k > E || chunk_size < 1)
    return MOE_ERR_INVALID_ARG;
  if (T * k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  const int64_t nblk = route_num_blocks(T);
  if (nblk * E > kRouteStaticScratchInts) return MOE_ERR_WORKSPACE;   // beyond the fixed array
  const void* ptrs[] = {logits, topk_idx, gates, expert_offsets, active, num_active,
                        chunk_offsets, num_chunks, perm_token, inv_perm};
  for (const void* p : ptrs) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  }
  if (x) {
    if (!x_perm || d < 8 || d % 8 != 0) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_MISALIGNED;
  }
  int32_t* scratch = nullptr;
  moe_status st = static_scratch_on_current_device(&scratch);
  if (st != MOE_OK) return st;
  // The histogram kernel writes every entry the later kernels of this call
  // read, so the array's leftover contents from an earlier call never matter.
  return cuda_status(launch_route(logits, x, static_cast<int>(T), E, k, d, chunk_size, topk_idx,
                                  gates, expert_offsets, active, num_active, chunk_offsets,
                                  num_chunks, perm_token, inv_perm, x ? x_perm : nullptr, scratch,
                                  static_cast<cudaStream_t>(stream)));
}

moe_status moe_grouped_qgemm_fwd(const void* a, const int32_t* a_rows, int64_t M,
                                 const moe_qweight* w, const moe_groups* g, const void* adapter,
                                 int32_t epi, void* out, void* saved_gu, void* ws,
                                 size_t* ws_bytes, void* stream) {
  MOEQ_TRACE("moe_grouped_qgemm_fwd");
  moe_status st = check_qweight(w);
  if (st != MOE_OK) return st;
  if (M < 1 || M >= (int64_t(1) << 31)) return MOE_ERR_INVALID_ARG;
  if (epi != MOE_EPI_NONE && epi != MOE_EPI_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (epi == MOE_EPI_SWIGLU && w->N % 128 != 0) return MOE_ERR_UNSUPPORTED;
  const int F = (epi == MOE_EPI_SWIGLU) ? w->N / 2 : w->N;
  // Experts with more than kWideMinRows rows run the wide-tile kernel (token
  // tiles of up to 384 rows, so each weight is dequantized once per 384 rows
  // of an expert instead of once per 96), the rest the narrow one: two
  // launches over the same active list, each taking one size class, once the
  // mean expert holds more than 96 rows (below that few experts are that
  // large, and the extra launch would cost more than it saves). MOEQ_WIDE=0
  // keeps every expert narrow, MOEQ_WIDE=1 makes every expert wide (tuning).
  // Not with gathered rows or CTA pairs.
  int wide_mode = (M > 96 * static_cast<int64_t>(w->E)) ? 2 : 0;   // 0 narrow, 1 wide, 2 both
  if (const char* env = getenv("MOEQ_WIDE")) wide_mode = (atoi(env) == 1) ? 1 : 0;
  if (const char* env = getenv("MOEQ_PAIR")) if (atoi(env) == 1) wide_mode = 0;
  if (a_rows && !adapter) wide_mode = 0;   // the wide kernel reads its rows by tensor map only
  const int tile_f = epi == MOE_EPI_SWIGLU ? 64 : 128;
  const GemmPlan pl = plan_gemm(wide_mode == 1 ? kModeFwdW : kModeFwd, M, w, F, tile_f, w->fmt);
  const GemmPlan plw = (wide_mode == 2) ? plan_gemm(kModeFwdW, M, w, F, tile_f, w->fmt) : pl;
  const size_t need = adapter ? align_up(static_cast<size_t>(M) * w->K * 2, 256) : 0;
  if ((st = check_workspace(ws, ws_bytes, need)) != MOE_OK) return st;
  if (!ws && ws_bytes) return MOE_OK;   // size query
  if ((st = check_groups(g, w->E)) != MOE_OK) return st;
  if (!a || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(out) || (saved_gu && !aligned16(saved_gu)) ||
      (adapter && !aligned16(adapter)) || (a_rows && !aligned16(a_rows)))
    return MOE_ERR_MISALIGNED;
  if (saved_gu && epi != MOE_EPI_SWIGLU) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (adapter) {
    // The adapter kernel gathers the rows (a_rows) and writes a' in expert
    // order; the GEMM then reads a' through its tensor map.
    void* xa = ws;
    cudaError_t e = launch_adapter_apply(a, a_rows, adapter, g->expert_offsets, w->E,
                                         static_cast<int>(M), w->K, xa, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    a = xa;
  }
  const int32_t* rows = adapter ? nullptr : a_rows;
  if (wide_mode == 2) {
    // MOEQ_WIDE_MIN moves the size-class cut (tuning).
    int cut = kWideMinRows;
    if (const char* env = getenv("MOEQ_WIDE_MIN")) {
      const int v = atoi(env);
      if (v >= 16 && v <= 2 * kWideHalfRows) cut = v;
    }
    st = run_gemm(kModeFwd, epi, a, M, w, g, out, F, saved_gu, pl, s, rows, 0, cut);
    if (st != MOE_OK) return st;
    return run_gemm(kModeFwdW, epi, a, M, w, g, out, F, saved_gu, plw, s, rows, cut + 1);
  }
  return run_gemm(wide_mode == 1 ? kModeFwdW : kModeFwd, epi, a, M, w, g, out, F, saved_gu, pl, s,
                  rows);
}

moe_status moe_grouped_qgemm_bwd_dx(const void* dout, int64_t M, const moe_qweight* w,
                                    const moe_groups* g, int32_t epi, const void* saved_gu,
                                    const void* adapter, const void* a, const int32_t* a_rows,
                                    void* din, float* d_adapter, void* ws, size_t* ws_bytes,
                                    void* stream) {
  MOEQ_TRACE("moe_grouped_qgemm_bwd_dx");
  moe_status st = check_qweight(w);
  if (st != MOE_OK) return st;
  if (M < 1 || M >= (int64_t(1) << 31)) return MOE_ERR_INVALID_ARG;
  if (epi != MOE_EPI_NONE && epi != MOE_EPI_SWIGLU_BWD) return MOE_ERR_INVALID_ARG;
  const bool with_adapter = adapter != nullptr;
  if (with_adapter && (epi != MOE_EPI_NONE || !a || !d_adapter)) return MOE_ERR_INVALID_ARG;
  if (!with_adapter && (a || a_rows || d_adapter)) return MOE_ERR_INVALID_ARG;
  if (epi == MOE_EPI_SWIGLU_BWD && !saved_gu) return MOE_ERR_INVALID_ARG;
  // A in tensor memory (128-wide fills, the dequantized rows transposed on
  // the way) unless MOEQ_BWD_SMEM_A=1 asks for the shared-memory form (tuning).
  int bmode = kModeBwdT;
  if (const char* env = getenv("MOEQ_BWD_SMEM_A")) bmode = (atoi(env) == 1) ? kModeBwd : kModeBwdT;
  const GemmPlan pl = plan_gemm(bmode, M, w, w->K, 128, w->fmt);
  const size_t need = with_adapter ? align_up(static_cast<size_t>(M) * w->K * 2, 256) : 0;
  if ((st = check_workspace(ws, ws_bytes, need)) != MOE_OK) return st;
  if (!ws && ws_bytes) return MOE_OK;   // size query
  if ((st = check_groups(g, w->E)) != MOE_OK) return st;
  if (!dout || !din) return MOE_ERR_INVALID_ARG;
  if (!aligned16(dout) || !aligned16(din) || (saved_gu && !aligned16(saved_gu)) ||
      (adapter && !aligned16(adapter)) || (a && !aligned16(a)) ||
      (a_rows && !aligned16(a_rows)) || (d_adapter && !aligned16(d_adapter)))
    return MOE_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (epi == MOE_EPI_SWIGLU_BWD) {
    return run_gemm(bmode, epi, dout, M, w, g, din, 2 * static_cast<int64_t>(w->K),
                    const_cast<void*>(saved_gu), pl, s);
  }
  if (!with_adapter) {
    return run_gemm(bmode, epi, dout, M, w, g, din, w->K, nullptr, pl, s);
  }
  void* dxa = ws;
  st = run_gemm(bmode, epi, dout, M, w, g, dxa, w->K, nullptr, pl, s);
  if (st != MOE_OK) return st;
  return cuda_status(launch_adapter_bwd(a, a_rows, dxa, adapter, g->expert_offsets, w->E, w->K,
                                        din, d_adapter, s));
}

moe_status moe_unpermute_combine(const void* rows, const int32_t* inv_perm, const float* gates,
                                 int64_t T, int32_t k, int64_t D, void* out, int32_t mode,
                                 void* stream) {
  MOEQ_TRACE("moe_unpermute_combine");
  if (!rows || !inv_perm || !out) return MOE_ERR_INVALID_ARG;
  if (T < 1 || k < 1 || k > 32 || D < 8 || D % 8 != 0 || (mode != 0 && mode != 1))
    return MOE_ERR_INVALID_ARG;
  if (T * k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(rows) || !aligned16(inv_perm) || !aligned16(out) || (gates && !aligned16(gates)))
    return MOE_ERR_MISALIGNED;
  return cuda_status(launch_combine(rows, inv_perm, gates, static_cast<int>(T), k, D, out, mode,
                                    static_cast<cudaStream_t>(stream)));
}

moe_status moe_get_device_error(int32_t* code, void* stream) {
  if (!code) return MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return MOE_ERR_CUDA;
  const int32_t zero = 0;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return MOE_ERR_CUDA;
  *code = v;
  return MOE_OK;
}

moe_status moe_test_dequant(const void* packed, const void* scales, int64_t R, int32_t K,
                            int32_t fmt, void* out, void* stream) {
  if (!packed || !scales || !out || R < 1 || K < 64 || K % 64 != 0) return MOE_ERR_INVALID_ARG;
  if (fmt != MOE_W_INT4_G32_BF16 && fmt != MOE_W_MXFP4_G32_E8M0) return MOE_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(scales) || !aligned16(out)) return MOE_ERR_MISALIGNED;
  return cuda_status(launch_dequant_rows(packed, scales, R, K, fmt, out,
                                         static_cast<cudaStream_t>(stream)));
}

moe_status moe_dequant_experts(const moe_qweight* w, const int32_t* experts, int32_t count,
                               void* out, void* stream) {
  MOEQ_TRACE("moe_dequant_experts");
  moe_status st = check_qweight(w);
  if (st != MOE_OK) return st;
  if (!experts || !out || count < 0) return MOE_ERR_INVALID_ARG;
  if (!aligned16(experts) || !aligned16(out)) return MOE_ERR_MISALIGNED;
  if (count == 0) return MOE_OK;
  const int64_t n = static_cast<int64_t>(count) * w->N * (w->K / 32);
  const int threads = 256;
  const int64_t blocks = (n + threads - 1) / threads;
  if (blocks >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint8_t* packed = static_cast<const uint8_t*>(w->packed);
  uint16_t* o = static_cast<uint16_t*>(out);
  cudaError_t e;
  if (w->fmt == MOE_W_INT4_G32_BF16)
    e = launch_pdl(dequant_experts_kernel<MOE_W_INT4_G32_BF16>, dim3(static_cast<unsigned>(blocks)),
                   dim3(threads), 0, s, packed, w->scales, experts, count, w->E, w->N, w->K, o);
  else
    e = launch_pdl(dequant_experts_kernel<MOE_W_MXFP4_G32_E8M0>, dim3(static_cast<unsigned>(blocks)),
                   dim3(threads), 0, s, packed, w->scales, experts, count, w->E, w->N, w->K, o);
  return cuda_status(e);
}

moe_status moe_ep_regroup(const int32_t* counts, int32_t W, int32_t E_loc, int64_t R,
                          const void* rows_in, void* rows_out, int64_t D, int32_t direction,
                          int32_t chunk_size, int32_t* expert_offsets, int32_t* active,
                          int32_t* num_active, int32_t* chunk_offsets, int32_t* num_chunks,
                          void* stream) {
  MOEQ_TRACE("moe_ep_regroup");
  if (!counts || W < 1 || E_loc < 1 || static_cast<int64_t>(W) * E_loc > ep_max_entries())
    return MOE_ERR_INVALID_ARG;
  if (R < 0 || R >= (int64_t(1) << 31) || D < 8 || D % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (direction != 0 && direction != 1) return MOE_ERR_INVALID_ARG;
  if (R > 0 && (!rows_in || !rows_out)) return MOE_ERR_INVALID_ARG;
  if (direction == 0 && (chunk_size < 1 || !expert_offsets || !active || !num_active ||
                         !chunk_offsets || !num_chunks))
    return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {counts, rows_in, rows_out, expert_offsets, active, num_active,
                        chunk_offsets, num_chunks};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  return cuda_status(launch_ep_regroup(counts, W, E_loc, static_cast<int>(R), rows_in, rows_out, D,
                                       direction, chunk_size, expert_offsets, active, num_active,
                                       chunk_offsets, num_chunks, num_sms(),
                                       static_cast<cudaStream_t>(stream)));
}

moe_status moe_test_set_wait_budget(int64_t cycles) {
  const long long v = cycles > 0 ? static_cast<long long>(cycles) : kDefaultWaitBudget;
  return cuda_status(cudaMemcpyToSymbol(g_wait_budget, &v, sizeof(v)));
}

}  // extern "C"

namespace moeq {

cudaError_t launch_dequant_rows(const void* packed, const void* scales, int64_t R, int K, int fmt,
                                void* out, cudaStream_t s) {
  const int64_t n = R * (K / 32);
  const int threads = 256;
  const int64_t blocks = (n + threads - 1) / threads;
  if (fmt == MOE_W_INT4_G32_BF16)
    dequant_rows_kernel<MOE_W_INT4_G32_BF16><<<static_cast<unsigned>(blocks), threads, 0, s>>>(
        static_cast<const uint8_t*>(packed), scales, R, K, static_cast<uint16_t*>(out));
  else
    dequant_rows_kernel<MOE_W_MXFP4_G32_E8M0><<<static_cast<unsigned>(blocks), threads, 0, s>>>(
        static_cast<const uint8_t*>(packed), scales, R, K, static_cast<uint16_t*>(out));
  return cudaGetLastError();
}

}  // namespace moeq
