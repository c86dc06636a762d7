// Grouped low-bit GEMM over the active experts (forward and dX backward).
//
// Orbit article, "Active-expert-chunked dequantization": the experts chosen
// by the router are taken in fixed-size chunks, their 4-bit weights are
// dequantized and a grouped GEMM runs over them. Here the dequantization
// happens inside the GEMM kernel, tile by tile, into tensor memory (forward)
// or shared memory (backward); no BF16 weight is ever written to global
// memory. The DeepSeek-V4 paragraph of the
// same section gives the backward form: only the activation gradient is
// formed, the frozen base gets none.
//
// One persistent CTA per SM walks a device-built tile list (active experts in
// ascending id, which is chunk order; inside an expert, feature tile major and
// token tile minor). A tile is 128 output features x BN token rows (BN a
// multiple of 16), accumulated in FP32 in tensor memory by tcgen05.mma with
// the dequantized weight as operand A (M = 128) and the token rows as operand
// B (N = BN):
//
//   forward  D[f, t] = sum_k W[e][f][k] * a[t][k]     (A K-major, in tensor memory)
//   backward D[f, t] = sum_n W[e][n][f] * dout[t][n]  (A K-major in tensor memory, the
//                                                      dequantized rows transposed on
//                                                      the way; or MN-major in shared
//                                                      memory)
//
// The reduction is walked in fills of 128 (A in tensor memory) or 64 (A in
// shared memory) elements. Fill f of the CTA belongs to pipeline lane f % kLanes, whose
// dequant group (four or eight warps covering the four tensor-memory lane
// quarters) turns its packed codes into BF16 in registers and then into the A
// stage; producer warp f % kProdWarps issues its copies (token rows, packed
// weights, group scales) into a shared-memory stage, and MMA-issuing warp
// f % n_issuers accumulates it into that issuer's partial accumulator. One
// issuing thread sustains only about one tcgen05.mma per 70-200 cycles, so
// splitting the reduction across issuers is what keeps the tensor core fed at
// small N. An epilogue warpgroup sums the partials in issuer order and writes
// BF16 (plain, SwiGLU with the saved gate/up, or the SwiGLU backward).
//
// The PAIR instantiations (forward, opt-in) run clusters of two CTAs on 256
// output features with M = 256 MMAs issued by the even CTA; each CTA holds
// its own weight rows and half of the token rows.
// Every wait is bounded; on a timeout the kernel records a device error,
// lets its in-flight copies and MMAs finish (again bounded), frees tensor
// memory and returns.
#include <algorithm>

#include "common.cuh"
#include "dequant.cuh"
#include "gemm.cuh"

namespace moeq {

namespace {

// 24 warps (16 dequant warps): six on each of the four SM sub-partitions, so
// 80 registers a thread; 16 warps (8 dequant warps): 128 registers a thread.
static_assert(gemm_threads(16) <= 1024 && ((gemm_threads(16) / 32 + 3) / 4) * 32 * 80 <= 16384,
              "roles must fit 80 registers a thread");
constexpr int kTileF = 128;            // output features per tile (MMA M)
constexpr uint32_t kABytes = kTileF * 64 * 2;   // 16 KiB dequantized A tile (backward fill)
constexpr uint32_t kStageBytesEpi = 2048;       // epilogue staging block per warp
constexpr uint32_t kScratchBytes = 1024;        // kModeBwdT transpose scratch per dequant warp
constexpr int kWideHalf = kWideHalfRows;        // kModeFwdW: token rows of a tile's first MMA

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

// A wait used only while shutting down: bounded, ignores the abort flag.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const long long budget = kDefaultWaitBudget;
  const long long t0 = clock64();
  while (!mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) {
    if (clock64() - t0 > budget) {
      raise_device_error(MOE_DEVERR_WAIT_TIMEOUT);
      return;
    }
  }
}

struct Tile {
  int e, ft, row0, row_end;
  int width;  // token rows of the tile's MMA (multiple of 16, <= BN)
};

// Tile t of the tile list: active index a with tile_start[a] <= t (shared
// memory), then feature tile major, token tile minor inside the expert. An
// expert's m rows make nrt = ceil(m / BN) token tiles: BN rows each and a last
// tile with the rest, rounded up to kRound (16, or 32 for CTA-pair MMAs), so
// only that last tile runs padding rows (p.split_even: nrt tiles of equal
// width ceil(m / nrt) rounded up to kRound instead).
template <int kRound>
__device__ __forceinline__ Tile decode_tile(const GemmArgs& p, const int32_t* tile_start, int A,
                                            int t) {
  int lo = 0, hi = A - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  Tile r;
  r.e = p.active[lo];
  const int local = t - tile_start[lo];
  const int seg0 = p.offsets[r.e];
  const int seg1 = p.offsets[r.e + 1];
  const int m = seg1 - seg0;
  const int nrt = (m + p.BN - 1) / p.BN;
  r.ft = local / nrt;
  const int tt = local - r.ft * nrt;
  if (p.split_even) {
    r.width = (((m + nrt - 1) / nrt) + kRound - 1) & ~(kRound - 1);
    r.row0 = seg0 + tt * r.width;
  } else {
    const int rows = (tt + 1 < nrt) ? p.BN : m - (nrt - 1) * p.BN;
    r.width = (rows + kRound - 1) & ~(kRound - 1);
    r.row0 = seg0 + tt * p.BN;
  }
  r.row_end = min(seg1, r.row0 + r.width);
  return r;
}

// Every CTA builds the tile list of the launch in shared memory:
// tile_start[a] = sum over active experts a' < a of n_ftiles * ceil(m_e / BN),
// tile_start[A] = total, counting only experts with m_lo <= m_e <= m_hi (the
// others get no tiles: a launch can take one size class of experts). Offsets that do not describe M rows give an empty
// list and raise the device error. Returns A (0 when inconsistent).
__device__ int build_tile_list(const GemmArgs& p, int32_t* tile_start, int32_t* warp_tot) {
  const int nthr = blockDim.x;
  const int tid = threadIdx.x;
  const int A_raw = *p.num_active;
  const bool bad = (A_raw < 0 || A_raw > p.E || p.offsets[0] != 0 || p.offsets[p.E] != p.M);
  if (bad) {
    if (tid == 0) {
      if (blockIdx.x == 0) raise_device_error(MOE_DEVERR_BAD_OFFSETS);
      tile_start[0] = 0;
    }
    __syncthreads();
    return 0;
  }
  const int A = A_raw;
  const int per = (A + nthr - 1) / nthr;           // experts per thread (<= 3 for A <= 1024)
  const int a0 = min(A, tid * per), a1 = min(A, a0 + per);
  int local = 0;
  for (int a = a0; a < a1; ++a) {
    const int e = p.active[a];
    const int m = p.offsets[e + 1] - p.offsets[e];
    if (m >= p.m_lo && m <= p.m_hi) local += p.n_ftiles * ((m + p.BN - 1) / p.BN);
  }
  const int lane = tid & 31, w = tid >> 5, nw = nthr >> 5;
  int x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  int before = 0;
  for (int i = 0; i < w; ++i) before += warp_tot[i];
  int run = before + x - local;                     // exclusive prefix of this thread
  for (int a = a0; a < a1; ++a) {
    tile_start[a] = run;
    const int e = p.active[a];
    const int m = p.offsets[e + 1] - p.offsets[e];
    if (m >= p.m_lo && m <= p.m_hi) run += p.n_ftiles * ((m + p.BN - 1) / p.BN);
  }
  if (tid == nthr - 1) {
    int total = 0;
    for (int i = 0; i < nw; ++i) total += warp_tot[i];
    tile_start[A] = total;
  }
  __syncthreads();
  return A;
}

// SiLU and the logistic function with the fast exponential and division
// intrinsics (a few fp32 ulps): their results are rounded to BF16 right after,
// and the epilogue runs them for every output element while the dequant warps
// compete for the same issue slots.
__device__ __forceinline__ float sigmoid_f(float g) { return __fdividef(1.0f, 1.0f + __expf(-g)); }
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

template <int MODE, int FMT, int EPI, int LANES, int PAIR, int DQW>
__global__ void __launch_bounds__(gemm_threads(DQW), 1)
grouped_qgemm_kernel(const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_wq,
                     const __grid_constant__ CUtensorMap tm_sc, const GemmArgs p) {
  constexpr int kLanes = LANES;
  constexpr int kDqWarps = DQW;
  constexpr int kEpiWarp0 = kDqWarp0 + kDqWarps;
  constexpr int kDqWarpsPerLane = kDqWarps / LANES;   // 4 or 8
  constexpr int kParts = kDqWarpsPerLane / 4;         // warps per lane quarter
  static_assert(LANES % kProdWarps == 0 && LANES % kMaxIssuers == 0, "lanes own their stages");
  static_assert(kDqWarpsPerLane % 4 == 0 && (kParts == 1 || kParts == 2), "whole lane quarters");
  // PAIR: a cluster of two CTAs works on 256 output features (128 each) of
  // the same token tile with M = 256 MMAs issued by the even CTA; each CTA
  // loads and dequantizes its own weight rows and loads half of the token
  // rows (forward only).
  static_assert(!PAIR || MODE == kModeFwd, "CTA pairs run the forward kernels");
  // kModeFwdW: token tiles of up to 2 x kWideHalf rows, each K step issued as
  // two MMAs (tile columns [0, kWideHalf) and the rest) into one accumulator;
  // 64-wide fills, so an A stage is 32 tensor-memory columns.
  constexpr bool kWide = (MODE == kModeFwdW);
  constexpr bool kFwd = gemm_is_fwd(MODE);
  static_assert(!kWide || (!PAIR && LANES == 2), "wide tiles run on single CTAs with two lanes");
  constexpr int kWRound = PAIR ? 32 : 16;
  constexpr uint32_t kScEl = (FMT == MOE_W_INT4_G32_BF16) ? 2 : 1;
  constexpr bool kGluRows = (kFwd && EPI == MOE_EPI_SWIGLU);
  // Forward and kModeBwdT: fills of 128 reduction elements; the dequantized
  // A tile goes to tensor memory (64 columns per fill). kModeBwd: fills of
  // 64, A in a 128B-swizzled MN-major shared-memory tile.
  constexpr bool kTmemA = (MODE != kModeBwd);
  constexpr int kFillK = (kTmemA && !kWide) ? 128 : 64;
  constexpr int kFillGroups = kFillK / 32;                        // quantization groups per fill row
  constexpr int kAStageCols = kFillK / 2;                         // tensor-memory columns of an A stage
  constexpr uint32_t kSmemA = kTmemA ? 0u : kABytes;
  // Packed and scale bytes per fill: 128 weight rows x kFillK elements
  // (forward: kFillK / 2 bytes and kFillK / 32 scales a row), or kFillK
  // reduction rows x 128 features (backward: 64 bytes and 4 scales a row).
  constexpr uint32_t kWqFill = 64u * kFillK;
  constexpr uint32_t kScFill = 4u * kFillK * kScEl;
  constexpr int kBChunks = kFillK / 64;                           // 128-byte K chunks of B

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const int S = p.stages;
  const uint32_t stage_bytes = p.stage_bytes;
  // One [rows][64] BF16 chunk of token rows; a pair's CTAs hold BN / 2 rows each.
  const uint32_t b_chunk = static_cast<uint32_t>(PAIR ? p.BN / 2 : p.BN) * 128u;
  // (wide tiles: one box of kWideHalf rows, two when tiles may be wider)
  const bool wide2 = kWide && p.BN > kWideHalf;
  const uint32_t b_bytes = kWide ? (wide2 ? 2u : 1u) * kWideHalf * 128u : b_chunk * kBChunks;
  // One stage: [B kBChunks x BN*128][A 16 KiB (backward only)][packed][scales]
  auto B_at = [&](int s) { return base + s * stage_bytes; };
  auto A_at = [&](int s) { return base + s * stage_bytes + b_bytes; };
  auto W_at = [&](int s) { return base + s * stage_bytes + b_bytes + kSmemA; };
  auto S_at = [&](int s) { return base + s * stage_bytes + b_bytes + kSmemA + kWqFill; };
  // Two rings: S shared-memory fills (TMA) and SA A stages. In the forward
  // kernels the A stages live in tensor memory and may be fewer than the
  // fills; in the backward kernels the A tile is part of the fill (SA = S).
  const int SA = p.a_stages;
  // Forward with A halves: each A stage (64 tensor-memory columns, a 128-wide
  // fill) is handed over in two 64-wide halves, each with its own pair of
  // barriers, so the MMAs of a fill's first half start as soon as it is
  // dequantized and the next fill's first half may be written while the
  // second half's MMAs run. A-barrier j of stage sa is 2 sa + half.
  const bool halves = kTmemA && p.a_halves != 0;
  const int SAB = 2 * SA;                          // A-barrier slots reserved (two per stage)
  const uint32_t bars = base + S * stage_bytes;
  auto full_tma = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (S + s); };
  auto full_a = [&](int s) { return bars + 8u * (2 * S + s); };
  auto a_free = [&](int s) { return bars + 8u * (2 * S + SAB + s); };
  // Accumulator handoff: one pair of barriers per pipeline (two with tile
  // pipelines, else only the first is used).
  auto acc_full = [&](int q) { return bars + 8u * (2 * S + 2 * SAB + q); };
  auto acc_empty = [&](int q) { return bars + 8u * (2 * S + 2 * SAB + 2 + q); };
  const uint32_t drain_bar = bars + 8u * (2 * S + 2 * SAB + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + S * stage_bytes + 8u * (2 * S + 2 * SAB + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* warp_tot = reinterpret_cast<int32_t*>(tmem_slot + 4);          // [32]
  int32_t* tile_start = warp_tot + 32;                                      // [E + 1]
  // Epilogue staging: one 2 KiB block per epilogue warp (16 token rows x 64
  // BF16); then, for kModeBwdT, a 1 KiB transpose scratch per dequant warp.
  const uint32_t stg_base = (smem_u32(tile_start + p.E + 1) + 127u) & ~127u;
  const uint32_t scratch_base = stg_base + 4u * kStageBytesEpi;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Position in the pair (0 issues the MMAs and owns the barriers they wait
  // on) and the tile walk: a pair takes tile t, t + pairs, ...
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int t_first = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int t_step = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  // Tile pipelines (two issuers, two producers): the CTA's i-th tile belongs
  // to pipeline i % 2 as a whole: its producer and its issuer, which
  // accumulates all of the tile's fills in one accumulator, in fill order, so
  // a token's sum never depends on how the rest of the batch is tiled. With
  // two lanes, lane i % 2 dequantizes every fill of the tile; with four,
  // lanes i % 2 and i % 2 + 2 take the pipeline's fills in turn. One tile's
  // epilogue overlaps the other pipeline's tile. Otherwise (one issuer, or
  // MOEQ_PIPES=0) every member takes every other fill of every tile.
  const bool pipes = p.n_issuers == 2 && p.pipes != 0;
  // Forward, token rows gathered through an index instead of a tensor map.
  const bool gather = MODE == kModeFwd && p.b_rows != nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      // Gathered token rows: the producer's arrival with the weights' byte
      // count, and its arrival once the stage's row copies have landed.
      mbar_init(full_tma(s), gather ? 2 : 1);
      mbar_init(empty(s), 1);
    }
    // Arrivals on an A barrier: every dequant warp of the lane, or, with
    // halves and two warps per lane quarter, the four warps of that half. A
    // pair's odd CTA relays its dequant arrivals to the even CTA with one
    // remote arrival per barrier (its own warps arrive locally).
    const int dq_arrivals = (halves && kParts == 2) ? kDqWarpsPerLane / 2 : kDqWarpsPerLane;
    for (int s = 0; s < (halves ? SAB : SA); ++s) {
      mbar_init(full_a(s), (PAIR && rank == 0) ? dq_arrivals + 1 : dq_arrivals);
      mbar_init(a_free(s), 1);
    }
    mbar_init(acc_full(0), pipes ? 1 : p.n_issuers);
    mbar_init(acc_full(1), 1);
    // (wide tiles with one accumulator: the four epilogue warps and every
    // dequant warp drain it)
    mbar_init(acc_empty(0), PAIR ? 8 : ((kWide && p.n_issuers == 1) ? 4 + kDqWarps : 4));
    mbar_init(acc_empty(1), PAIR ? 8 : 4);
    mbar_init(drain_bar, p.n_issuers);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp < kProdWarps && lane == 0) {
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_wq);
    tma_prefetch_desc(&tm_sc);
  }
  if (warp == kIssuerWarp0) {
    if constexpr (PAIR) tmem_alloc_pair(smem_u32(tmem_slot), p.tmem_cols);
    else tmem_alloc(smem_u32(tmem_slot), p.tmem_cols);
  }
  tc_fence_before();
  // A pair also waits here until the other CTA's barriers are initialised.
  if constexpr (PAIR) cluster_sync_all(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above touches only this CTA's shared and tensor memory; the
  // routing tables and operands below come from earlier kernels.
  grid_dependency_wait();
  grid_dependents_launch();

  const int A = build_tile_list(p, tile_start, warp_tot);
  const int total = tile_start[A];
  // Tile t of the list as this CTA sees it (a pair's CTAs take feature tiles
  // 2 ft and 2 ft + 1 of the pair's feature tile ft).
  auto tile_at = [&](int t) {
    Tile tl = decode_tile<kWRound>(p, tile_start, A, t);
    if (PAIR) tl.ft = 2 * tl.ft + static_cast<int>(rank);
    return tl;
  };
  const int nkb = (p.R + kFillK - 1) / kFillK;   // forward K % 128 may be 64: zero tail
  const int N = p.N, K = p.K;
  // Tensor-memory columns: [partial accumulator 0 .. NI-1][A stage 0 .. S-1 (forward)].
  const int NI = p.n_issuers;
  const uint32_t a_col0 = static_cast<uint32_t>(NI * p.acc_cols);
  // Wide tiles with one accumulator: no MMA can start while a tile's
  // accumulator drains, and the dequant warps have then run out of A stages.
  // So the tile's 16-column chunks are shared by the five warps of each lane
  // quarter, its epilogue warp (helper 0) and its four dequant warps (helpers
  // 1-4, by index in the quarter): chunk i goes to helper i % 5. Each helper
  // stores its results straight from registers (a row's 16 or 32 values per
  // store instruction are contiguous), without the staging block.
  const bool helpers = kWide && NI == 1;
  constexpr int kHelpers = 1 + kDqWarps / 4;
  auto wide_chunk = [&](const Tile& tl, int c0) {
    const int qq = warp & 3;
    float v[16];
    {
      uint32_t ua[16];
      tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(qq * 32) << 16) + static_cast<uint32_t>(c0), ua);
      tmem_wait_ld();
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) v[jj] = __uint_as_float(ua[jj]);
    }
    const int nrows = min(16, tl.row_end - (tl.row0 + c0));
    uint16_t* out16 = reinterpret_cast<uint16_t*>(p.out);
    if constexpr (kGluRows) {
      // lanes 0-15: gate values of features pr, lanes 16-31: their up values
      const int pr = lane & 15;
      const bool is_gate = lane < 16;
      const int hrow0 = is_gate ? 0 : 8;
      const int fcol = tl.ft * 64 + qq * 16 + pr;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const float mine = is_gate ? v[jj] : v[jj + 8];
        const float got = __shfl_xor_sync(0xffffffffu, is_gate ? v[jj + 8] : v[jj], 16);
        const float g = is_gate ? mine : got;
        const float u = is_gate ? got : mine;
        const uint16_t h = __bfloat16_as_ushort(__float2bfloat16_rn(silu_f(g) * u));
        if (hrow0 + jj < nrows)
          out16[static_cast<int64_t>(tl.row0 + c0 + hrow0 + jj) * p.ldo + fcol] = h;
      }
      if (p.saved) {
        uint16_t* sv16 = reinterpret_cast<uint16_t*>(p.saved);
        const int scol = is_gate ? fcol : N / 2 + fcol;
#pragma unroll
        for (int jj = 0; jj < 16; ++jj)
          if (jj < nrows)
            sv16[static_cast<int64_t>(tl.row0 + c0 + jj) * N + scol] =
                __bfloat16_as_ushort(__float2bfloat16_rn(v[jj]));
      }
    } else {
      const int f = tl.ft * kTileF + qq * 32 + lane;
      if (f < p.F) {
#pragma unroll
        for (int jj = 0; jj < 16; ++jj)
          if (jj < nrows)
            out16[static_cast<int64_t>(tl.row0 + c0 + jj) * p.ldo + f] =
                __bfloat16_as_ushort(__float2bfloat16_rn(v[jj]));
      }
    }
  };
  // Helper h's share of tile tl's epilogue (the tile is the CTA's it-th).
  auto wide_epilogue = [&](const Tile& tl, int it, int h) {
    // lane 0's result decides for the warp, so the tensor-memory loads below
    // (warp-collective) run on all lanes or none
    const bool r = mbar_wait(acc_full(0), static_cast<uint32_t>(it & 1), abort_flag);
    if (!__shfl_sync(0xffffffffu, r ? 1 : 0, 0)) return false;
    tc_fence_after();
    for (int c0 = 16 * h; c0 < tl.width; c0 += 16 * kHelpers) wide_chunk(tl, c0);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acc_empty(0));
    return true;
  };

  if (warp < kProdWarps && gather) {
    // ------------------------------------------------------------ gathering producers
    // The whole warp copies the stage's token rows, 16 bytes a lane, from the
    // token rows b_src[b_rows[p]] into the 128B-swizzled [2 chunks][rows][64]
    // layout the tensor map would have written (16-byte unit u of row r at
    // unit u ^ (r % 8)), zero-filling rows past the tile and a reduction tail
    // past R; lane 0 issues the weight and scale copies. The row copies run in
    // the generic proxy and the MMAs read them through the async proxy, so a
    // stage is handed over only after its copies have completed and the lane
    // has fenced between the proxies: each fill's copies form one group, and
    // the previous own fill is signalled once only the newest group is in
    // flight (the ring has at least four stages, so this never waits on a
    // fill it has not released).
    const int pw = warp;
    const uint64_t pol_w = l2_policy_evict_first();
    const uint32_t tx = kWqFill + kScFill;
    int st = pw;
    uint32_t ph = 0;
    int pending = -1;                        // stage of the own fill not yet signalled
    long long g_next = pw, last_own = -1;    // ring index of the next / last issued own fill
    int r0 = 0;
    bool ok = true;
    int li = 0;
    constexpr int kTokRegs = 8;              // 32-row blocks of a tile (at most 256 rows)
    for (int t = t_first; t < total && ok; t += t_step, ++li) {
      int kb0 = (pw - r0 + kProdWarps) % kProdWarps, kbs = kProdWarps;
      r0 = (r0 + nkb) % kProdWarps;
      if (pipes) {
        if ((li & 1) != pw) continue;
        kb0 = 0;
        kbs = 1;
      }
      const Tile tl = tile_at(t);
      const int rows_here = PAIR ? (tl.width >> 1) : tl.width;
      const int brow = tl.row0 + static_cast<int>(rank) * rows_here;
      // Lane l holds the token of rows l, l + 32, ... of this CTA's share (-1 past the expert).
      int tok[kTokRegs];
#pragma unroll
      for (int j = 0; j < kTokRegs; ++j) {
        const int rr = 32 * j + lane;
        tok[j] = (rr < rows_here && brow + rr < tl.row_end) ? __ldg(p.b_rows + brow + rr) : -1;
      }
      for (int kb = kb0; kb < nkb; kb += kbs) {
        bool w_ok = true;
        if (lane == 0) w_ok = mbar_wait(empty(st), ph ^ 1u, abort_flag);
        if (!__shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0)) { ok = false; break; }
        const uint32_t bar = full_tma(st);
        if (lane == 0) {
          mbar_arrive_expect_tx(bar, tx);
          if constexpr (EPI == MOE_EPI_SWIGLU) {
            tma_load_3d_hint(W_at(st), &tm_wq, bar, kb * 64, tl.ft * 64, 2 * tl.e, pol_w);
            tma_load_3d_hint(S_at(st), &tm_sc, bar, tl.ft * 64, 0, tl.e * (K / 32) + kb * 4, pol_w);
          } else {
            tma_load_3d_hint(W_at(st), &tm_wq, bar, kb * 64, tl.e * N + tl.ft * kTileF, 0, pol_w);
            tma_load_3d_hint(S_at(st), &tm_sc, bar, tl.ft * kTileF, tl.e * (K / 32) + kb * 4, 0, pol_w);
          }
        }
        // Row rl of a 32-row block: lanes 0-15 row 2 mm, lanes 16-31 row 2 mm + 1;
        // lanes 8-15 (24-31) the second 64-element chunk; unit u = lane % 8.
        const int c = (lane >> 3) & 1, u = lane & 7;
        const bool k_ok = kb * kFillK + c * 64 < p.R;
        const uint32_t bst = B_at(st) + static_cast<uint32_t>(c) * b_chunk;
#pragma unroll
        for (int j = 0; j < kTokRegs; ++j) {
          if (32 * j >= rows_here) break;
#pragma unroll 4
          for (int mm = 0; mm < 16; ++mm) {
            const int rl = 2 * mm + (lane >> 4);
            const int r = 32 * j + rl;
            const int tk = __shfl_sync(0xffffffffu, tok[j], rl);
            const bool valid = k_ok && tk >= 0;
            const __nv_bfloat16* src =
                p.b_src + (valid ? static_cast<int64_t>(tk) * p.R + kb * kFillK + c * 64 + u * 8 : 0);
            if (r < rows_here)
              cp_async_16(bst + static_cast<uint32_t>(r) * 128u + ((u ^ (r & 7)) << 4), src,
                          valid ? 16u : 0u);
          }
        }
        cp_async_commit();
        if (pending >= 0) {
          cp_async_wait<1>();
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(full_tma(pending));
        }
        pending = st;
        last_own = g_next;
        g_next += kProdWarps;
        st += kProdWarps;
        if (st >= S) { st -= S; ph ^= 1u; }
      }
    }
    // The last own fill (also after an abort: its copies land, then it is
    // signalled, so no consumer waits on it in vain and no copy outlives the CTA).
    cp_async_wait<0>();
    fence_proxy_async_smem();
    __syncwarp();
    if (pending >= 0 && lane == 0) mbar_arrive(full_tma(pending));
    if (!ok && lane == 0) {
      // Weight copies that may still be in flight (own fills within the last
      // S) land before the CTA can exit: each such stage's phase completes.
      for (long long g = last_own; g >= 0 && g > last_own - S; g -= kProdWarps)
        mbar_drain(full_tma(static_cast<int>(g % S)), static_cast<uint32_t>((g / S) & 1));
    }
  } else if (warp < kProdWarps) {
    // ------------------------------------------------------------ TMA producers
    // Producer pw issues fills f with f % kProdWarps == pw: one thread issues
    // the fill's three bulk tensor copies (token rows, packed weights, group
    // scales) on the fill's stage f % S. A single thread needs a few hundred
    // cycles per fill for the barrier wait and the copy issue; two producers
    // overlap that latency.
    if (lane == 0) {
      const int pw = warp;
      const uint64_t pol_b = l2_policy_evict_last();
      const uint64_t pol_w = l2_policy_evict_first();
      const uint32_t tx = b_bytes + kWqFill + kScFill;
      int st = pw;                           // stage of the next own fill
      uint32_t ph = 0;
      // g: ring index of the next own fill (pw, pw + 2, ...; with tile
      // pipelines a virtual index, since the member then takes whole tiles).
      long long g_next = pw, last_own = -1;
      int r0 = 0;                            // (first fill of the tile) % kProdWarps
      bool ok = true;
      int li = 0;                            // this CTA's tile count
      for (int t = t_first; t < total && ok; t += t_step, ++li) {
        int kb0 = (pw - r0 + kProdWarps) % kProdWarps, kbs = kProdWarps;
        r0 = (r0 + nkb) % kProdWarps;
        if (pipes) {
          if ((li & 1) != pw) continue;
          kb0 = 0;
          kbs = 1;
        }
        const Tile tl = tile_at(t);
        // A pair's CTAs hold token rows [0, w/2) and [w/2, w) of the tile.
        const int brow = tl.row0 + static_cast<int>(rank) * (tl.width >> 1);
        for (int kb = kb0; kb < nkb; kb += kbs) {
          if (!mbar_wait(empty(st), ph ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t bar = full_tma(st);
          mbar_arrive_expect_tx(bar, tx);
          if constexpr (kWide) {
            // token rows in two boxes of kWideHalf rows: [2 x kWideHalf][64]
            tma_load_3d_hint(B_at(st), &tm_b, bar, 0, brow, kb, pol_b);
            if (wide2)
              tma_load_3d_hint(B_at(st) + kWideHalf * 128u, &tm_b, bar, 0, brow + kWideHalf, kb, pol_b);
          } else {
            tma_load_3d_hint(B_at(st), &tm_b, bar, 0, brow, kb * kBChunks, pol_b);
          }
          if constexpr (kFwd) {
            // kFillK / 2 packed bytes and kFillGroups scales per weight row
            if constexpr (EPI == MOE_EPI_SWIGLU) {
              // packed: [2 halves][64 rows][kFillK / 2 B]; scales: [groups][2 halves][64]
              tma_load_3d_hint(W_at(st), &tm_wq, bar, kb * (kFillK / 2), tl.ft * 64, 2 * tl.e, pol_w);
              tma_load_3d_hint(S_at(st), &tm_sc, bar, tl.ft * 64, 0, tl.e * (K / 32) + kb * kFillGroups, pol_w);
            } else {
              // packed: [128 rows][kFillK / 2 B]; scales: [groups][128 rows]
              tma_load_3d_hint(W_at(st), &tm_wq, bar, kb * (kFillK / 2), tl.e * N + tl.ft * kTileF, 0, pol_w);
              tma_load_3d_hint(S_at(st), &tm_sc, bar, tl.ft * kTileF, tl.e * (K / 32) + kb * kFillGroups, 0, pol_w);
            }
          } else {
            // packed: [64 rows][64 B]; scales: [4 groups][64 rows]
            tma_load_3d_hint(W_at(st), &tm_wq, bar, tl.ft * 64, tl.e * N + kb * kFillK, 0, pol_w);
            tma_load_3d_hint(S_at(st), &tm_sc, bar, kb * kFillK, tl.e * (K / 32) + tl.ft * 4, 0, pol_w);
          }
          last_own = g_next;
          g_next += kProdWarps;
          st += kProdWarps;
          if (st >= S) { st -= S; ph ^= 1u; }
        }
      }
      if (!ok) {
        // Let this producer's copies that may still be in flight land before
        // the CTA can exit (its fills within the last S).
        for (long long g = last_own; g >= 0 && g > last_own - S; g -= kProdWarps)
          mbar_drain(full_tma(static_cast<int>(g % S)), static_cast<uint32_t>((g / S) & 1));
      }
    }
  } else if (warp >= kIssuerWarp0 && warp < kIssuerWarp0 + NI) {
    if constexpr (PAIR) {
      // -------------------------------------------------------- pair relay
      // The odd CTA issues no MMA. One thread of its first issuer warp waits
      // for each A stage of this CTA to be complete (its dequant warps
      // arrive locally) and passes that on with a single arrival on the even
      // CTA's barrier of the stage.
      // With tile pipelines, issuer warp j's lane relays pipeline j's fills.
      const int j = warp - kIssuerWarp0;
      if (rank == 1 && lane == 0 && (pipes || j == 0)) {
        int sa = pipes ? j : 0;
        const int sa_step = pipes ? NI : 1;
        uint32_t pha = 0;
        bool ok = true;
        int li = 0;
        for (int t = t_first; t < total && ok; t += t_step, ++li) {
          if (pipes && (li & 1) != j) continue;
          for (int kb = 0; kb < nkb && ok; ++kb) {
            for (int h = 0; h < (halves ? 2 : 1); ++h) {
              const int jb = halves ? 2 * sa + h : sa;
              if (!mbar_wait(full_a(jb), pha, abort_flag)) { ok = false; break; }
              mbar_arrive_cluster(cluster_addr(full_a(jb), 0));
            }
            sa += sa_step;
            if (sa >= SA) { sa -= SA; pha ^= 1u; }
          }
        }
      }
    }
    // ------------------------------------------------------------ MMA issuers
    // Two issuing warps: with tile pipelines each accumulates whole tiles;
    // otherwise issuer j takes the fills f with f % NI == j into its own
    // partial accumulator and the epilogue adds the partials in issuer order.
    // The whole warp runs the loop and waits; one elected lane issues the
    // MMAs and commits. In a pair only the even CTA issues; its MMAs read the
    // A stages and token rows of both CTAs and write both accumulators, and
    // its commits arrive on the barriers of both.
    if (rank == 0) {
      const int j = warp - kIssuerWarp0;
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(j * p.acc_cols);
      int st = j, sa = j;                     // stages of the next own fill (f = j, j + NI, ...)
      uint32_t pha = 0;
      int it = 0;
      int r0 = 0;                             // (first fill of the tile) % NI
      bool ok = true;
      auto commit = [](uint32_t bar) {
        if constexpr (PAIR) mma_commit_pair(bar, 3); else mma_commit(bar);
      };
      auto mma_ts = [](uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t accum) {
        if constexpr (PAIR) mma_bf16_ts_pair(d, a, b, id, accum); else mma_bf16_ts(d, a, b, id, accum);
      };
      // Barriers the other CTA of a pair arrives on are waited with cluster
      // scope. Every lane waits; lane 0's result decides for the warp.
      auto wait_x = [&](uint32_t bar, uint32_t parity) {
        bool r;
        if constexpr (PAIR) r = mbar_wait_cluster(bar, parity, abort_flag);
        else r = mbar_wait(bar, parity, abort_flag);
        return __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
      };
      int li = 0;                             // this CTA's tile count
      for (int t = t_first; t < total && ok; t += t_step, ++li) {
        int kb0 = (j - r0 + NI) % NI, kbs = NI;
        r0 = (r0 + nkb) % NI;
        if (pipes) {
          if ((li & 1) != j) continue;
          kb0 = 0;
          kbs = 1;
        }
        const int q_acc = pipes ? j : 0;       // accumulator handoff barriers of this tile
        const int width = tile_at(t).width;
        // Wide tiles: columns [0, kWideHalf) and [kWideHalf, width) as two MMAs.
        const int n2 = kWide ? width - kWideHalf : 0;
        const uint32_t idesc = idesc_bf16_f32(PAIR ? 2 * kTileF : kTileF,
                                              (kWide && n2 > 0) ? kWideHalf : width,
                                              MODE == kModeBwd ? 1u : 0u, 0u);
        const uint32_t idesc2 = idesc_bf16_f32(kTileF, n2 > 0 ? n2 : 16, 0u, 0u);
        if (!wait_x(acc_empty(q_acc), static_cast<uint32_t>(it & 1) ^ 1u)) { ok = false; break; }
        tc_fence_after();
        uint32_t acc = 0;
        for (int kb = kb0; kb < nkb; kb += kbs) {
          if (kTmemA && halves) {
            // Two halves: four MMAs each (K = 64), each after its own barrier;
            // the first half's A columns are released while the second runs.
            const uint64_t b0 = smem_desc_sw128(B_at(st), 16, 1024);
            const uint32_t a0 = tmem_base + a_col0 + static_cast<uint32_t>(sa * 64);
            if (!wait_x(full_a(2 * sa), pha)) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) {
              mma_ts(d_tmem, a0, b0, idesc, acc);
              mma_ts(d_tmem, a0 + 8, b0 + 2, idesc, 1u);
              mma_ts(d_tmem, a0 + 16, b0 + 4, idesc, 1u);
              mma_ts(d_tmem, a0 + 24, b0 + 6, idesc, 1u);
              commit(a_free(2 * sa));
            }
            __syncwarp();
            if (!wait_x(full_a(2 * sa + 1), pha)) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) {
              const uint64_t b1 = b0 + (b_chunk >> 4);
              mma_ts(d_tmem, a0 + 32, b1, idesc, 1u);
              mma_ts(d_tmem, a0 + 40, b1 + 2, idesc, 1u);
              mma_ts(d_tmem, a0 + 48, b1 + 4, idesc, 1u);
              mma_ts(d_tmem, a0 + 56, b1 + 6, idesc, 1u);
              commit(a_free(2 * sa + 1));
              commit(empty(st));
            }
            __syncwarp();
            acc = 1u;
          } else {
            if (!wait_x(full_a(sa), pha)) { ok = false; break; }
            tc_fence_after();
            const uint64_t b0 = smem_desc_sw128(B_at(st), 16, 1024);
            if (elect_one()) {
              if constexpr (kWide) {
                // A stage sa: 128 lanes x 32 columns (64 K); each K step of 16
                // (8 columns) multiplies the tile's first kWideHalf token rows
                // and, for wider tiles, the rest into accumulator columns
                // kWideHalf onward.
                const uint32_t a0 = tmem_base + a_col0 + static_cast<uint32_t>(sa * kAStageCols);
                const uint64_t b1 = b0 + ((kWideHalf * 128u) >> 4);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                  const uint32_t accum = (ks == 0) ? acc : 1u;
                  mma_ts(d_tmem, a0 + 8 * ks, b0 + 2 * ks, idesc, accum);
                  if (n2 > 0) mma_ts(d_tmem + kWideHalf, a0 + 8 * ks, b1 + 2 * ks, idesc2, accum);
                }
              } else if constexpr (kTmemA) {
                // A stage st: 128 lanes x 64 columns (two BF16 per column): K=16 = 8 columns.
                const uint32_t a0 = tmem_base + a_col0 + static_cast<uint32_t>(sa * 64);
                const uint64_t b1 = b0 + (b_chunk >> 4);
                mma_ts(d_tmem, a0, b0, idesc, acc);
                mma_ts(d_tmem, a0 + 8, b0 + 2, idesc, 1u);
                mma_ts(d_tmem, a0 + 16, b0 + 4, idesc, 1u);
                mma_ts(d_tmem, a0 + 24, b0 + 6, idesc, 1u);
                mma_ts(d_tmem, a0 + 32, b1, idesc, 1u);
                mma_ts(d_tmem, a0 + 40, b1 + 2, idesc, 1u);
                mma_ts(d_tmem, a0 + 48, b1 + 4, idesc, 1u);
                mma_ts(d_tmem, a0 + 56, b1 + 6, idesc, 1u);
              } else {
                const uint64_t a0 = smem_desc_sw128(A_at(st), 8192, 1024);
                mma_bf16_ss(d_tmem, a0, b0, idesc, acc);
                mma_bf16_ss(d_tmem, a0 + 128, b0 + 2, idesc, 1u);
                mma_bf16_ss(d_tmem, a0 + 256, b0 + 4, idesc, 1u);
                mma_bf16_ss(d_tmem, a0 + 384, b0 + 6, idesc, 1u);
              }
              commit(empty(st));
              if constexpr (kTmemA) commit(a_free(sa));
            }
            __syncwarp();
            acc = 1u;
          }
          st += NI;
          if (st >= S) st -= S;
          sa += NI;
          if (sa >= SA) { sa -= SA; pha ^= 1u; }
        }
        if (ok && elect_one()) commit(acc_full(q_acc));   // arrives even when this issuer had no fill
        __syncwarp();
        ++it;                                 // tiles this issuer has handed over
      }
      // All MMAs of this CTA (of the pair) done before tensor memory is released.
      if (elect_one()) commit(drain_bar);
      __syncwarp();
      if (lane == 0) mbar_drain(drain_bar, 0);
      __syncwarp();
    }
  } else if (warp >= kDqWarp0 && warp < kDqWarp0 + kLanes * kDqWarpsPerLane) {
    // ------------------------------------------------------------ dequantizers
    // kLanes groups of kDqWarpsPerLane warps take the fills in turn (fill f
    // goes to group f % kLanes). In a group, warp (q, hk) covers tensor-memory
    // lane quarter q (32 rows of the A tile) and part hk of the kParts parts
    // of the fill's reduction span (forward: 4 / kParts 32-element groups).
    const int grp = (warp - kDqWarp0) / kDqWarpsPerLane;
    const int hk = ((warp - kDqWarp0) >> 2) % kParts;
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int i = q * 32 + lane;            // A row (forward) / thread slot (backward)
    // Forward: A row i is one output feature. With SwiGLU each warp's 32 rows
    // hold 16 gate rows (lanes 0-15: packed rows 16q + l) and the 16 matching
    // up rows (lanes 16-31: packed rows 64 + 16q + l - 16), so every 8-lane
    // phase of a 128-bit shared load touches 8 distinct swizzle slots.
    const int src = kGluRows ? ((lane < 16) ? (16 * q + lane) : (64 + 16 * q + lane - 16)) : i;
    // Fill f of the CTA uses stage f % S with parity (f / S) & 1; this group
    // owns fills grp, grp + kLanes, ... and steps its stage and parity
    // incrementally.
    int r0 = 0;                             // (first fill of the tile) % kLanes
    // With tile pipelines: lanes grp % 2 + 2 h (h < kLanes / 2) serve pipeline
    // grp % 2, taking its fills n (counted across the pipeline's tiles) with
    // n % (kLanes / 2) == h; rp = (fills of the pipeline so far) % (kLanes / 2).
    constexpr int kPipeLanes = kLanes / 2;
    const int pipe_of = grp & 1, pipe_h = grp >> 1;
    int rp = 0;
    int st = grp, sa = grp;                 // fill ring and A ring positions of the next own fill
    uint32_t ph = 0, pha = 0;
    bool ok = true;
    int li = 0;                             // this CTA's tile count
    for (int t = t_first; t < total && ok; t += t_step, ++li) {
      int kb_first = (grp - r0 + kLanes) % kLanes, kb_step = kLanes;
      r0 = (r0 + nkb) % kLanes;
      if (pipes) {
        if ((li & 1) != pipe_of) continue;
        kb_first = (pipe_h - rp + kPipeLanes) % kPipeLanes;
        kb_step = kPipeLanes;
        rp = (rp + nkb) % kPipeLanes;
      }
      for (int kb = kb_first; kb < nkb; kb += kb_step) {
        const int cur = st, cur_a = sa;
        const uint32_t cur_ph = ph, cur_pha = pha;
        const int kb_cur = kb;
        st += kLanes;
        if (st >= S) { st -= S; ph ^= 1u; }
        sa += kLanes;
        if (sa >= SA) { sa -= SA; pha ^= 1u; }
        if (!mbar_wait(full_tma(cur), cur_ph, abort_flag)) { ok = false; break; }
        const uint32_t wq = W_at(cur);
        const uint32_t sc = S_at(cur);
        if constexpr (kFwd) {
          // Packed rows are kFillK / 2 bytes with the TMA swizzle of that width
          // (16-byte chunk index ^= (row >> 1) & 3 for 64-byte rows, ^= (row >> 2)
          // & 1 for 32-byte rows). Scales: [kFillGroups groups][128 rows].
          const uint32_t prow = wq + src * (kFillK / 2);
          const uint32_t sw = (kFillK == 128) ? ((src >> 1) & 3) : ((src >> 2) & 1);
          const uint32_t trow = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a_col0 +
                                static_cast<uint32_t>(cur_a * kAStageCols);
          // The A stage (or, with halves, each half of it) must have been
          // released by the MMAs of the fill that used it SA fills ago. A
          // warp covers the fill's four 32-element groups (one warp per lane
          // quarter) or two of them (one half); with halves it hands each
          // half over on that half's barrier, else the whole fill at once.
          // Each group is stored to tensor memory as soon as it is
          // dequantized (16 columns, two BF16 per column, low half = even
          // k), which keeps only 16 results live. A half past the reduction
          // length (K % 128 == 64) is written as zeros, so neither the
          // zero-filled codes nor a foreign scale can reach the MMA.
          constexpr int kGroups = kFillGroups / kParts;
          const int units = (halves && kParts == 1) ? 2 : 1;
          for (int u = 0; u < units && ok; ++u) {
            const int half = (kParts == 2) ? hk : u;
            const int jb = halves ? 2 * cur_a + half : cur_a;
            if (!mbar_wait(a_free(jb), cur_pha ^ 1u, abort_flag)) { ok = false; break; }
#pragma unroll
            for (int cc = 0; cc < kGroups; ++cc) {
              const int c = hk * kGroups + cc;
              if (units == 2 && (c >> 1) != half) continue;
              uint32_t o[16];
              if (kb_cur * kFillK + c * 32 >= p.R) {
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) o[jj] = 0u;
              } else {
                const uint4 pk = lds128(prow + ((c ^ sw) << 4));
                const uint32_t soff = c * 128 + src;
                const uint32_t sbits = (FMT == MOE_W_INT4_G32_BF16) ? lds_u16(sc + soff * 2)
                                                                    : lds_u8(sc + soff);
                dequant32<FMT>(pk, sbits, o);
              }
              tmem_st_32x32b_x16(trow + static_cast<uint32_t>(c * 16), o);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            // (In a pair the odd CTA's relay thread passes this on.)
            if (lane == 0) mbar_arrive(full_a(jb));
          }
          if (!ok) break;
        } else if constexpr (MODE == kModeBwdT) {
          // A in tensor memory, K-major: lane = output feature (k) of the
          // tile, column = a pair of reduction rows (n, n + 1), low half n.
          // A packed row runs along k, and the warp's lane quarter q holds
          // exactly quantization group q of every row, so a lane dequantizes
          // one row n (32 features) at a time. The warp stages its 32 rows
          // in its scratch 16 features at a time ([32 rows][32 B]; chunk c of
          // row r at c ^ ((r >> 2) & 1), conflict-free for these writes and
          // for the reads) and reads them back transposed with ldmatrix: in
          // its fragments thread t holds feature t / 4 and the row pair
          // (2 (t%4), 2 (t%4) + 1), which is the register layout of the
          // tcgen05.st 16x128b shape (lane t / 4, column t % 4). Packed rows
          // are 64 bytes with the TMA 64-byte swizzle, scales [4 groups][128
          // rows]; rows past the reduction length (N % 128 == 64) are zeros.
          constexpr int kRowsPerWarp = kFillK / kParts;    // 64 or 128
          const uint32_t scr = scratch_base + static_cast<uint32_t>(warp - kDqWarp0) * kScratchBytes;
          const uint32_t wr = scr + static_cast<uint32_t>(lane) * 32u;
          const uint32_t wsw = static_cast<uint32_t>(lane >> 2) & 1u;
          // ldmatrix: lane l gives row l % 8 of matrix l / 8; the matrices are
          // (rows 0-7, features 0-7), (rows 0-7, 8-15), (rows 8-15, 0-7),
          // (rows 8-15, 8-15), i.e. registers (lane, column) blocks (0, 0),
          // (8, 0), (0, 4), (8, 4) of the 16x128b store.
          const int lm_row = (lane & 7) + ((lane >> 4) << 3);
          const int lm_chunk = (lane >> 3) & 1;
          const uint32_t lm0 = scr + static_cast<uint32_t>(lm_row) * 32u +
                               (static_cast<uint32_t>(lm_chunk ^ ((lm_row >> 2) & 1)) << 4);
          const uint32_t lm1 = lm0 + 16u * 32u;   // rows 16-31 (same swizzle)
          if (!mbar_wait(a_free(cur_a), cur_pha ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t tstage = tmem_base + a_col0 + static_cast<uint32_t>(cur_a * 64);
          for (int sj = 0; sj < kRowsPerWarp / 32; ++sj) {
            const int nb = hk * kRowsPerWarp + sj * 32;     // first row of the 32
            const int n = nb + lane;
            uint32_t o[16];
            if (kb_cur * kFillK + n >= p.R) {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) o[jj] = 0u;
            } else {
              const uint4 pk = lds128(wq + n * 64 + ((q ^ ((n >> 1) & 3)) << 4));
              const uint32_t soff = q * 128 + n;
              const uint32_t sbits = (FMT == MOE_W_INT4_G32_BF16) ? lds_u16(sc + soff * 2)
                                                                  : lds_u8(sc + soff);
              dequant32<FMT>(pk, sbits, o);
            }
            const uint32_t tcol = tstage + static_cast<uint32_t>(nb >> 1);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              // features 16h .. 16h + 15 of the 32 rows
              sts128(wr + (wsw << 4), o[8 * h], o[8 * h + 1], o[8 * h + 2], o[8 * h + 3]);
              sts128(wr + ((wsw ^ 1u) << 4), o[8 * h + 4], o[8 * h + 5], o[8 * h + 6], o[8 * h + 7]);
              __syncwarp();
              uint32_t tr[8];
              ldsm_x4_trans(lm0, tr[0], tr[1], tr[2], tr[3]);
              ldsm_x4_trans(lm1, tr[4], tr[5], tr[6], tr[7]);
              tmem_st_16x128b_x4(tcol + (static_cast<uint32_t>(q * 32 + 16 * h) << 16), tr);
              __syncwarp();
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(full_a(cur_a));
        } else {
          // Thread = (reduction row r, feature half hf): 64 features = 2
          // groups, split over the kParts warps of the lane quarter. Packed
          // rows are 64 bytes with the TMA 64-byte swizzle (chunk ^= (r >> 1)
          // & 3). Scales: [4 groups][64 rows].
          const uint32_t a_st = A_at(cur);
          const int r = i & 63;
          const int hf = i >> 6;
#pragma unroll
          for (int jj = 0; jj < 2 / kParts; ++jj) {
            const int jh = hk * (2 / kParts) + jj;
            const int c = 2 * hf + jh;
            const uint4 pk = lds128(wq + r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
            const uint32_t soff = c * 64 + r;
            const uint32_t sbits = (FMT == MOE_W_INT4_G32_BF16) ? lds_u16(sc + soff * 2)
                                                                : lds_u8(sc + soff);
            uint32_t o[16];
            dequant32<FMT>(pk, sbits, o);
            // MN-major, 128B swizzle: features in 64-wide blocks 8 KiB apart,
            // reduction row r at (r/8)*1024 + (r%8)*128, 16-byte chunk cc ^ (r%8).
            const uint32_t rowb = a_st + hf * 8192 + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const uint32_t chunk = (4 * jh + w) ^ (r & 7);
              sts128(rowb + (chunk << 4), o[4 * w], o[4 * w + 1], o[4 * w + 2], o[4 * w + 3]);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(full_a(cur_a));
        }
      }
      // Wide tiles: this warp's share of the tile's epilogue, once its MMAs
      // are done (every dequant warp arrives on the accumulator's barrier).
      if (helpers && ok) ok = wide_epilogue(tile_at(t), li, 1 + ((warp - kDqWarp0) >> 2));
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    // Sums the partial accumulators (fixed order), converts to BF16, stages 32
    // token rows at a time in this warp's shared block and writes them with
    // 16-byte stores, only for rows that belong to the tile's expert.
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int fr = q * 32 + lane;           // accumulator row = tile feature
    const uint32_t stg = stg_base + static_cast<uint32_t>(q) * kStageBytesEpi;
    uint16_t* stg_ptr = reinterpret_cast<uint16_t*>(gbase + (stg - base));
    static_assert(kMaxIssuers <= 3, "the epilogue sums at most three partial accumulators");
    // SwiGLU backward: the saved g and u of 16 token rows x this warp's 32
    // features come into the warp's staging block ([16 rows][32 g | 32 u],
    // 2 KiB) by cp.async, 16 bytes a copy and four copies a lane, one chunk
    // ahead: the first chunk of a tile before its accumulator is waited for,
    // the next one as soon as the previous chunk has been written out. Rows
    // past the tile are zero-filled; a warp whose features lie past F copies
    // nothing.
    constexpr bool kGuStaged = (MODE != kModeFwd && EPI == MOE_EPI_SWIGLU_BWD);
    auto prefetch_gu = [&](const Tile& tl, int c0) {
      const int fb = tl.ft * kTileF + q * 32;
      if (fb >= p.F) return;
      const int nrows = min(16, tl.row_end - (tl.row0 + c0));
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int idx = lane + 32 * j;
        const int rr = idx >> 3, pc = idx & 7;          // row, 16-byte piece (4 of g, 4 of u)
        const bool ok = rr < nrows;
        const __nv_bfloat16* src =
            p.saved + (ok ? static_cast<int64_t>(tl.row0 + c0 + rr) * (2 * K) + (pc < 4 ? 0 : K) +
                                fb + (pc & 3) * 8
                          : 0);
        cp_async_16(stg + static_cast<uint32_t>(rr * 128 + pc * 16), src, ok ? 16u : 0u);
      }
      cp_async_commit();
    };
    int it = 0;
    int r0 = 0;                             // (first fill of the tile) % NI
    for (int t = t_first; t < total; t += t_step, ++it) {
      const Tile tl = tile_at(t);
      if (helpers) {                        // wide tiles: helper 0's share of the chunks
        if (!wide_epilogue(tl, it, 0)) break;
        continue;
      }
      if constexpr (kGuStaged) prefetch_gu(tl, 0);
      // Issuer j wrote its partial in this tile iff one of the tile's nkb
      // fills f has f % NI == j. With tile pipelines the tile's whole sum is
      // in accumulator it % 2.
      const bool has0 = ((NI - r0) % NI) < nkb;
      const bool has1 = NI > 1 && ((1 + NI - r0) % NI) < nkb;
      const bool has2 = kMaxIssuers > 2 && NI > 2 && ((2 + NI - r0) % NI) < nkb;
      r0 = (r0 + nkb) % NI;
      const int q_acc = pipes ? (it & 1) : 0;
      // Tensor-memory column offsets of the written partials, in issuer order.
      const uint32_t acc = static_cast<uint32_t>(p.acc_cols);
      const int nv = pipes ? 1 : int(has0) + int(has1) + int(has2);
      const uint32_t pc0 = pipes ? static_cast<uint32_t>(q_acc) * acc
                                 : (has0 ? 0u : (has1 ? acc : 2 * acc));
      const uint32_t pc1 = (has0 && has1) ? acc : 2 * acc;
      const uint32_t pc2 = 2 * acc;
      if (!mbar_wait(acc_full(q_acc), static_cast<uint32_t>((pipes ? (it >> 1) : it) & 1),
                     abort_flag))
        break;
      tc_fence_after();
      const uint32_t tcol = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      for (int c0 = 0; c0 < tl.width; c0 += 16) {
        float v[16];
        {
          // The partials written in this tile, in issuer order: the first two
          // loaded together, the third after them.
          uint32_t ua[16], ub[16];
          tmem_ld_32x32b_x16(tcol + pc0 + c0, ua);
          if (nv > 1) tmem_ld_32x32b_x16(tcol + pc1 + c0, ub);
          tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            v[jj] = __uint_as_float(ua[jj]);
            if (nv > 1) v[jj] += __uint_as_float(ub[jj]);
          }
          if (nv > 2) {
            tmem_ld_32x32b_x16(tcol + pc2 + c0, ua);
            tmem_wait_ld();
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) v[jj] += __uint_as_float(ua[jj]);
          }
        }
        const int nrows = min(16, tl.row_end - (tl.row0 + c0));
        if constexpr (kGluRows) {
          // Lanes 0-15 hold gate values g, lanes 16-31 the up values u of the
          // same 16 features (pr = lane & 15). Each lane forms h = silu(g) * u
          // for 8 of the 16 token columns, gate lanes columns 0-7 and up lanes
          // 8-15, after swapping the missing operand with lane ^ 16. The code
          // has no branch, so the eight columns' exponentials, divisions and
          // shuffles overlap. Staging row (64 BF16): [0,16) h, [16,32) g, [32,48) u.
          const int pr = lane & 15;
          const bool is_gate = lane < 16;
          const int hrow0 = is_gate ? 0 : 8;
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const float mine = is_gate ? v[jj] : v[jj + 8];
            const float got = __shfl_xor_sync(0xffffffffu, is_gate ? v[jj + 8] : v[jj], 16);
            const float g = is_gate ? mine : got;
            const float u = is_gate ? got : mine;
            stg_ptr[(hrow0 + jj) * 64 + pr] = __bfloat16_as_ushort(__float2bfloat16_rn(silu_f(g) * u));
          }
          if (p.saved) {
            // g to columns [16, 32) from the gate lanes, u to [32, 48) from the up lanes.
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
              stg_ptr[jj * 64 + 16 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(v[jj]));
          }
          __syncwarp();
          // 16 H features of this warp: 32 B per row = 2 chunks; g and u likewise.
          const int fcol = tl.ft * 64 + q * 16;
          const int nseg = p.saved ? 3 : 1;
          for (int idx = lane; idx < 16 * 2 * nseg; idx += 32) {
            const int seg = idx / 32, rr = (idx % 32) >> 1, ch = idx & 1;
            if (rr < nrows) {
              const uint4 val = *reinterpret_cast<const uint4*>(stg_ptr + rr * 64 + seg * 16 + ch * 8);
              const int64_t grow = static_cast<int64_t>(tl.row0 + c0 + rr);
              __nv_bfloat16* dst = (seg == 0) ? p.out + grow * p.ldo + fcol
                                 : (seg == 1) ? p.saved + grow * N + fcol
                                              : p.saved + grow * N + N / 2 + fcol;
              *reinterpret_cast<uint4*>(dst + ch * 8) = val;
            }
          }
          __syncwarp();
        } else if constexpr (MODE != kModeFwd && EPI == MOE_EPI_SWIGLU_BWD) {
          const int f = tl.ft * kTileF + fr;      // feature of dh (< K)
          const bool fok = f < p.F;
          // This chunk's g and u have landed; each lane turns its own two
          // slots of every row (g -> dg, u -> du) in place, so the block is
          // then the [16 rows][32 dg | 32 du] staging of the output.
          cp_async_wait<0>();
          __syncwarp();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const bool ok = fok && jj < nrows;
            const float g = __uint_as_float(static_cast<uint32_t>(stg_ptr[jj * 64 + lane]) << 16);
            const float u = __uint_as_float(static_cast<uint32_t>(stg_ptr[jj * 64 + 32 + lane]) << 16);
            const float s = sigmoid_f(g);
            const float x = v[jj];
            const uint16_t dg = ok ? __bfloat16_as_ushort(__float2bfloat16_rn(x * u * s * (1.0f + g * (1.0f - s)))) : uint16_t(0);
            const uint16_t du = ok ? __bfloat16_as_ushort(__float2bfloat16_rn(x * g * s)) : uint16_t(0);
            stg_ptr[jj * 64 + lane] = dg;
            stg_ptr[jj * 64 + 32 + lane] = du;
          }
          __syncwarp();
          const int fb = tl.ft * kTileF + q * 32;
          if (fb < p.F) {
            for (int idx = lane; idx < 16 * 8; idx += 32) {
              const int rr = idx >> 3, ch = idx & 7;     // 8 chunks: 4 of dg, 4 of du
              if (rr < nrows) {
                const uint4 val = *reinterpret_cast<const uint4*>(stg_ptr + rr * 64 + ch * 8);
                const int64_t rb = static_cast<int64_t>(tl.row0 + c0 + rr) * (2 * K);
                __nv_bfloat16* dst = p.out + rb + (ch < 4 ? 0 : K) + fb + (ch & 3) * 8;
                *reinterpret_cast<uint4*>(dst) = val;
              }
            }
          }
          __syncwarp();
          if (c0 + 16 < tl.width) prefetch_gu(tl, c0 + 16);
        } else {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj)
            stg_ptr[jj * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(v[jj]));
          __syncwarp();
          const int fb = tl.ft * kTileF + q * 32;
          if (fb < p.F) {
            for (int idx = lane; idx < 16 * 4; idx += 32) {
              const int rr = idx >> 2, ch = idx & 3;
              if (rr < nrows) {
                const uint4 val = *reinterpret_cast<const uint4*>(stg_ptr + rr * 32 + ch * 8);
                *reinterpret_cast<uint4*>(p.out + static_cast<int64_t>(tl.row0 + c0 + rr) * p.ldo +
                                          fb + ch * 8) = val;
              }
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_cluster(cluster_addr(acc_empty(pipes ? (it & 1) : 0), 0));
        else mbar_arrive(acc_empty(pipes ? (it & 1) : 0));
      }
    }
    // A staged chunk prefetched for a tile that was then abandoned lands
    // before the CTA can exit.
    if constexpr (kGuStaged) cp_async_wait<0>();
  }

  tc_fence_before();
  __syncwarp();
  // A pair frees its tensor memory only when the even CTA's MMAs, which write
  // both CTAs' accumulators, have drained and both epilogues are done.
  if constexpr (PAIR) cluster_sync_all(); else __syncthreads();
  tc_fence_after();
  if (warp == kIssuerWarp0) {
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, p.tmem_cols);
    else tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace

template <int MODE, int FMT, int EPI, int LANES, int PAIR, int DQW>
static cudaError_t launch_grouped_qgemm_t(const CUtensorMap& tb, const CUtensorMap& tw,
                                          const CUtensorMap& ts, const GemmArgs& p, int grid,
                                          size_t smem, cudaStream_t s) {
  auto k = grouped_qgemm_kernel<MODE, FMT, EPI, LANES, PAIR, DQW>;
  constexpr int kThreads = gemm_threads(DQW);
  // Raise the dynamic shared-memory limit once per (device, kernel) and, for
  // pairs, count the clusters that can be resident at once; later calls,
  // including ones under stream capture, skip both.
  static int set_for[64] = {0};
  static int max_pairs[64] = {0};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (set_for[dev] < static_cast<int>(smem)) {
    err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (err != cudaSuccess) return err;
    set_for[dev] = 227 * 1024;
  }
  if constexpr (PAIR) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (max_pairs[dev] == 0) {
      cfg.gridDim = dim3(2 * ((grid + 1) / 2));
      int n = 0;
      err = cudaOccupancyMaxActiveClusters(&n, k, &cfg);
      if (err != cudaSuccess) return err;
      if (n < 1) return cudaErrorInvalidConfiguration;
      max_pairs[dev] = n;
    }
    // Persistent pairs: at most as many as can be resident together.
    const int pairs = std::max(1, std::min((grid + 1) / 2, max_pairs[dev]));
    cfg.gridDim = dim3(2 * pairs);
    cfg.numAttrs = 2;
    err = cudaLaunchKernelEx(&cfg, k, tb, tw, ts, p);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
  } else {
    return launch_pdl(k, dim3(grid), dim3(kThreads), smem, s, tb, tw, ts, p);
  }
}

cudaError_t launch_grouped_qgemm(int mode, int fmt, int epi, int lanes, int dq_warps, bool pair,
                                 const CUtensorMap& tb, const CUtensorMap& tw,
                                 const CUtensorMap& ts, const GemmArgs& p, int grid, size_t smem,
                                 cudaStream_t s) {
  // Eight dequant warps only with two lanes (one warp per lane quarter) and
  // single CTAs.
  if (dq_warps != 16 && !(dq_warps == 8 && lanes == 2 && !pair)) return cudaErrorInvalidValue;
#define MOEQ_LANES(M_, F_, E_, P_)                                                               \
  if (dq_warps == 8) return launch_grouped_qgemm_t<M_, F_, E_, 2, 0, 8>(tb, tw, ts, p, grid, smem, s); \
  return lanes == 4 ? launch_grouped_qgemm_t<M_, F_, E_, 4, P_, 16>(tb, tw, ts, p, grid, smem, s) \
                    : launch_grouped_qgemm_t<M_, F_, E_, 2, P_, 16>(tb, tw, ts, p, grid, smem, s);
#define MOEQ_CASE(M_, F_, E_)                                                  \
  if (mode == M_ && fmt == F_ && epi == E_) {                                  \
    if (pair) { MOEQ_LANES(M_, F_, E_, 1) } else { MOEQ_LANES(M_, F_, E_, 0) } \
  }
#define MOEQ_CASE_SINGLE(M_, F_, E_) \
  if (mode == M_ && fmt == F_ && epi == E_ && !pair) { MOEQ_LANES(M_, F_, E_, 0) }
  if (lanes != 2 && lanes != 4) return cudaErrorInvalidValue;
  MOEQ_CASE(kModeFwd, MOE_W_INT4_G32_BF16, MOE_EPI_NONE)
  MOEQ_CASE(kModeFwd, MOE_W_INT4_G32_BF16, MOE_EPI_SWIGLU)
  MOEQ_CASE(kModeFwd, MOE_W_MXFP4_G32_E8M0, MOE_EPI_NONE)
  MOEQ_CASE(kModeFwd, MOE_W_MXFP4_G32_E8M0, MOE_EPI_SWIGLU)
  MOEQ_CASE_SINGLE(kModeBwd, MOE_W_INT4_G32_BF16, MOE_EPI_NONE)
  MOEQ_CASE_SINGLE(kModeBwd, MOE_W_INT4_G32_BF16, MOE_EPI_SWIGLU_BWD)
  MOEQ_CASE_SINGLE(kModeBwd, MOE_W_MXFP4_G32_E8M0, MOE_EPI_NONE)
  MOEQ_CASE_SINGLE(kModeBwd, MOE_W_MXFP4_G32_E8M0, MOE_EPI_SWIGLU_BWD)
  if (mode == kModeFwdW) {
    // one plan only: two lanes of eight dequant warps each, single CTAs
    if (pair || lanes != 2 || dq_warps != 16) return cudaErrorInvalidValue;
#define MOEQ_WIDE(F_, E_) \
    if (fmt == F_ && epi == E_) return launch_grouped_qgemm_t<kModeFwdW, F_, E_, 2, 0, 16>(tb, tw, ts, p, grid, smem, s);
    MOEQ_WIDE(MOE_W_INT4_G32_BF16, MOE_EPI_NONE)
    MOEQ_WIDE(MOE_W_INT4_G32_BF16, MOE_EPI_SWIGLU)
    MOEQ_WIDE(MOE_W_MXFP4_G32_E8M0, MOE_EPI_NONE)
    MOEQ_WIDE(MOE_W_MXFP4_G32_E8M0, MOE_EPI_SWIGLU)
#undef MOEQ_WIDE
    return cudaErrorInvalidValue;
  }
  MOEQ_CASE_SINGLE(kModeBwdT, MOE_W_INT4_G32_BF16, MOE_EPI_NONE)
  MOEQ_CASE_SINGLE(kModeBwdT, MOE_W_INT4_G32_BF16, MOE_EPI_SWIGLU_BWD)
  MOEQ_CASE_SINGLE(kModeBwdT, MOE_W_MXFP4_G32_E8M0, MOE_EPI_NONE)
  MOEQ_CASE_SINGLE(kModeBwdT, MOE_W_MXFP4_G32_E8M0, MOE_EPI_SWIGLU_BWD)
#undef MOEQ_CASE_SINGLE
#undef MOEQ_CASE
#undef MOEQ_LANES
  return cudaErrorInvalidValue;
}

uint32_t gemm_stage_bytes(int mode, int BN, int fmt, bool pair) {
  const uint32_t el = (fmt == MOE_W_INT4_G32_BF16) ? 2u : 1u;
  uint32_t b;
  if (mode == kModeFwdW)  // B 1 or 2 boxes of kWideHalf rows x 1 chunk, packed 128 rows x 32 B, scales 2 x 128
    b = (BN > kWideHalf ? 2u : 1u) * kWideHalf * 128u + 4096u + 256u * el;
  else if (mode != kModeBwd)   // B 2 chunks (BN / 2 rows in a pair), packed 128 rows x 64 B, scales 4 x 128
    b = static_cast<uint32_t>(pair ? BN / 2 : BN) * 256u + 8192u + 512u * el;
  else                    // B 1 chunk, A 16 KiB, packed 64 rows x 64 B, scales 4 x 64
    b = static_cast<uint32_t>(BN) * 128u + kABytes + 4096u + 256u * el;
  return (b + 1023u) & ~1023u;
}

uint32_t gemm_fixed_smem_bytes(int mode, int stages, int a_stages, int E) {
  // barriers (two per A stage reserved for halves), TMEM slot + abort flag
  // (16 B), warp totals, tile list, epilogue staging (4 blocks, 128-byte
  // aligned), the transpose scratch of kModeBwdT (16 dequant warps at most),
  // alignment slack
  return 8u * (2u * stages + 4u * a_stages + 5u) + 16u + 32u * 4u +
         static_cast<uint32_t>(E + 1) * 4u + 128u + 4u * kStageBytesEpi +
         (mode == kModeBwdT ? 16u * kScratchBytes : 0u) + 1024u;
}

}  // namespace moeq
