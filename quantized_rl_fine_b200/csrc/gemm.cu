// Grouped low-bit GEMM over the active experts (forward and dX backward).
//
// Orbit article, "Active-expert-chunked dequantization": the experts chosen
// by the router are taken in fixed-size chunks, their 4-bit weights are
// dequantized and a grouped GEMM runs over them. Here the dequantization
// happens inside the GEMM kernel, tile by tile, into shared memory; no BF16
// weight is ever written to global memory. The DeepSeek-V4 paragraph of the
// same section gives the backward form: only the activation gradient is
// formed, the frozen base gets none.
//
// One persistent CTA per SM walks a device-built tile list (active experts in
// ascending id, which is chunk order; inside an expert, feature tile major and
// token tile minor). A tile is 128 output features x BN token rows (BN a
// multiple of 16, <= 256), accumulated in FP32 in tensor memory by
// tcgen05.mma with the dequantized weight as operand A (M = 128) and the
// token rows as operand B (N = BN):
//
//   forward  D[f, t] = sum_k W[e][f][k] * a[t][k]     (A K-major)
//   backward D[f, t] = sum_n W[e][n][f] * dout[t][n]  (A MN-major)
//
// Warp roles (384 threads): warp 0 lane 0 issues TMA loads (token rows,
// packed weights, group scales) into a ring of stages; warp 1 owns tensor
// memory and lane 0 issues the MMAs; warps 4-7 dequantize each stage into a
// 128B-swizzled BF16 tile; warps 8-11 drain the double-buffered accumulator
// (epilogue: plain, SwiGLU, SwiGLU backward) while the next tile runs.
// Every wait is bounded; on a timeout the kernel records a device error,
// lets its in-flight copies and MMAs finish (again bounded), frees tensor
// memory and returns.
#include "common.cuh"
#include "dequant.cuh"
#include "gemm.cuh"

namespace moeq {

namespace {

constexpr int kThreads = kGemmThreads;
constexpr int kStageK = 64;            // reduction elements per pipeline stage
constexpr int kTileF = 128;            // output features per tile (MMA M)
constexpr uint32_t kABytes = kTileF * kStageK * 2;   // 16 KiB dequantized tile
constexpr uint32_t kWqBytes = 4096;    // packed weights of one stage

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
  const long long budget = g_wait_budget;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > budget) {
      raise_device_error(MOE_DEVERR_WAIT_TIMEOUT);
      return;
    }
  }
}

struct Tile {
  int e, ft, row0, row_end;
};

// Tile t of the tile list: active index a with tile_start[a] <= t (shared
// memory), then feature tile major, token tile minor inside the expert.
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
  const int nrt = (seg1 - seg0 + p.BN - 1) / p.BN;
  r.ft = local / nrt;
  r.row0 = seg0 + (local - r.ft * nrt) * p.BN;
  r.row_end = seg1;
  return r;
}

// Every CTA builds the tile list of the launch in shared memory:
// tile_start[a] = sum over active experts a' < a of n_ftiles * ceil(m_e / BN),
// tile_start[A] = total. Offsets that do not describe M rows give an empty
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
    local += p.n_ftiles * ((m + p.BN - 1) / p.BN);
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
    run += p.n_ftiles * ((m + p.BN - 1) / p.BN);
  }
  if (tid == nthr - 1) {
    int total = 0;
    for (int i = 0; i < nw; ++i) total += warp_tot[i];
    tile_start[A] = total;
  }
  __syncthreads();
  return A;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

template <int MODE, int FMT, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
grouped_qgemm_kernel(const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_wq,
                     const __grid_constant__ CUtensorMap tm_sc, const GemmArgs p) {
  constexpr uint32_t kScEl = (FMT == MOE_W_INT4_G32_BF16) ? 2 : 1;
  constexpr uint32_t kScBytes = 256 * kScEl;   // scales of one stage
  constexpr bool kGluRows = (MODE == kModeFwd && EPI == MOE_EPI_SWIGLU);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const int S = p.stages;
  const uint32_t stage_bytes = p.stage_bytes;
  const uint32_t b_bytes = static_cast<uint32_t>(p.BN) * 128u;
  // One stage: [A 16 KiB][B BN*128][packed 4 KiB][scales 256 or 512 B]
  auto A_at = [&](int s) { return base + s * stage_bytes; };
  auto B_at = [&](int s) { return base + s * stage_bytes + kABytes; };
  auto W_at = [&](int s) { return base + s * stage_bytes + kABytes + b_bytes; };
  auto S_at = [&](int s) { return base + s * stage_bytes + kABytes + b_bytes + kWqBytes; };
  const uint32_t bars = base + S * stage_bytes;
  auto full_tma = [&](int s) { return bars + 8u * s; };
  auto full_a = [&](int s) { return bars + 8u * (S + s); };
  auto empty = [&](int s) { return bars + 8u * (2 * S + s); };
  auto acc_full = [&](int b) { return bars + 8u * (3 * S + b); };
  auto acc_empty = [&](int b) { return bars + 8u * (3 * S + 2 + b); };
  const uint32_t drain_bar = bars + 8u * (3 * S + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + S * stage_bytes + 8u * (3 * S + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* warp_tot = reinterpret_cast<int32_t*>(tmem_slot + 4);          // [32]
  int32_t* tile_start = warp_tot + 32;                                      // [E + 1]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_tma(s), 1);
      mbar_init(full_a(s), 4);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full(b), 1);
      mbar_init(acc_empty(b), 4);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_wq);
    tma_prefetch_desc(&tm_sc);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), p.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int A = build_tile_list(p, tile_start, warp_tot);
  const int total = tile_start[A];
  const int nkb = p.R / kStageK;
  const int N = p.N, K = p.K;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t keep = l2_policy_evict_last();
      const uint64_t stream_once = l2_policy_evict_first();
      const uint32_t tx = b_bytes + kWqBytes + kScBytes;
      int st = 0;
      uint32_t ph = 0;
      long long fills = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile tl = decode_tile(p, tile_start, A, t);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(empty(st), ph ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(full_tma(st), tx);
          tma_load_2d_hint(B_at(st), &tm_b, full_tma(st), kb * kStageK, tl.row0, keep);
          if constexpr (MODE == kModeFwd) {
            int fa, fb;
            if constexpr (EPI == MOE_EPI_SWIGLU) {
              fa = tl.ft * 64;            // gate rows
              fb = N / 2 + tl.ft * 64;    // the matching up rows
            } else {
              fa = tl.ft * kTileF;
              fb = fa + 64;
            }
            const int g0 = tl.e * (K / 32) + kb * 2;
            tma_load_2d_hint(W_at(st), &tm_wq, full_tma(st), kb * 32, tl.e * N + fa, stream_once);
            tma_load_2d_hint(W_at(st) + 2048, &tm_wq, full_tma(st), kb * 32, tl.e * N + fb,
                             stream_once);
            tma_load_2d_hint(S_at(st), &tm_sc, full_tma(st), fa, g0, stream_once);
            tma_load_2d_hint(S_at(st) + 128 * kScEl, &tm_sc, full_tma(st), fb, g0, stream_once);
          } else {
            tma_load_2d_hint(W_at(st), &tm_wq, full_tma(st), tl.ft * 64, tl.e * N + kb * kStageK,
                             stream_once);
            tma_load_2d_hint(S_at(st), &tm_sc, full_tma(st), kb * kStageK,
                             tl.e * (K / 32) + tl.ft * 4, stream_once);
          }
          ++fills;
          if (++st == S) { st = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        // Let every issued copy land before the CTA can exit.
        const long long first = fills > S ? fills - S : 0;
        for (long long f = first; f < fills; ++f)
          mbar_drain(full_tma(static_cast<int>(f % S)), static_cast<uint32_t>((f / S) & 1));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kTileF, p.BN, MODE == kModeBwd ? 1u : 0u, 0u);
      int st = 0;
      uint32_t ph = 0;
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait(acc_empty(buf), aph ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * p.acc_cols);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(full_tma(st), ph, abort_flag)) { ok = false; break; }
          if (!mbar_wait(full_a(st), ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kStageK / 16; ++kk) {
            uint64_t adesc;
            if constexpr (MODE == kModeFwd) {
              adesc = smem_desc_sw128(A_at(st) + kk * 32, 16, 1024);
            } else {
              adesc = smem_desc_sw128(A_at(st) + kk * 2048, 8192, 1024);
            }
            const uint64_t bdesc = smem_desc_sw128(B_at(st) + kk * 32, 16, 1024);
            mma_bf16_ss(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit(empty(st));
          if (++st == S) { st = 0; ph ^= 1u; }
        }
        if (ok) mma_commit(acc_full(buf));
      }
      // All MMAs of this CTA done before tensor memory is released.
      mma_commit(drain_bar);
      mbar_drain(drain_bar, 0);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ dequantizers
    const int i = threadIdx.x - 128;   // 0..127
    // Forward: thread i writes A row i (one output feature). With SwiGLU the
    // rows interleave gate and up: row 2j <- gate row j (packed row j), row
    // 2j+1 <- up row j (packed row 64 + j).
    const int src = kGluRows ? ((i & 1) ? 64 + (i >> 1) : (i >> 1)) : i;
    int st = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(full_tma(st), ph, abort_flag)) { ok = false; break; }
        const uint32_t wq = W_at(st);
        const uint32_t sc = S_at(st);
        const uint32_t a_st = A_at(st);
        if constexpr (MODE == kModeFwd) {
          // Packed rows are 32 bytes with the TMA 32-byte swizzle (16-byte chunk
          // index ^= row bit 2). Scales: two boxes [2 groups][64 rows].
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint4 pk = lds128(wq + src * 32 + ((h ^ ((src >> 2) & 1)) << 4));
            const uint32_t soff = (src >> 6) * 128 + h * 64 + (src & 63);
            const uint32_t sbits = (FMT == MOE_W_INT4_G32_BF16) ? lds_u16(sc + soff * 2)
                                                                : lds_u8(sc + soff);
            uint32_t o[16];
            dequant32<FMT>(pk, sbits, o);
            // K-major, 128B swizzle: row i at (i/8)*1024 + (i%8)*128, chunk c ^ (i%8).
            const uint32_t rowb = a_st + (i >> 3) * 1024 + (i & 7) * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint32_t chunk = (h * 4 + c) ^ (i & 7);
              sts128(rowb + (chunk << 4), o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
            }
          }
        } else {
          // Thread = (reduction row r, feature half hf): 64 features = 2 groups.
          // Packed rows are 64 bytes with the TMA 64-byte swizzle (chunk ^= (r >> 1) & 3).
          // Scales: one box [4 groups][64 rows].
          const int r = i & 63;
          const int hf = i >> 6;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int c = 2 * hf + j;
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
              const uint32_t chunk = (4 * j + w) ^ (r & 7);
              sts128(rowb + (chunk << 4), o[4 * w], o[4 * w + 1], o[4 * w + 2], o[4 * w + 3]);
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(full_a(st));
        if (++st == S) { st = 0; ph ^= 1u; }
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int fr = q * 32 + lane;           // accumulator row = tile feature
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const Tile tl = decode_tile(p, tile_start, A, t);
      const int buf = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      if (!mbar_wait(acc_full(buf), aph, abort_flag)) break;
      tc_fence_after();
      const uint32_t tcol = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                            static_cast<uint32_t>(buf * p.acc_cols);
      for (int c0 = 0; c0 < p.BN; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tcol + c0, v);
        tmem_wait_ld();
        if constexpr (kGluRows) {
          // Even rows hold gate values, odd rows the up values of the same feature.
          const int fcol = tl.ft * 64 + (fr >> 1);
          const bool is_gate = (lane & 1) == 0;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float mine = __uint_as_float(v[j]);
            const float other = __shfl_xor_sync(0xffffffffu, mine, 1);
            const int c = c0 + j;
            const int row = tl.row0 + c;
            if (c < p.BN && row < tl.row_end) {
              const int64_t r64 = static_cast<int64_t>(row);
              if (is_gate) {
                p.out[r64 * p.ldo + fcol] = __float2bfloat16_rn(silu_f(mine) * other);
                if (p.saved) p.saved[r64 * N + fcol] = __float2bfloat16_rn(mine);
              } else if (p.saved) {
                p.saved[r64 * N + N / 2 + fcol] = __float2bfloat16_rn(mine);
              }
            }
          }
        } else if constexpr (MODE == kModeBwd && EPI == MOE_EPI_SWIGLU_BWD) {
          const int f = tl.ft * kTileF + fr;      // feature of dh (< K)
          if (f < p.F) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int c = c0 + j;
              const int row = tl.row0 + c;
              if (c < p.BN && row < tl.row_end) {
                const int64_t rb = static_cast<int64_t>(row) * (2 * K);
                const float g = __bfloat162float(p.saved[rb + f]);
                const float u = __bfloat162float(p.saved[rb + K + f]);
                const float dh = __uint_as_float(v[j]);
                const float s = 1.0f / (1.0f + expf(-g));
                p.out[rb + f] = __float2bfloat16_rn(dh * u * s * (1.0f + g * (1.0f - s)));
                p.out[rb + K + f] = __float2bfloat16_rn(dh * g * s);
              }
            }
          }
        } else {
          const int f = tl.ft * kTileF + fr;
          if (f < p.F) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int c = c0 + j;
              const int row = tl.row0 + c;
              if (c < p.BN && row < tl.row_end)
                p.out[static_cast<int64_t>(row) * p.ldo + f] =
                    __float2bfloat16_rn(__uint_as_float(v[j]));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty(buf));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, p.tmem_cols);
}

}  // namespace

template <int MODE, int FMT, int EPI>
static cudaError_t launch_grouped_qgemm_t(const CUtensorMap& tb, const CUtensorMap& tw,
                                          const CUtensorMap& ts, const GemmArgs& p, int grid,
                                          size_t smem, cudaStream_t s) {
  auto k = grouped_qgemm_kernel<MODE, FMT, EPI>;
  // Raise the dynamic shared-memory limit once per (device, kernel); later
  // calls, including ones under stream capture, skip it.
  static int set_for[64] = {0};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (set_for[dev] < static_cast<int>(smem)) {
    err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (err != cudaSuccess) return err;
    set_for[dev] = 227 * 1024;
  }
  k<<<grid, kThreads, smem, s>>>(tb, tw, ts, p);
  return cudaGetLastError();
}

cudaError_t launch_grouped_qgemm(int mode, int fmt, int epi, const CUtensorMap& tb,
                                 const CUtensorMap& tw, const CUtensorMap& ts, const GemmArgs& p,
                                 int grid, size_t smem, cudaStream_t s) {
#define MOEQ_CASE(M_, F_, E_)                                               \
  if (mode == M_ && fmt == F_ && epi == E_)                                 \
    return launch_grouped_qgemm_t<M_, F_, E_>(tb, tw, ts, p, grid, smem, s);
  MOEQ_CASE(kModeFwd, MOE_W_INT4_G32_BF16, MOE_EPI_NONE)
  MOEQ_CASE(kModeFwd, MOE_W_INT4_G32_BF16, MOE_EPI_SWIGLU)
  MOEQ_CASE(kModeFwd, MOE_W_MXFP4_G32_E8M0, MOE_EPI_NONE)
  MOEQ_CASE(kModeFwd, MOE_W_MXFP4_G32_E8M0, MOE_EPI_SWIGLU)
  MOEQ_CASE(kModeBwd, MOE_W_INT4_G32_BF16, MOE_EPI_NONE)
  MOEQ_CASE(kModeBwd, MOE_W_INT4_G32_BF16, MOE_EPI_SWIGLU_BWD)
  MOEQ_CASE(kModeBwd, MOE_W_MXFP4_G32_E8M0, MOE_EPI_NONE)
  MOEQ_CASE(kModeBwd, MOE_W_MXFP4_G32_E8M0, MOE_EPI_SWIGLU_BWD)
#undef MOEQ_CASE
  return cudaErrorInvalidValue;
}

uint32_t gemm_stage_bytes(int BN, int fmt) {
  const uint32_t sc = 256u * (fmt == MOE_W_INT4_G32_BF16 ? 2u : 1u);
  const uint32_t b = kABytes + static_cast<uint32_t>(BN) * 128u + kWqBytes + sc;
  return (b + 1023u) & ~1023u;
}

uint32_t gemm_fixed_smem_bytes(int stages, int E) {
  // barriers, TMEM slot + abort flag (16 B), warp totals, tile list, alignment slack
  return 8u * (3u * stages + 5u) + 16u + 32u * 4u + static_cast<uint32_t>(E + 1) * 4u + 1024u;
}

}  // namespace moeq
