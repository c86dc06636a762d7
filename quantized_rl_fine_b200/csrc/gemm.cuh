// Host-side interface of the grouped low-bit GEMM kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moeq {

constexpr int kModeFwd = 0;    // D[f, t] = sum_k W[e][f][k] a[t][k]
constexpr int kModeBwd = 1;    // D[f, t] = sum_n W[e][n][f] dout[t][n], A in shared memory
constexpr int kModeBwdT = 2;   // the same, A in tensor memory (128-wide fills, transposed dequant)
constexpr int kModeFwdW = 3;   // forward with wide token tiles (up to 384 rows: two MMAs per
                               // K step), 64-wide fills, one accumulator
__host__ __device__ constexpr bool gemm_is_fwd(int mode) { return mode == kModeFwd || mode == kModeFwdW; }
constexpr int kWideHalfRows = 192;   // kModeFwdW: token rows of a tile's first MMA (and TMA box)

struct GemmArgs {
  const int32_t* offsets;     // [E+1] expert row offsets
  const int32_t* active;      // [E] active experts (ascending)
  const int32_t* num_active;  // [1] number of active experts
  int32_t E, N, K;            // weight stack dims, W[e] is [N][K]
  int32_t M;                  // rows of a / dout / out
  int32_t BN;                 // token rows per tile (multiple of 16, of 32 for pairs; <= 256)
  int32_t n_ftiles;           // feature tiles per expert (pairs: pair tiles of 2 feature tiles)
  int32_t n_issuers;          // MMA-issuing warps (1..kMaxIssuers), each with a partial accumulator
  int32_t acc_cols;           // TMEM columns per partial accumulator (>= BN, multiple of 32)
  int32_t tmem_cols;          // TMEM columns allocated (power of two, >= 2 * acc_cols)
  int32_t F;                  // output features (fwd: N or N/2 with SwiGLU; bwd: K)
  int32_t R;                  // reduction length (fwd: K; bwd: N)
  int32_t stages;             // shared-memory fills in flight (multiple of the lane count)
  int32_t a_stages;           // A stages (in tensor memory; shared-memory backward: = stages);
                              // multiple of the lane count
  uint32_t stage_bytes;       // bytes of one stage (1 KiB multiple)
  int32_t pipes;              // 1: two tile pipelines (two issuers, each accumulating whole tiles)
  int32_t a_halves;           // forward: 1 = each A stage handed over in two 64-wide halves
  int32_t split_even;         // 1: an expert's token tiles have equal widths; 0: BN-row tiles
                              // and a shorter last one
  int32_t m_lo, m_hi;         // only experts with m_lo <= rows <= m_hi get tiles in this launch
  __nv_bfloat16* out;         // [M][ldo]
  int64_t ldo;
  __nv_bfloat16* saved;       // fwd SwiGLU: written [M][N]; bwd SwiGLU: read [M][2K]
  // Forward with gathered token rows: row p of the GEMM input is
  // b_src[b_rows[p]] ([*][R] BF16); NULL: the rows come from the tensor map.
  const int32_t* b_rows;
  const __nv_bfloat16* b_src;
};

// pair: forward only; a cluster of two CTAs per 256 output features with
// M = 256 MMAs (BN a multiple of 32, an even number of feature tiles); the
// grid is clamped to the pairs that can be resident together.
cudaError_t launch_grouped_qgemm(int mode, int fmt, int epi, int lanes, int dq_warps, bool pair,
                                 const CUtensorMap& tb, const CUtensorMap& tw,
                                 const CUtensorMap& ts, const GemmArgs& p, int grid, size_t smem,
                                 cudaStream_t s);
uint32_t gemm_stage_bytes(int mode, int BN, int fmt, bool pair);
uint32_t gemm_fixed_smem_bytes(int mode, int stages, int a_stages, int E);
// Warp roles, in order: kProdWarps TMA producers, up to kMaxIssuers
// MMA-issuing warps, kDqWarps dequant warps split into LANES groups (LANES is a
// kernel template parameter, 2 or 4), one epilogue warpgroup. Fill f (the
// CTA's f-th 128-wide reduction step, counted across tiles) belongs to
// pipeline lane f % LANES (its dequant group), to producer f % kProdWarps and
// to issuer f % n_issuers. The shared-memory ring and the tensor-memory A ring
// have a multiple of LANES stages (LANES is a multiple of both other counts),
// so each stage is waited on by exactly one member of each role, which sees
// every phase of the stage's barriers: a phase-parity wait can then never
// mistake a phase two behind for the one it waits for.
// The number of dequant warps (16, or 8 with two lanes) is a kernel template
// parameter; the epilogue warpgroup follows them.
constexpr int kProdWarps = 2;
constexpr int kMaxIssuers = 2;
constexpr int kIssuerWarp0 = kProdWarps;
constexpr int kDqWarp0 = kIssuerWarp0 + kMaxIssuers;
constexpr int gemm_threads(int dq_warps) { return 32 * (kDqWarp0 + dq_warps + 4); }

}  // namespace moeq
