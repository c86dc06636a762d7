// BF16 block-diagonal adapter on the activations (per expert, 32 x 32 blocks).
//
// Orbit issue #1: the trainable adapter is orthogonal fine-tuning applied on
// top of a quantized base that is never dequantized into storage. Its form
// here is one block-diagonal d x d matrix R_e per expert:
//   forward   x'[p][32b+j] = sum_i x[p][32b+i] * R[e][b][i][j]
//   backward  dx[p][32b+i] = sum_j dx'[p][32b+j] * R[e][b][i][j]
//             dR[e][b][i][j] = sum over rows p of expert e of x[p][32b+i] * dx'[p][32b+j]
// FP32 accumulation; dR is summed in ascending row order by one warp per
// (expert, block) pair, so it is deterministic.
#include "launchers.cuh"
#include "common.cuh"

namespace moeq {

namespace {

constexpr int kBlocksPerCta = 8;   // 32-column blocks per CTA (one warp each)

__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    f[2 * q] = __uint_as_float(w[q] << 16);
    f[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
  }
}

constexpr int kApplyRowGroups = 2;   // 32-row groups per warp of the apply kernel

// Expert of row `row` (the same row in every lane): the largest e with
// offsets[e] <= row, which is the number of boundaries offsets[1..E-1] at or
// below the row (offsets are nondecreasing and offsets[E] = M > row); the
// lanes count them in parallel.
__device__ __forceinline__ int warp_expert_of_row(const int32_t* offsets, int E, int row, int lane) {
  int cnt = 0;
  for (int e = 1 + lane; e < E; e += 32) cnt += (__ldg(offsets + e) <= row) ? 1 : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  return cnt;
}

// grid (ceil(M / 64), ceil(K / 256)), 256 threads. Warp w covers column block
// b = 8 * blockIdx.y + w for 64 rows, 32 at a time (one row per lane): the lane
// keeps its row's 32 inputs in registers and reads its expert's 32 x 32 block
// from shared memory (a broadcast when the warp's rows share an expert, the
// common case since rows are sorted by expert); the block is staged again only
// when the expert changes. TRANS = 0: x . R, 1: x . R^T.
template <int TRANS>
__global__ void __launch_bounds__(256)
adapter_apply_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ R,
                     const int32_t* __restrict__ offsets, int E, int M, int K,
                     __nv_bfloat16* __restrict__ out) {
  __shared__ __align__(16) float rs[kBlocksPerCta][32][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y * kBlocksPerCta + warp;
  const int nb = K / 32;
  if (b >= nb) return;                   // warp-uniform; the warps never sync with each other
  const int row_base = blockIdx.x * 32 * kApplyRowGroups;
  if (row_base >= M) return;
  int e = warp_expert_of_row(offsets, E, row_base, lane);   // expert of the warp's first row
  int staged = -1;                       // expert whose block is in rs[warp]
  for (int g = 0; g < kApplyRowGroups; ++g) {
    const int row = row_base + g * 32 + lane;
    const bool valid = row < M;
    if (__ballot_sync(0xffffffffu, valid) == 0) break;
    // this lane's expert: step forward from the warp's first expert
    int my_e = -1;
    if (valid) {
      my_e = e;
      while (my_e + 1 < E && __ldg(offsets + my_e + 1) <= row) ++my_e;
    }
    float xv[32];
    if (valid) {
      const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(row) * K + 32 * b);
#pragma unroll
      for (int v = 0; v < 4; ++v) unpack_bf16x8(__ldg(src + v), xv + 8 * v);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) xv[i] = 0.0f;
    }
    float acc[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] = 0.0f;
    int pending = my_e;
    while (true) {
      const unsigned live = __ballot_sync(0xffffffffu, pending >= 0);
      if (live == 0) break;
      const int cur = __shfl_sync(0xffffffffu, pending, __ffs(live) - 1);
      if (cur != staged) {
        // stage R[cur][b] (TRANS: its transpose) as rs[warp][i][j] = coefficient
        // of input i in output j; lane writes column `lane` of row i (no bank conflict)
        __syncwarp();
        const __nv_bfloat16* Rb = R + ((static_cast<int64_t>(cur) * nb + b) * 32) * 32;
#pragma unroll 4
        for (int i = 0; i < 32; ++i)
          rs[warp][i][lane] = __bfloat162float(TRANS ? Rb[lane * 32 + i] : Rb[i * 32 + lane]);
        __syncwarp();
        staged = cur;
      }
      if (pending == cur) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float xi = xv[i];
          const float4* r4 = reinterpret_cast<const float4*>(&rs[warp][i][0]);
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const float4 c = r4[m];
            acc[4 * m] = fmaf(xi, c.x, acc[4 * m]);
            acc[4 * m + 1] = fmaf(xi, c.y, acc[4 * m + 1]);
            acc[4 * m + 2] = fmaf(xi, c.z, acc[4 * m + 2]);
            acc[4 * m + 3] = fmaf(xi, c.w, acc[4 * m + 3]);
          }
        }
        pending = -1;
      }
    }
    if (valid) {
      uint4* dst = reinterpret_cast<uint4*>(out + static_cast<int64_t>(row) * K + 32 * b);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint4 o;
        o.x = pack_bf16x2(acc[8 * v + 0], acc[8 * v + 1]);
        o.y = pack_bf16x2(acc[8 * v + 2], acc[8 * v + 3]);
        o.z = pack_bf16x2(acc[8 * v + 4], acc[8 * v + 5]);
        o.w = pack_bf16x2(acc[8 * v + 6], acc[8 * v + 7]);
        dst[v] = o;
      }
    }
    // the next group starts from the last expert of this one
    e = __shfl_sync(0xffffffffu, valid ? my_e : -1, 31);
    if (e < 0) break;
  }
}

constexpr int kGradRows = 16;   // rows staged per step of the gradient kernel

// grid (E, ceil(K / 256)), 256 threads: dR[e][b] for the 8 column blocks b of this
// CTA (one warp each) over the rows of expert e, in ascending row order.
// Lane i owns row i of the 32 x 32 result (32 accumulators).
__global__ void __launch_bounds__(256)
adapter_grad_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ dxp,
                    const int32_t* __restrict__ offsets, int K, float* __restrict__ dR) {
  __shared__ float xs[kBlocksPerCta][kGradRows][33];
  __shared__ __align__(16) float gs[kBlocksPerCta][kGradRows][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x;
  const int b = blockIdx.y * kBlocksPerCta + warp;
  const int nb = K / 32;
  if (b >= nb) return;                   // warp-uniform; the warps never sync with each other
  const int p0 = offsets[e], p1 = offsets[e + 1];
  float acc[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) acc[j] = 0.0f;
  for (int c0 = p0; c0 < p1; c0 += kGradRows) {
    const int n = min(kGradRows, p1 - c0);
    // lane r < n loads row c0 + r of both operands (64 bytes each)
    if (lane < n) {
      const int64_t gi = static_cast<int64_t>(c0 + lane) * K + 32 * b;
      const uint4* xsrc = reinterpret_cast<const uint4*>(x + gi);
      const uint4* gsrc = reinterpret_cast<const uint4*>(dxp + gi);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        float f[8];
        unpack_bf16x8(__ldg(xsrc + v), f);
#pragma unroll
        for (int q = 0; q < 8; ++q) xs[warp][lane][8 * v + q] = f[q];
        unpack_bf16x8(__ldg(gsrc + v), f);
#pragma unroll
        for (int q = 0; q < 8; ++q) gs[warp][lane][8 * v + q] = f[q];
      }
    }
    __syncwarp();
    for (int r = 0; r < n; ++r) {
      const float xi = xs[warp][r][lane];
      const float4* g4 = reinterpret_cast<const float4*>(&gs[warp][r][0]);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float4 c = g4[m];
        acc[4 * m] = fmaf(xi, c.x, acc[4 * m]);
        acc[4 * m + 1] = fmaf(xi, c.y, acc[4 * m + 1]);
        acc[4 * m + 2] = fmaf(xi, c.z, acc[4 * m + 2]);
        acc[4 * m + 3] = fmaf(xi, c.w, acc[4 * m + 3]);
      }
    }
    __syncwarp();
  }
  float4* dst = reinterpret_cast<float4*>(dR + ((static_cast<int64_t>(e) * nb + b) * 32 + lane) * 32);
#pragma unroll
  for (int v = 0; v < 8; ++v) dst[v] = make_float4(acc[4 * v], acc[4 * v + 1], acc[4 * v + 2], acc[4 * v + 3]);
}

}  // namespace

cudaError_t launch_adapter_apply(const void* x, const void* R, const int32_t* offsets, int E,
                                 int M, int K, void* out, bool transpose, cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  const int nb = K / 32;
  dim3 grid((M + 32 * kApplyRowGroups - 1) / (32 * kApplyRowGroups),
            (nb + kBlocksPerCta - 1) / kBlocksPerCta);
  if (transpose)
    adapter_apply_kernel<1><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x),
                                                 static_cast<const __nv_bfloat16*>(R), offsets, E,
                                                 M, K, static_cast<__nv_bfloat16*>(out));
  else
    adapter_apply_kernel<0><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x),
                                                 static_cast<const __nv_bfloat16*>(R), offsets, E,
                                                 M, K, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

cudaError_t launch_adapter_grad(const void* x, const void* dxp, const int32_t* offsets, int E,
                                int K, float* dR, cudaStream_t s) {
  const int nb = K / 32;
  dim3 grid(E, (nb + kBlocksPerCta - 1) / kBlocksPerCta);
  adapter_grad_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x),
                                           static_cast<const __nv_bfloat16*>(dxp), offsets, K, dR);
  return cudaGetLastError();
}

}  // namespace moeq
