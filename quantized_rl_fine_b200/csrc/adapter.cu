// BF16 block-diagonal adapter on the activations (per expert, 32 x 32 blocks).
//
// Orbit issue #1: the trainable adapter is orthogonal fine-tuning applied on
// top of a quantized base that is never dequantized into storage. Its form
// here is one block-diagonal d x d matrix R_e per expert:
//   forward   x'[p][32b+j] = sum_i x[p][32b+i] * R[e][b][i][j]
//   backward  dx[p][32b+i] = sum_j dx'[p][32b+j] * R[e][b][i][j]
//             dR[e][b][i][j] = sum over rows p of expert e of x[p][32b+i] * dx'[p][32b+j]
// FP32 accumulation; dR is summed in ascending row order by one block per
// (expert, block) pair, so it is deterministic.
#include "launchers.cuh"
#include "common.cuh"

namespace moeq {

namespace {

constexpr int kRows = 64;   // rows per block of the apply kernel

__device__ __forceinline__ int expert_of_row(const int32_t* offsets, int E, int row) {
  int lo = 0, hi = E - 1;       // largest e with offsets[e] <= row
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= row) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// grid (ceil(M / 64), K / 32), 256 threads. TRANS = 0: x . R, 1: x . R^T.
template <int TRANS>
__global__ void __launch_bounds__(256)
adapter_apply_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ R,
                     const int32_t* __restrict__ offsets, int E, int M, int K,
                     __nv_bfloat16* __restrict__ out) {
  __shared__ float xs[kRows][33];
  __shared__ float rs[32][33];
  __shared__ int re[kRows];
  const int b = blockIdx.y;
  const int r0 = blockIdx.x * kRows;
  const int nb = K / 32;
  for (int i = threadIdx.x; i < kRows * 32; i += blockDim.x) {
    const int r = i >> 5, c = i & 31;
    xs[r][c] = (r0 + r < M) ? __bfloat162float(x[static_cast<int64_t>(r0 + r) * K + 32 * b + c]) : 0.0f;
  }
  if (threadIdx.x < kRows) re[threadIdx.x] = (r0 + threadIdx.x < M) ? expert_of_row(offsets, E, r0 + threadIdx.x) : -1;
  __syncthreads();
  const int j = threadIdx.x & 31;
  const int rsub = threadIdx.x >> 5;   // 0..7
  int r = 0;
  while (r < kRows && re[r] >= 0) {
    const int e = re[r];
    int rend = r;
    while (rend < kRows && re[rend] == e) ++rend;
    for (int i = threadIdx.x; i < 1024; i += blockDim.x) {
      const int a = i >> 5, c = i & 31;
      const float v = __bfloat162float(R[((static_cast<int64_t>(e) * nb + b) * 32 + a) * 32 + c]);
      if (TRANS) rs[c][a] = v; else rs[a][c] = v;
    }
    __syncthreads();
    for (int rr = r + rsub; rr < rend; rr += 8) {
      float acc = 0.0f;
#pragma unroll
      for (int i = 0; i < 32; ++i) acc = fmaf(xs[rr][i], rs[i][j], acc);
      out[static_cast<int64_t>(r0 + rr) * K + 32 * b + j] = __float2bfloat16_rn(acc);
    }
    __syncthreads();
    r = rend;
  }
}

// grid (E, K / 32), 256 threads: dR[e][b] over the rows of expert e.
__global__ void __launch_bounds__(256)
adapter_grad_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ dxp,
                    const int32_t* __restrict__ offsets, int K, float* __restrict__ dR) {
  __shared__ float xs[kRows][33];
  __shared__ float gs[kRows][33];
  const int e = blockIdx.x, b = blockIdx.y;
  const int nb = K / 32;
  const int p0 = offsets[e], p1 = offsets[e + 1];
  const int i = threadIdx.x >> 3;          // 0..31
  const int j0 = (threadIdx.x & 7) * 4;    // 0..28
  float acc[4] = {0, 0, 0, 0};
  for (int c0 = p0; c0 < p1; c0 += kRows) {
    const int n = min(kRows, p1 - c0);
    for (int u = threadIdx.x; u < kRows * 32; u += blockDim.x) {
      const int r = u >> 5, c = u & 31;
      const bool in = r < n;
      const int64_t gi = static_cast<int64_t>(c0 + r) * K + 32 * b + c;
      xs[r][c] = in ? __bfloat162float(x[gi]) : 0.0f;
      gs[r][c] = in ? __bfloat162float(dxp[gi]) : 0.0f;
    }
    __syncthreads();
    for (int r = 0; r < n; ++r) {
      const float xv = xs[r][i];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = fmaf(xv, gs[r][j0 + q], acc[q]);
    }
    __syncthreads();
  }
  float* dst = dR + ((static_cast<int64_t>(e) * nb + b) * 32 + i) * 32 + j0;
#pragma unroll
  for (int q = 0; q < 4; ++q) dst[q] = acc[q];
}

}  // namespace

cudaError_t launch_adapter_apply(const void* x, const void* R, const int32_t* offsets, int E,
                                 int M, int K, void* out, bool transpose, cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  dim3 grid((M + kRows - 1) / kRows, K / 32);
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
  dim3 grid(E, K / 32);
  adapter_grad_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x),
                                           static_cast<const __nv_bfloat16*>(dxp), offsets, K, dR);
  return cudaGetLastError();
}

}  // namespace moeq
