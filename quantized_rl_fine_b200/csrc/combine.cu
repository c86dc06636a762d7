// Unpermute + gate-weighted combine of the per-slot rows, and its backward
// (gate-scaled scatter of the upstream gradient to the per-slot rows).
// The gates are applied here rather than inside the GEMM epilogue.
//
// One warp per token; each lane moves 16-byte slices (8 BF16) of the rows,
// so every row access is a fully coalesced 512-byte warp transaction.
#include "launchers.cuh"
#include "common.cuh"

namespace moeq {

namespace {

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// BF16 nearest-even of the exact product g * x (x a BF16 value). The FP32
// product can land exactly on a BF16 halfway point while the exact product
// does not; the FMA residual decides that case, so the result has one rounding.
__device__ __forceinline__ uint32_t bf16_of_product(float g, float x) {
  float p = g * x;
  const uint32_t pb = __float_as_uint(p);
  if ((pb & 0xFFFFu) == 0x8000u) {
    const float r = fmaf(g, x, -p);
    if (r != 0.0f) {
      const bool up = (r > 0.0f) == (p > 0.0f);   // exact magnitude above |p|
      p = __uint_as_float(up ? pb + 1u : pb - 1u);
    }
  }
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(p)));
}

__global__ void combine_kernel(const uint4* __restrict__ rows, const int32_t* __restrict__ inv_perm,
                               const float* __restrict__ gates, int T, int k, int64_t dvec,
                               uint4* __restrict__ out) {
  grid_dependency_wait();
  grid_dependents_launch();
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  int32_t idx[32];
  float g[32];
  for (int j = 0; j < k; ++j) {
    idx[j] = inv_perm[static_cast<int64_t>(t) * k + j];
    g[j] = gates ? gates[static_cast<int64_t>(t) * k + j] : 1.0f;
  }
  for (int64_t c = lane; c < dvec; c += 32) {
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j = 0; j < k; ++j) {
      float f[8];
      unpack8(rows[static_cast<int64_t>(idx[j]) * dvec + c], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(g[j], f[i], acc[i]);
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    out[static_cast<int64_t>(t) * dvec + c] = o;
  }
}

__global__ void scatter_kernel(const uint4* __restrict__ rows, const int32_t* __restrict__ inv_perm,
                               const float* __restrict__ gates, int T, int k, int64_t dvec,
                               uint4* __restrict__ out) {
  grid_dependency_wait();
  grid_dependents_launch();
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  for (int j = 0; j < k; ++j) {
    const int64_t p = inv_perm[static_cast<int64_t>(t) * k + j];
    const float g = gates ? gates[static_cast<int64_t>(t) * k + j] : 1.0f;
    for (int64_t c = lane; c < dvec; c += 32) {
      float f[8];
      unpack8(rows[static_cast<int64_t>(t) * dvec + c], f);
      uint32_t h[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) h[i] = bf16_of_product(g, f[i]);
      uint4 o;
      o.x = h[0] | (h[1] << 16);
      o.y = h[2] | (h[3] << 16);
      o.z = h[4] | (h[5] << 16);
      o.w = h[6] | (h[7] << 16);
      out[p * dvec + c] = o;
    }
  }
}

}  // namespace

cudaError_t launch_combine(const void* rows, const int32_t* inv_perm, const float* gates, int T,
                           int k, int64_t D, void* out, int mode, cudaStream_t s) {
  const int warps = 8;
  const int blocks = (T + warps - 1) / warps;
  return launch_pdl(mode == 0 ? combine_kernel : scatter_kernel, dim3(blocks), dim3(warps * 32), 0,
                    s, static_cast<const uint4*>(rows), inv_perm, gates, T, k, D / 8,
                    static_cast<uint4*>(out));
}

}  // namespace moeq
