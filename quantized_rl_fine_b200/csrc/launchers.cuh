// Host launchers of the non-GEMM kernels (internal to libmoeq).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moeq {

int route_num_blocks(int64_t T);
// True when a routing launch takes the single-pass tail (no per-block
// histograms, so no scratch memory).
bool route_single_pass(int64_t T, int E);
// One-time per-device setup of the routing kernels (thread-safe); writes the
// device's SM count when sm_count is not NULL.
cudaError_t route_prepare_device(int* sm_count);
cudaError_t launch_route(const float* logits, const void* x, int T, int E, int k, int64_t d,
                         int chunk_size, int32_t* topk_idx, float* gates, int32_t* offsets,
                         int32_t* active, int32_t* num_active, int32_t* chunk_offsets,
                         int32_t* num_chunks, int32_t* perm_token, int32_t* inv_perm,
                         void* x_perm, int32_t* block_counts, cudaStream_t s);
cudaError_t launch_combine(const void* rows, const int32_t* inv_perm, const float* gates, int T,
                           int k, int64_t D, void* out, int mode, cudaStream_t s);
// out = x . R_e for the rows of each expert (forward adapter); with rows (not
// NULL), row p reads x[rows[p]].
cudaError_t launch_adapter_apply(const void* x, const int32_t* rows, const void* R,
                                 const int32_t* offsets, int E, int M, int K, void* out,
                                 cudaStream_t s);
// dx = dxp . R_e^T and dR = sum over each expert's rows of x^T dxp, in one pass;
// with rows (not NULL), row p of x is x[rows[p]].
cudaError_t launch_adapter_bwd(const void* x, const int32_t* rows, const void* dxp, const void* R,
                               const int32_t* offsets, int E, int K, void* dx, float* dR,
                               cudaStream_t s);
// Expert parallelism: received rows, source-major <-> local expert-major
// (dir 0 / 1); dir 0 also writes the local group tables.
cudaError_t launch_ep_regroup(const int32_t* counts, int W, int E_loc, int R, const void* in,
                              void* out, int64_t D, int dir, int chunk_size, int32_t* offsets,
                              int32_t* active, int32_t* num_active, int32_t* chunk_offsets,
                              int32_t* num_chunks, int sm_count, cudaStream_t s);
int ep_max_entries();
cudaError_t launch_dequant_rows(const void* packed, const void* scales, int64_t R, int K, int fmt,
                                void* out, cudaStream_t s);

}  // namespace moeq
