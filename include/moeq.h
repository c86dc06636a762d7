/*
 * moeq.h -- C ABI of the B200 (sm_100a) low-bit MoE grouped-GEMM library.
 *
 * The library computes one layer of a mixture-of-experts FFN whose expert
 * weights are a frozen 4-bit base (INT4 or MXFP4) and whose trainable part is
 * a BF16 block-diagonal adapter on the activations:
 *
 *   router top-k -> per-expert token groups -> active-expert chunks ->
 *   dequantize inside the GEMM kernel -> grouped BF16 GEMM (forward, and the
 *   activation-gradient backward with no base-weight gradient) -> combine.
 *
 * Source of the method: Orbit article, section "technical details",
 * paragraphs "Active-expert-chunked dequantization" (group the router-selected
 * experts into fixed-size batches, dequantize, grouped GEMM, release the
 * high-precision weights) and the DeepSeek-V4 paragraph (GEMM backward that
 * bypasses the frozen base's weight gradient); Orbit issue #1 (OFT adapter,
 * quantized weights fine-tuned directly without storing a dequantized base);
 * open-weight MoE explainer, section 3 (MXFP4: 4-bit elements in groups of 32
 * with one shared scale). Here no dequantized weight is ever written to
 * global memory: each GEMM kernel dequantizes a tile into tensor memory
 * (forward) or shared memory (backward) and feeds the tensor cores from
 * there.
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers, allocated and owned by the
 *    caller; the library never allocates, frees or synchronizes (except
 *    moe_get_device_error, which synchronizes the given stream).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). Work is enqueued on it in order; no host round trip happens
 *    inside any call, so counts and tables produced on the device are
 *    consumed on the device.
 *  - Every tensor pointer must be 16-byte aligned; every call validates its
 *    arguments on the host and returns a status without launching anything
 *    when they are wrong. No exception crosses the ABI.
 *  - Kernels never trap. A device-side anomaly (a pipeline wait that ran out
 *    of its time budget, an offsets table inconsistent with M) sets a device
 *    error word that moe_get_device_error reads and clears.
 *  - Workspace: calls that take (ws, ws_bytes) report the bytes they need
 *    when ws == NULL and ws_bytes != NULL (then nothing is launched and
 *    *ws_bytes is written). With ws == NULL and ws_bytes == NULL the call
 *    runs without a workspace, which is valid only when the query returned
 *    0. Otherwise *ws_bytes must hold the size of ws, which must be at least
 *    the queried size and 256-byte aligned.
 *  - BF16 tensors are row-major with the last dimension contiguous.
 *
 * Weight formats (moe_qweight)
 *  - packed: uint8 [E][N][K/2]; byte i of a row holds element 2i in its low
 *    nibble and element 2i+1 in its high nibble.
 *  - scales: [E][K/32][N] (group-major): the scale of row n, elements
 *    32g..32g+31, is scales[e][g][n].
 *  - MOE_W_INT4_G32_BF16: codes are two's-complement nibbles -8..7 and scales
 *    BF16; w = bf16(q * s), one rounding to nearest even.
 *  - MOE_W_MXFP4_G32_E8M0: codes are E2M1 (sign bit 3; magnitudes 0, 0.5, 1,
 *    1.5, 2, 3, 4, 6) and scales E8M0 (2^(X-127), X = 255 is NaN);
 *    w = bf16(e2m1 * 2^(X-127)), exact except overflow to inf.
 *  Requirements: K % 64 == 0, N % 64 == 0 (N % 128 == 0 for the SwiGLU
 *  gate/up weight, whose rows 0..N/2-1 are the gate and N/2..N-1 the up
 *  projection), 1 <= E <= 1024, E*N < 2^31. Other shapes return
 *  MOE_ERR_UNSUPPORTED without launching. (The kernels stream the reduction
 *  in 64-element halves of 128-wide steps and write output features in
 *  blocks of 32 or 64; every expert shape of the Orbit and MXFP4 pages is a
 *  multiple of 512.)
 */
#ifndef MOEQ_H
#define MOEQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t moe_status;
enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* a size, enum or pointer argument is invalid */
  MOE_ERR_MISALIGNED = 2,   /* a pointer is not 16-byte aligned (ws: 256) */
  MOE_ERR_UNSUPPORTED = 3,  /* a shape the kernels do not handle */
  MOE_ERR_WORKSPACE = 4,    /* ws smaller than required */
  MOE_ERR_CUDA = 5,         /* a CUDA runtime/driver call failed */
  MOE_ERR_DEVICE = 6        /* the device error word was set (see below) */
};

/* Weight format tags. */
enum { MOE_W_INT4_G32_BF16 = 1, MOE_W_MXFP4_G32_E8M0 = 2 };

/* GEMM epilogues. */
enum {
  MOE_EPI_NONE = 0,        /* out = bf16(acc) */
  MOE_EPI_SWIGLU = 1,      /* forward gate/up: out = bf16(silu(g) * u) */
  MOE_EPI_SWIGLU_BWD = 2   /* backward of the down projection: out = bf16([dg | du]) */
};

/* Device error word values (moe_get_device_error). */
enum {
  MOE_DEVERR_NONE = 0,
  MOE_DEVERR_WAIT_TIMEOUT = 1,  /* a pipeline wait exceeded its budget; the kernel returned */
  MOE_DEVERR_BAD_OFFSETS = 2    /* expert offsets do not describe M rows */
};

/* A frozen 4-bit expert stack W[e] of shape [N, K] (see "Weight formats"). */
typedef struct moe_qweight {
  const void* packed;   /* device, uint8 [E][N][K/2] */
  const void* scales;   /* device, [E][K/32][N]: bf16 (INT4) or uint8 E8M0 (MXFP4) */
  int32_t E, N, K;
  int32_t fmt;          /* MOE_W_* */
} moe_qweight;

/* Per-expert row groups produced by moe_route_permute (all device pointers). */
typedef struct moe_groups {
  const int32_t* expert_offsets;  /* [E+1]: rows of expert e are [off[e], off[e+1]) */
  const int32_t* active;          /* [E]: experts with rows, ascending (first *num_active valid) */
  const int32_t* num_active;      /* [1] */
  const int32_t* chunk_offsets;   /* [E+1]: chunk c = active[chunk_offsets[c] .. chunk_offsets[c+1]) */
  const int32_t* num_chunks;      /* [1] */
  int32_t E;
} moe_groups;

/*
 * moe_route_permute -- router top-k, per-expert groups, active-expert
 * chunks and the stable permutation (Orbit article, "Active-expert-chunked
 * dequantization": the router-selected experts are grouped into fixed-size
 * batches).
 *
 *  logits      [T][E] fp32 router logits.
 *  x           [T][d] bf16 token activations; may be NULL (then x_perm is
 *              not written and d is ignored).
 *  k           experts per token, 1 <= k <= min(E, 32).
 *  chunk_size  experts per chunk, >= 1.
 * Outputs (device, caller-allocated):
 *  topk_idx    [T][k] int32: the k largest logits per token, descending,
 *              ties to the lower expert id.
 *  gates       [T][k] fp32: softmax over the k selected logits.
 *  expert_offsets [E+1], active [E], num_active [1], chunk_offsets [E+1],
 *  num_chunks [1]: see moe_groups. Chunk c covers active experts
 *              chunk_size*c .. chunk_size*(c+1)-1; the last may be short.
 *  perm_token  [T*k] int32: token of permuted row p. Rows are expert-major,
 *              then ascending token id.
 *  inv_perm    [T*k] int32: permuted row of (token t, slot j) at t*k + j.
 *  x_perm      [T*k][d] bf16: x_perm[p] = x[perm_token[p]] (bit copy).
 *  ws          scratch of the per-block expert histograms. Launches that
 *              take the single-pass tail (T <= 1024 and E*ceil(T/32) <= 8192)
 *              need none: the size query returns 0 and (ws, ws_bytes) may both
 *              be NULL. Larger launches need ceil(T/64)*E int32 (rounded up to
 *              256 bytes).
 * Requires T >= 1, 1 <= E <= 1024, d % 8 == 0 when x is given,
 * T*k < 2^31.
 */
moe_status moe_route_permute(const float* logits, const void* x, int64_t T, int32_t E,
                             int32_t k, int64_t d, int32_t chunk_size, int32_t* topk_idx,
                             float* gates, int32_t* expert_offsets, int32_t* active,
                             int32_t* num_active, int32_t* chunk_offsets, int32_t* num_chunks,
                             int32_t* perm_token, int32_t* inv_perm, void* x_perm, void* ws,
                             size_t* ws_bytes, void* stream);

/*
 * moe_route_permute_noalloc -- moe_route_permute for callers that cannot give
 * the library any scratch memory. The source pages have no counterpart of
 * this entry point; it exists for callers such as a serving runtime that
 * reserves all device memory in one arena at start-up and allocates nothing
 * afterwards, code that enqueues work while a CUDA graph is being captured
 * (where cudaMalloc is not allowed), or a C host without a caching allocator,
 * for which a cudaMalloc/cudaFree pair per call would synchronize the device.
 *
 * Arguments, outputs and results are those of moe_route_permute, without
 * (ws, ws_bytes). The caller still allocates every input and output. The
 * per-block expert histograms live in a fixed 4 MiB array inside the library
 * (2^20 int32 entries), which every GPU that loads the library holds until
 * the process exits. Sizes whose histograms do not fit, that is
 * ceil(T/64) * E > 2^20, are rejected with MOE_ERR_WORKSPACE before anything
 * is launched. The call itself never allocates or frees device memory.
 *
 * The first call on a device does this library's one-time setup there: it
 * looks up the array's device address (with that device current) and caches
 * it, and it sets the routing kernels' shared-memory limit. Make that first
 * call before any stream capture; later calls do no setup. The cached
 * address belongs to the device's current context: after cudaDeviceReset the
 * array may live elsewhere, so do not call this entry point again in that
 * process after a reset. All calls on a device share the one array: calls
 * whose kernels overlap on the GPU (different streams without ordering
 * between them) race on it and give wrong results. Calls ordered on one
 * stream are safe; each call rewrites the entries it reads, so leftovers of
 * an earlier call do not matter.
 */
moe_status moe_route_permute_noalloc(const float* logits, const void* x, int64_t T, int32_t E,
                                     int32_t k, int64_t d, int32_t chunk_size, int32_t* topk_idx,
                                     float* gates, int32_t* expert_offsets, int32_t* active,
                                     int32_t* num_active, int32_t* chunk_offsets,
                                     int32_t* num_chunks, int32_t* perm_token, int32_t* inv_perm,
                                     void* x_perm, void* stream);

/*
 * moe_grouped_qgemm_fwd -- forward grouped GEMM over the dequantized experts
 * (Orbit article, "Active-expert-chunked dequantization"). For every row p of
 * expert e:  acc[p] = a'[p] . W[e]^T  (fp32 accumulation on the tensor cores),
 * where a' = a, or with an adapter a'[p] = bf16(a[p] . R_e) with R_e the
 * block-diagonal matrix of adapter[e][b] (32 x 32 blocks, row-vector
 * convention, x'[32b+j] = sum_i x[32b+i] R[e][b][i][j]).
 *
 *  a        [M][K] bf16 permuted rows (x_perm), grouped by expert offsets;
 *           or, with a_rows, the token rows [T][K] themselves.
 *  a_rows   NULL, or device int32 [M]: row p of the GEMM input is
 *           a[a_rows[p]] (perm_token from moe_route_permute). The kernels
 *           then gather the rows as they go, and the permuted rows never
 *           need to be written to memory (moe_route_permute may be called
 *           with x = NULL). Each index must be a valid row of a.
 *  w        frozen weights, W[e] is [N][K].
 *  g        groups from moe_route_permute; g->E == w->E, off[E] == M.
 *  adapter  NULL or [E][K/32][32][32] bf16.
 *  epi      MOE_EPI_NONE: out [M][N] = bf16(acc).
 *           MOE_EPI_SWIGLU: out [M][N/2] = bf16(silu(acc[:, :N/2]) *
 *           acc[:, N/2:]) and, if saved_gu != NULL, saved_gu [M][N] =
 *           bf16(acc) (kept for the backward).
 *  ws       scratch: M*K bf16 for a' with an adapter; none without one.
 * Experts with no rows cost nothing: their weight bytes are never read.
 */
moe_status moe_grouped_qgemm_fwd(const void* a, const int32_t* a_rows, int64_t M,
                                 const moe_qweight* w, const moe_groups* g, const void* adapter,
                                 int32_t epi, void* out, void* saved_gu, void* ws,
                                 size_t* ws_bytes, void* stream);

/*
 * moe_grouped_qgemm_bwd_dx -- activation-gradient grouped GEMM; the frozen
 * base gets no gradient (Orbit article, DeepSeek-V4 paragraph: the GEMM
 * backward bypasses the base-weight gradient). For every row p of expert e:
 * acc[p] = dout[p] . W[e]  (contraction over W's N rows, output over K).
 *
 *  dout     [M][N] bf16.
 *  epi      MOE_EPI_NONE: din [M][K] = bf16(acc), or with an adapter:
 *             dx' = bf16(acc); din[p][32b+i] = bf16(sum_j dx'[p][32b+j] *
 *             R[e][b][i][j]); d_adapter[e][b][i][j] = sum over rows p of e of
 *             a[p][32b+i] * dx'[p][32b+j] (fp32, overwritten, deterministic
 *             order; experts without rows get 0).
 *           MOE_EPI_SWIGLU_BWD (down projection, W = W_d [N=d][K=f]):
 *             acc = dh; with saved_gu [M][2K] = bf16(g | u) from the forward,
 *             s = sigmoid(g): din [M][2K] = bf16([dh*u*s*(1+g*(1-s)) |
 *             dh*g*s]). adapter must be NULL.
 *  adapter, a, d_adapter: NULL, or all three given (a = the forward's a).
 *  a_rows   NULL, or device int32 [M] as in moe_grouped_qgemm_fwd: row p of
 *           the adapter's input is a[a_rows[p]] (only with an adapter).
 *  ws       scratch: M*K bf16 for dx' with an adapter; none without one.
 */
moe_status moe_grouped_qgemm_bwd_dx(const void* dout, int64_t M, const moe_qweight* w,
                                    const moe_groups* g, int32_t epi, const void* saved_gu,
                                    const void* adapter, const void* a, const int32_t* a_rows,
                                    void* din, float* d_adapter, void* ws, size_t* ws_bytes,
                                    void* stream);

/*
 * moe_unpermute_combine -- the two row moves around the grouped GEMMs.
 *  mode 0 (combine):  out[t] = bf16(sum_{j<k} g[t][j] * rows[inv_perm[t*k+j]]),
 *                     fp32 sum in slot order; rows [T*k][D], out [T][D].
 *  mode 1 (scatter):  out[inv_perm[t*k+j]] = bf16(g[t][j] * rows[t]);
 *                     rows [T][D], out [T*k][D] (backward of mode 0 with
 *                     respect to the per-slot rows).
 *  gates [T][k] fp32, or NULL for all ones. D % 8 == 0.
 * The gate weights are applied here, not inside the GEMM.
 */
moe_status moe_unpermute_combine(const void* rows, const int32_t* inv_perm, const float* gates,
                                 int64_t T, int32_t k, int64_t D, void* out, int32_t mode,
                                 void* stream);

/*
 * moe_dequant_experts -- whole experts of a 4-bit stack dequantized into a
 * BF16 buffer: out[i] = W[experts[i]] ([N][K] bf16, row-major) for i < count.
 * This is the step the Orbit article's own scheme runs on each chunk of active
 * experts ("Active-expert-chunked dequantization": the selected experts'
 * weights are dequantized into a temporary high-precision buffer before the
 * grouped GEMM, and the buffer is released after it). The grouped GEMMs of
 * this library never call it; it serves the comparison with that scheme.
 *
 *  experts  device int32 [count], expert ids in [0, E). An id outside that
 *           range gives zeros and sets MOE_DEVERR_BAD_OFFSETS.
 *  out      device bf16 [count][N][K], caller-allocated (count*N*K*2 bytes).
 * Same dequantization as the GEMM kernels, bit for bit. count == 0 launches
 * nothing.
 */
moe_status moe_dequant_experts(const moe_qweight* w, const int32_t* experts, int32_t count,
                               void* out, void* stream);

/*
 * moe_ep_regroup -- expert parallelism over W ranks: reorders the rows one
 * rank received from its peers. The experts are split into W contiguous
 * ranges of E_loc (rank r owns experts r*E_loc .. (r+1)*E_loc-1); every rank
 * routes its own tokens, and the run of its x_perm rows that belongs to rank
 * r's experts goes to rank r in one all-to-all exchange. The pages' setting
 * (Orbit article: a trillion-parameter INT4 MoE trained in one 8xB200 node)
 * needs this split: its base weights do not fit one GPU.
 *
 *  counts     device int32 [W][E_loc]: rows received from source rank s for
 *             local expert e. The received rows are source-major: for s =
 *             0..W-1, for e = 0..E_loc-1, the source's rows of e in its order.
 *  R          total rows (the sum of counts, which the exchange needs on the
 *             host anyway). A mismatch sets MOE_DEVERR_BAD_OFFSETS and copies
 *             nothing.
 *  rows_in, rows_out  device bf16 [R][D], D % 8 == 0.
 *  direction  0: rows_out = rows_in reordered to local expert-major order
 *             (expert, then source, then the source's order), and the local
 *             group tables are written for the local grouped GEMMs:
 *             expert_offsets [E_loc+1], active [E_loc], num_active [1],
 *             chunk_offsets [E_loc+1], num_chunks [1] (as moe_route_permute
 *             writes them, with chunk_size experts per chunk).
 *             1: the inverse (local expert-major -> source-major, to send the
 *             results back); the table pointers are not used and may be NULL.
 * Requires 1 <= W, 1 <= E_loc, W*E_loc <= 2048.
 */
moe_status moe_ep_regroup(const int32_t* counts, int32_t W, int32_t E_loc, int64_t R,
                          const void* rows_in, void* rows_out, int64_t D, int32_t direction,
                          int32_t chunk_size, int32_t* expert_offsets, int32_t* active,
                          int32_t* num_active, int32_t* chunk_offsets, int32_t* num_chunks,
                          void* stream);

/* Synchronizes `stream`, then reads and clears the device error word of the
 * current device (MOE_DEVERR_*). Debug/test use. */
moe_status moe_get_device_error(int32_t* code, void* stream);

/* Human-readable status name (static storage). */
const char* moe_status_string(moe_status s);

/* ABI revision of this header, for bindings to check. */
int32_t moe_abi_version(void);

/* 1 when the library was built with NVTX ranges (the default): every entry
 * point that launches work opens a range named after itself for its
 * duration on the host (a no-op unless a profiler is attached). 0 when built
 * with -DMOEQ_NVTX=0. */
int32_t moe_nvtx_enabled(void);

/*
 * Test hooks (not on the hot path).
 *
 * moe_test_dequant: dequantizes rows [R][K/2] with group-major scales
 * [K/32][R] into out [R][K] bf16 using the same device functions the GEMM
 * kernels use. fmt = MOE_W_*; K % 64 == 0.
 *
 * moe_test_set_wait_budget: sets the cycle budget of every pipeline wait
 * (default about one second); a tiny budget makes the waits of the next
 * GEMM run out so that the error path can be tested. 0 restores the default.
 */
moe_status moe_test_dequant(const void* packed, const void* scales, int64_t R, int32_t K,
                            int32_t fmt, void* out, void* stream);
moe_status moe_test_set_wait_budget(int64_t cycles);

#define MOEQ_ABI_VERSION 2

#ifdef __cplusplus
}
#endif

#endif /* MOEQ_H */
