// Router top-k -> per-expert groups -> active-expert chunks -> stable
// permutation of the token rows.
//
// Orbit article, "Active-expert-chunked dequantization": each token only
// activates the experts its router selects, and the selected experts are
// batched into fixed-size groups before the grouped GEMM.
//
// Four kernels, no host round trip:
//  1. route_topk_kernel: one warp per token (2 tokens per warp, 64 per
//     1024-thread block; one token per warp for small launches); k rounds of a
//     warp-wide argmax (ties to the lower expert id), softmax of the k
//     selected logits, and a per-block expert histogram in shared memory.
//  2. route_scan_kernel: one block; per expert, an exclusive scan of the
//     block histograms (block bases for step 3), then scans over experts for
//     the offsets, the active list and the chunk table.
//  3. route_scatter_kernel: per block, a 64-bit token mask per expert built
//     with shared-memory atomicOr; the rank of token t inside expert e is the
//     popcount of the mask below t, which gives the stable position
//     offsets[e] + block_base[e] + rank.
//  4. permute_rows_kernel: one warp per token reads its row once, with
//     16-byte loads, and writes it to each of its k permuted rows. (One warp
//     per permuted row reads every token row k times; at 16384 tokens x 14 KB
//     those re-reads miss L2 and cost as much DRAM traffic as the writes.)
// Small launches (T <= 1024 and a token-by-expert bit matrix of at most 8192
// words) replace steps 2 and 3 by route_tail_kernel: one block builds, for
// every expert, the bit mask of its tokens over all T, and takes counts,
// offsets and stable ranks from popcounts of those masks; the serial walk
// over the per-block histograms, and one launch, go away.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "launchers.cuh"

namespace moeq {

namespace {

constexpr int kRouteTokensPerBlock = 64;
constexpr int kRouteThreads = 256;
constexpr int kTopkThreads = 1024;
constexpr int kTailMaxWords = 8192;   // token-by-expert bit matrix of the routing tail
constexpr int kTailRowsPerBlock = 256; // permuted rows a tail block writes and copies

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// NPER: logits held per lane (>= ceil(E / 32)); the selection loops run over
// exactly NPER slots.
// tpb tokens per block (a multiple of 32); block_counts == nullptr skips the
// per-block histogram.
template <int NPER>
__global__ void __launch_bounds__(kTopkThreads)
route_topk_kernel(const float* __restrict__ logits, int T, int E, int k, int tpb,
                  int32_t* __restrict__ topk_idx, float* __restrict__ gates,
                  int32_t* __restrict__ block_counts) {
  extern __shared__ int32_t hist[];   // [E]
  grid_dependency_wait();
  grid_dependents_launch();
  const bool with_hist = block_counts != nullptr;
  if (with_hist)
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_warp = tpb / (kTopkThreads / 32);
  for (int u = 0; u < per_warp; ++u) {
    const int t = blockIdx.x * tpb + warp * per_warp + u;
    if (t >= T) break;
    const float* row = logits + static_cast<int64_t>(t) * E;
    float v[NPER];
#pragma unroll
    for (int i = 0; i < NPER; ++i) {
      const int e = lane + 32 * i;
      v[i] = (e < E) ? row[e] : 0.0f;
    }
    uint32_t taken = 0;
    float my_val = 0.0f;
    int my_idx = 0;
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < NPER; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !((taken >> i) & 1u) && better(v[i], e, bv, bi)) {
          bv = v[i];
          bi = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (better(ov, oi, bv, bi)) {
          bv = ov;
          bi = oi;
        }
      }
      // Only rows with NaN logits can leave no candidate; keep the index in
      // range (their routing is unspecified).
      bi = min(bi, E - 1);
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      if (lane == j) {
        my_val = bv;
        my_idx = bi;
      }
    }
    // gates: softmax over the k selected logits (the first is the largest)
    const float top = __shfl_sync(0xffffffffu, my_val, 0);
    const float z = (lane < k) ? expf(my_val - top) : 0.0f;
    float sum = z;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane < k) {
      topk_idx[static_cast<int64_t>(t) * k + lane] = my_idx;
      gates[static_cast<int64_t>(t) * k + lane] = z / sum;
      if (with_hist) atomicAdd(&hist[my_idx], 1);
    }
  }
  if (!with_hist) return;
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    block_counts[static_cast<int64_t>(blockIdx.x) * E + e] = hist[e];
}

// Block-wide step shared by the scan kernels (blockDim = 1024, E <= 1024):
// thread e holds the row count of expert e; writes offsets[0..E], the active
// list (ascending ids), num_active and the chunk table, and returns the
// exclusive offset of expert e.
__device__ int scan_experts(int cnt, int E, int chunk_size, int32_t* __restrict__ offsets,
                            int32_t* __restrict__ active, int32_t* __restrict__ num_active,
                            int32_t* __restrict__ chunk_offsets, int32_t* __restrict__ num_chunks,
                            bool write = true) {
  __shared__ int32_t ws_cnt[32];
  __shared__ int32_t ws_act[32];
  const int e = threadIdx.x;
  const int act = (e < E && cnt > 0) ? 1 : 0;
  const int lane = e & 31, w = e >> 5;
  int xc = cnt, xa = act;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int yc = __shfl_up_sync(0xffffffffu, xc, o);
    const int ya = __shfl_up_sync(0xffffffffu, xa, o);
    if (lane >= o) {
      xc += yc;
      xa += ya;
    }
  }
  if (lane == 31) {
    ws_cnt[w] = xc;
    ws_act[w] = xa;
  }
  __syncthreads();
  if (w == 0) {
    int sc = ws_cnt[lane], sa = ws_act[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yc = __shfl_up_sync(0xffffffffu, sc, o);
      const int ya = __shfl_up_sync(0xffffffffu, sa, o);
      if (lane >= o) {
        sc += yc;
        sa += ya;
      }
    }
    ws_cnt[lane] = sc;
    ws_act[lane] = sa;
  }
  __syncthreads();
  const int incl_c = xc + (w > 0 ? ws_cnt[w - 1] : 0);
  const int incl_a = xa + (w > 0 ? ws_act[w - 1] : 0);
  if (!write) return incl_c - cnt;
  if (e < E) {
    offsets[e] = incl_c - cnt;
    if (act) active[incl_a - 1] = e;
  }
  if (e == E - 1) offsets[E] = incl_c;
  const int A = ws_act[(E - 1) >> 5];   // inclusive total of the last warp holding an expert
  const int nch = (A + chunk_size - 1) / chunk_size;
  if (e == 0) {
    *num_active = A;
    *num_chunks = nch;
  }
  for (int c = e; c <= nch; c += blockDim.x) chunk_offsets[c] = min(c * chunk_size, A);
  return incl_c - cnt;
}

// One block of 1024 threads, E <= 1024.
__global__ void __launch_bounds__(1024)
route_scan_kernel(int32_t* __restrict__ block_counts, int nblk, int E, int chunk_size,
                  int32_t* __restrict__ offsets, int32_t* __restrict__ active,
                  int32_t* __restrict__ num_active, int32_t* __restrict__ chunk_offsets,
                  int32_t* __restrict__ num_chunks) {
  grid_dependency_wait();
  grid_dependents_launch();
  const int e = threadIdx.x;
  int cnt = 0;
  if (e < E) {
    for (int b = 0; b < nblk; ++b) {
      const int64_t i = static_cast<int64_t>(b) * E + e;
      const int c = block_counts[i];
      block_counts[i] = cnt;      // becomes the block's base inside expert e
      cnt += c;
    }
  }
  scan_experts(cnt, E, chunk_size, offsets, active, num_active, chunk_offsets, num_chunks);
}

// Blocks of 1024 threads, E <= 1024, W = ceil(T / 32) <= 32 words per
// expert, E * W <= kTailMaxWords. mask[e][w] bit b is set when token 32 w + b
// chose expert e; pre[e][w] counts the tokens of expert e in words before w
// (one warp per expert scans its W word popcounts). Rows of the two tables
// are W + 1 words apart, so that the entries of one word index for different
// experts fall in different shared-memory banks. The rank of token t in
// expert e is pre[e][w] + popc(mask[e][w] below bit b), so rows stay in
// ascending token order inside each expert.
// Every block builds the tables (a few microseconds of shared-memory work);
// block 0 writes the offsets, the active list and the chunk table, and block
// b writes the permutation entries of the permuted rows [p0, p1) it owns and,
// when x is given, copies those rows (x_perm[p] = x[perm_token[p]]), so the
// row copy needs no launch of its own.
__global__ void __launch_bounds__(1024)
route_tail_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k, int chunk_size,
                  int32_t* __restrict__ offsets, int32_t* __restrict__ active,
                  int32_t* __restrict__ num_active, int32_t* __restrict__ chunk_offsets,
                  int32_t* __restrict__ num_chunks, int32_t* __restrict__ perm_token,
                  int32_t* __restrict__ inv_perm, const uint4* __restrict__ x,
                  uint4* __restrict__ x_perm, int64_t row_vec) {
  grid_dependency_wait();
  grid_dependents_launch();
  extern __shared__ uint32_t tail_sm[];
  __shared__ int32_t cnt_s[1024];
  __shared__ int32_t off_s[1024];
  __shared__ int32_t tok_s[kTailRowsPerBlock];
  const int W = (T + 31) >> 5;
  const int WP = W + 1;                                        // row pitch in words
  uint32_t* mask = tail_sm;                                    // [E][WP]
  int32_t* pre = reinterpret_cast<int32_t*>(tail_sm + WP * E);  // [E][WP]
  const int n = T * k;
  const int per = (n + gridDim.x - 1) / gridDim.x;             // permuted rows per block
  const int p0 = min(n, static_cast<int>(blockIdx.x) * per), p1 = min(n, p0 + per);
  for (int i = threadIdx.x; i < WP * E; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int t = i / k;
    const int e = __ldg(topk_idx + i);
    atomicOr(&mask[e * WP + (t >> 5)], 1u << (t & 31));
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = warp; e < E; e += 32) {
    const int c = (lane < W) ? __popc(mask[e * WP + lane]) : 0;
    int xs = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, xs, o);
      if (lane >= o) xs += y;
    }
    if (lane < W) pre[e * WP + lane] = xs - c;
    if (lane == 31) cnt_s[e] = xs;
  }
  __syncthreads();
  const int e = threadIdx.x;
  const int off = scan_experts(e < E ? cnt_s[e] : 0, E, chunk_size, offsets, active, num_active,
                               chunk_offsets, num_chunks, blockIdx.x == 0);
  if (e < E) off_s[e] = off;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int t = i / k;
    const int ex = __ldg(topk_idx + i);
    const int w = t >> 5, b = t & 31;
    const int p = off_s[ex] + pre[ex * WP + w] + __popc(mask[ex * WP + w] & ((1u << b) - 1u));
    if (p >= p0 && p < p1) {
      perm_token[p] = t;
      inv_perm[i] = p;
      tok_s[p - p0] = t;
    }
  }
  if (x == nullptr) return;
  __syncthreads();
  // One warp per owned row, 16-byte moves, four loads in flight per lane.
  for (int r = warp; r < p1 - p0; r += 32) {
    const uint4* src = x + static_cast<int64_t>(tok_s[r]) * row_vec;
    uint4* dst = x_perm + static_cast<int64_t>(p0 + r) * row_vec;
    int64_t c = lane;
    for (; c + 96 < row_vec; c += 128) {
      const uint4 a0 = src[c], a1 = src[c + 32], a2 = src[c + 64], a3 = src[c + 96];
      dst[c] = a0;
      dst[c + 32] = a1;
      dst[c + 64] = a2;
      dst[c + 96] = a3;
    }
    for (; c < row_vec; c += 32) dst[c] = src[c];
  }
}

__global__ void __launch_bounds__(kRouteThreads)
route_scatter_kernel(const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ block_base,
                     const int32_t* __restrict__ offsets, int T, int E, int k,
                     int32_t* __restrict__ perm_token, int32_t* __restrict__ inv_perm) {
  grid_dependency_wait();
  grid_dependents_launch();
  extern __shared__ uint32_t sm[];      // lo[E], hi[E]
  uint32_t* lo = sm;
  uint32_t* hi = sm + E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    lo[e] = 0;
    hi[e] = 0;
  }
  __syncthreads();
  const int t0 = blockIdx.x * kRouteTokensPerBlock;
  const int ntok = min(kRouteTokensPerBlock, T - t0);
  const int nent = ntok * k;
  for (int i = threadIdx.x; i < nent; i += blockDim.x) {
    const int tl = i / k;
    const int e = topk_idx[static_cast<int64_t>(t0) * k + i];
    atomicOr(tl < 32 ? &lo[e] : &hi[e], 1u << (tl & 31));
  }
  __syncthreads();
  const int32_t* base = block_base + static_cast<int64_t>(blockIdx.x) * E;
  for (int i = threadIdx.x; i < nent; i += blockDim.x) {
    const int tl = i / k;
    const int e = topk_idx[static_cast<int64_t>(t0) * k + i];
    const int rank = (tl < 32) ? __popc(lo[e] & ((1u << tl) - 1u))
                               : __popc(lo[e]) + __popc(hi[e] & ((1u << (tl - 32)) - 1u));
    const int p = offsets[e] + base[e] + rank;
    perm_token[p] = t0 + tl;
    inv_perm[static_cast<int64_t>(t0) * k + i] = p;
  }
}

// One warp per token t: x_perm[inv_perm[t * k + j]] = x[t] for j < k
// (16-byte moves; the row is read once).
__global__ void __launch_bounds__(256)
permute_rows_kernel(const int32_t* __restrict__ inv_perm, int T, int k, const uint4* __restrict__ x,
                    uint4* __restrict__ x_perm, int64_t row_vec) {
  grid_dependency_wait();
  grid_dependents_launch();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  // Lane j < k holds the permuted row of (t, j); k <= 32.
  const int64_t my_dst =
      (lane < k) ? static_cast<int64_t>(__ldg(inv_perm + static_cast<int64_t>(t) * k + lane)) * row_vec : 0;
  const uint4* src = x + static_cast<int64_t>(t) * row_vec;
  // 128 16-byte units of the row per step (four a lane); the loops stay
  // warp-uniform around the shuffles, and units past the row are skipped.
  for (int64_t base = 0; base < row_vec; base += 128) {
    uint4 a[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t c = base + lane + 32 * u;
      a[u] = (c < row_vec) ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    }
    for (int j = 0; j < k; ++j) {
      const int64_t dst = __shfl_sync(0xffffffffu, my_dst, j);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t c = base + lane + 32 * u;
        if (c < row_vec) x_perm[dst + c] = a[u];
      }
    }
  }
}

}  // namespace

int route_num_blocks(int64_t T) {
  return static_cast<int>((T + kRouteTokensPerBlock - 1) / kRouteTokensPerBlock);
}

bool route_single_pass(int64_t T, int E) {
  const int64_t W = (T + 31) / 32;
  return W <= 32 && W * E <= kTailMaxWords;
}

namespace {

std::mutex g_route_setup_mutex;
bool g_route_setup_done[64] = {false};
int g_route_sm_count[64] = {0};

}  // namespace

// The tail's dynamic shared memory may pass 48 KiB: its limit is raised once
// per device, and the SM count read once, under a lock (so concurrent host
// threads are safe); later calls only read the cached values, so calls made
// during stream capture do no setup once a call on that device has run.
cudaError_t route_prepare_device(int* sm_count) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_route_setup_mutex);
  if (!g_route_setup_done[dev]) {
    err = cudaFuncSetAttribute(route_tail_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(2 * (kTailMaxWords + 1024) * sizeof(uint32_t)));
    if (err != cudaSuccess) return err;
    err = cudaDeviceGetAttribute(&g_route_sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    g_route_setup_done[dev] = true;
  }
  if (sm_count) *sm_count = g_route_sm_count[dev];
  return cudaSuccess;
}

cudaError_t launch_route(const float* logits, const void* x, int T, int E, int k, int64_t d,
                         int chunk_size, int32_t* topk_idx, float* gates, int32_t* offsets,
                         int32_t* active, int32_t* num_active, int32_t* chunk_offsets,
                         int32_t* num_chunks, int32_t* perm_token, int32_t* inv_perm,
                         void* x_perm, int32_t* block_counts, cudaStream_t s) {
  const int W = (T + 31) / 32;
  // Small launches: one token per warp, then the single-block tail.
  const bool small = route_single_pass(T, E);
  if (!small && block_counts == nullptr) return cudaErrorInvalidValue;
  const int tpb = small ? kTopkThreads / 32 : kRouteTokensPerBlock;
  const int nblk = small ? (T + tpb - 1) / tpb : route_num_blocks(T);
  int32_t* hist_out = small ? nullptr : block_counts;
  const int nper = (E + 31) / 32;
  const size_t hsm = small ? 0 : E * sizeof(int32_t);
#define MOEQ_TOPK(N_)                                                                  \
  launch_pdl(route_topk_kernel<N_>, dim3(nblk), dim3(kTopkThreads), hsm, s, logits, T, E, k, \
             tpb, topk_idx, gates, hist_out)
  cudaError_t err;
  if (nper <= 1) err = MOEQ_TOPK(1);
  else if (nper <= 2) err = MOEQ_TOPK(2);
  else if (nper <= 4) err = MOEQ_TOPK(4);
  else if (nper <= 8) err = MOEQ_TOPK(8);
  else if (nper <= 12) err = MOEQ_TOPK(12);
  else if (nper <= 16) err = MOEQ_TOPK(16);
  else err = MOEQ_TOPK(32);
#undef MOEQ_TOPK
  if (err != cudaSuccess) return err;
  if (small) {
    int sm_count = 0;
    err = route_prepare_device(&sm_count);
    if (err != cudaSuccess) return err;
    const size_t tsm = 2 * static_cast<size_t>(W + 1) * E * sizeof(uint32_t);
    // With x, one block per SM (at least enough for kTailRowsPerBlock rows
    // each) shares the row copy; without it one block does the tail alone.
    const int M = T * k;
    int blocks = 1;
    if (x != nullptr) {
      blocks = std::max(1, std::min(sm_count, (M + 7) / 8));
      blocks = std::max(blocks, (M + kTailRowsPerBlock - 1) / kTailRowsPerBlock);
    } else if (M > kTailRowsPerBlock) {
      blocks = (M + kTailRowsPerBlock - 1) / kTailRowsPerBlock;
    }
    return launch_pdl(route_tail_kernel, dim3(blocks), dim3(1024), tsm, s,
                      static_cast<const int32_t*>(topk_idx), T, E, k, chunk_size, offsets,
                      active, num_active, chunk_offsets, num_chunks, perm_token, inv_perm,
                      static_cast<const uint4*>(x), static_cast<uint4*>(x_perm), d / 8);
  } else {
    err = launch_pdl(route_scan_kernel, dim3(1), dim3(1024), 0, s, block_counts, nblk, E,
                     chunk_size, offsets, active, num_active, chunk_offsets, num_chunks);
    if (err != cudaSuccess) return err;
    const size_t sm = 2 * E * sizeof(uint32_t);
    err = launch_pdl(route_scatter_kernel, dim3(nblk), dim3(kRouteThreads), sm, s,
                     static_cast<const int32_t*>(topk_idx), static_cast<const int32_t*>(block_counts),
                     static_cast<const int32_t*>(offsets), T, E, k, perm_token, inv_perm);
  }
  if (err != cudaSuccess || x == nullptr) return err;
  return launch_pdl(permute_rows_kernel, dim3((T + 7) / 8), dim3(256), 0, s,
                    static_cast<const int32_t*>(inv_perm), T, k, static_cast<const uint4*>(x),
                    static_cast<uint4*>(x_perm), d / 8);
}

}  // namespace moeq
