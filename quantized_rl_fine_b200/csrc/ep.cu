// Expert parallelism: reordering of the rows a rank receives from its peers.
//
// With the experts split over W ranks (rank r owns experts [r E/W, (r+1) E/W)),
// each rank routes its own tokens, and the rows of its expert-major x_perm
// that belong to rank r's experts form one contiguous run, which an
// all-to-all exchange delivers to rank r. The received rows arrive
// source-major: for source s = 0..W-1, the source's rows of each local expert
// e = 0..E_loc-1 in the source's own order. The local grouped GEMMs want them
// expert-major (expert, then source, then the source's order): one row
// permutation, the same one backwards for the results. This file builds it
// from the per-(source, expert) counts on the device, copies the rows, and
// writes the local group tables (offsets, active experts, chunks) that the
// GEMMs read, so the host never needs the counts for the GEMMs themselves.
//
// The pages' setting (Orbit article: a trillion-parameter INT4 model trained
// in one 8xB200 node) holds about 562 GB of base weights, more than one GPU;
// splitting the experts over the node's GPUs is what makes it fit.
#include <algorithm>

#include "common.cuh"
#include "launchers.cuh"

namespace moeq {

namespace {

constexpr int kEpThreads = 1024;
constexpr int kEpMaxEntries = 2048;   // W * E_loc (the routing allows E <= 1024)

// Inclusive block scan of one value per thread (1024 threads); `tot` gets
// the block total. `warp_tot` is 32 ints of shared memory.
__device__ int block_inclusive_scan(int v, int32_t* warp_tot, int* tot) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_tot[lane] = t;   // inclusive over warps
  }
  __syncthreads();
  const int before = (w > 0) ? warp_tot[w - 1] : 0;
  *tot = warp_tot[31];
  __syncthreads();
  return before + x;
}

// Every block builds, in shared memory, for each (source s, local expert e)
// entry j = s * E_loc + e: src_start[j], where its rows start in the
// source-major order, and dst_start[j], where they start in the local
// expert-major order. Then warps copy rows; block 0 writes the group tables
// (direction 0). dir 0: out[dst] = in[src]; dir 1: out[src] = in[dst].
__global__ void __launch_bounds__(kEpThreads)
ep_regroup_kernel(const int32_t* __restrict__ counts, int W, int E_loc, int R,
                  const uint4* __restrict__ in, uint4* __restrict__ out, int64_t row_vec, int dir,
                  int chunk_size, int32_t* __restrict__ offsets, int32_t* __restrict__ active,
                  int32_t* __restrict__ num_active, int32_t* __restrict__ chunk_offsets,
                  int32_t* __restrict__ num_chunks) {
  __shared__ int32_t src_start[kEpMaxEntries + 1];
  __shared__ int32_t dst_start[kEpMaxEntries];
  __shared__ int32_t exp_off[kEpMaxEntries + 1];   // local expert offsets (E_loc + 1)
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t bad;
  grid_dependency_wait();
  grid_dependents_launch();
  const int n = W * E_loc;
  const int tid = threadIdx.x;
  const int per = (n + kEpThreads - 1) / kEpThreads;     // entries per thread (<= 2)
  if (tid == 0) bad = 0;
  __syncthreads();
  // source-major exclusive scan of the counts
  int local = 0;
  for (int j = tid * per; j < min(n, (tid + 1) * per); ++j) {
    const int c = counts[j];
    if (c < 0) bad = 1;
    local += max(c, 0);
  }
  int total = 0;
  int run = block_inclusive_scan(local, warp_tot, &total) - local;
  for (int j = tid * per; j < min(n, (tid + 1) * per); ++j) {
    src_start[j] = run;
    run += max(counts[j], 0);
  }
  if (tid == 0) src_start[n] = total;
  // rows per local expert, and their exclusive scan
  const int per_e = (E_loc + kEpThreads - 1) / kEpThreads;
  int le = 0;
  for (int e = tid * per_e; e < min(E_loc, (tid + 1) * per_e); ++e)
    for (int s = 0; s < W; ++s) le += max(counts[s * E_loc + e], 0);
  int etot = 0;
  int erun = block_inclusive_scan(le, warp_tot, &etot) - le;
  for (int e = tid * per_e; e < min(E_loc, (tid + 1) * per_e); ++e) {
    exp_off[e] = erun;
    int d = erun;
    for (int s = 0; s < W; ++s) {
      dst_start[s * E_loc + e] = d;
      d += max(counts[s * E_loc + e], 0);
    }
    erun = d;
  }
  if (tid == 0) exp_off[E_loc] = etot;
  __syncthreads();
  if (bad || total != R) {
    if (blockIdx.x == 0 && tid == 0) raise_device_error(MOE_DEVERR_BAD_OFFSETS);
    return;
  }
  if (dir == 0 && blockIdx.x == 0) {
    // local group tables: offsets, active experts (ascending), chunks of them
    for (int e = tid; e <= E_loc; e += kEpThreads) offsets[e] = exp_off[e];
    int na = 0;
    for (int e = tid * per_e; e < min(E_loc, (tid + 1) * per_e); ++e)
      na += (exp_off[e + 1] > exp_off[e]) ? 1 : 0;
    int atot = 0;
    int arun = block_inclusive_scan(na, warp_tot, &atot) - na;
    for (int e = tid * per_e; e < min(E_loc, (tid + 1) * per_e); ++e)
      if (exp_off[e + 1] > exp_off[e]) active[arun++] = e;
    const int nch = (atot + chunk_size - 1) / chunk_size;
    for (int c = tid; c <= nch; c += kEpThreads) chunk_offsets[c] = min(c * chunk_size, atot);
    if (tid == 0) {
      *num_active = atot;
      *num_chunks = nch;
    }
  }
  // rows: warp per row, 16-byte vectors
  const int lane = tid & 31;
  const int wpb = kEpThreads / 32;
  for (int i = blockIdx.x * wpb + (tid >> 5); i < R; i += gridDim.x * wpb) {
    // the last entry whose rows start at or before i (empty entries share a
    // start with the next one, so taking the last skips them)
    int lo = 0, hi = n - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (src_start[mid] <= i) lo = mid; else hi = mid - 1;
    }
    const int64_t src = i;
    const int64_t dst = dst_start[lo] + (i - src_start[lo]);
    const uint4* from = in + (dir == 0 ? src : dst) * row_vec;
    uint4* to = out + (dir == 0 ? dst : src) * row_vec;
    for (int64_t c = lane; c < row_vec; c += 32) to[c] = from[c];
  }
}

}  // namespace

cudaError_t launch_ep_regroup(const int32_t* counts, int W, int E_loc, int R, const void* in,
                              void* out, int64_t D, int dir, int chunk_size, int32_t* offsets,
                              int32_t* active, int32_t* num_active, int32_t* chunk_offsets,
                              int32_t* num_chunks, int sm_count, cudaStream_t s) {
  const int wpb = kEpThreads / 32;
  const int want = (R + wpb - 1) / wpb;
  const int blocks = std::max(1, std::min(want, 4 * sm_count));
  return launch_pdl(ep_regroup_kernel, dim3(blocks), dim3(kEpThreads), 0, s, counts, W, E_loc, R,
                    static_cast<const uint4*>(in), static_cast<uint4*>(out), D / 8, dir,
                    chunk_size, offsets, active, num_active, chunk_offsets, num_chunks);
}

int ep_max_entries() { return kEpMaxEntries; }

}  // namespace moeq
