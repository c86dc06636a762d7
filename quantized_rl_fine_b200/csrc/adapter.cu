// BF16 block-diagonal adapter on the activations (per expert, 32 x 32 blocks).
//
// Orbit issue #1: the trainable adapter is orthogonal fine-tuning applied on
// top of a quantized base that is never dequantized into storage. Its form
// here is one block-diagonal d x d matrix R_e per expert:
//   forward   x'[p][32b+j] = sum_i x[p][32b+i] * R[e][b][i][j]
//   backward  dx[p][32b+i] = sum_j dx'[p][32b+j] * R[e][b][i][j]
//             dR[e][b][i][j] = sum over rows p of expert e of x[p][32b+i] * dx'[p][32b+j]
// Both kernels multiply on the warp-level tensor-core MMA (mma.sync m16n8k16:
// BF16 operands, exact products, FP32 accumulation): the operation moves each
// element of x once, and 32 multiply-adds per element on the FP32 pipes take
// longer than that. dR is accumulated in ascending row order by one warp per
// (expert, block) pair, so it is deterministic.
#include "launchers.cuh"
#include "common.cuh"

namespace moeq {

namespace {

// d (16 x 8, FP32) += a (16 x 16, BF16, row-major) * b (16 x 8, BF16, column-major).
// Fragments (g = lane / 4, t = lane % 4): a = rows g and g + 8 at k pairs 2t and
// 2t + 8 ({row g, k 2t}, {row g + 8, k 2t}, {row g, k 2t + 8}, {row g + 8, k 2t + 8});
// b = column g at k pairs 2t and 2t + 8; d = rows g and g + 8 at columns 2t, 2t + 1.
// A pair packs the lower k (or column) in the low 16 bits.
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t ldg_u32(const __nv_bfloat16* p) {
  return __ldg(reinterpret_cast<const unsigned int*>(p));
}

__device__ __forceinline__ uint32_t ldg_u16(const __nv_bfloat16* p) {
  return __ldg(reinterpret_cast<const unsigned short*>(p));
}

// Largest e with offsets[e] <= row, for 0 <= row < offsets[E] (offsets nondecreasing).
__device__ __forceinline__ int expert_of_row(const int32_t* offsets, int E, int row) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(offsets + mid) <= row) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The same for a row at or after one whose expert e is known: step forward.
__device__ __forceinline__ int expert_of_row_from(const int32_t* offsets, int E, int e, int row) {
  while (e + 1 < E && __ldg(offsets + e + 1) <= row) ++e;
  return e;
}

constexpr int kApplyGroups = 4;   // 16-row groups per warp task of the apply kernel
constexpr int kStageLd = 40;      // staged row length in BF16 (80 bytes: conflict-free ldmatrix)

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// The expert's R block (e, b) as B fragments of the four 8-column tiles and two
// 16-deep k steps: TRANS = 0 multiplies by R_e (B[k][n] = R[k][n]), 1 by R_e^T
// (B[k][n] = R[n][k]).
template <int TRANS>
__device__ __forceinline__ void load_r_frags(const __nv_bfloat16* __restrict__ Rb, int g, int t,
                                             uint32_t (&bf)[4][2][2]) {
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (TRANS) {
        // row 8 nt + g of R, k pairs 16 s + 2t and + 8
        const __nv_bfloat16* c = Rb + (8 * nt + g) * 32 + 16 * s + 2 * t;
        bf[nt][s][0] = ldg_u32(c);
        bf[nt][s][1] = ldg_u32(c + 8);
      } else {
        // column 8 nt + g of R, rows 16 s + 2t (+1) and + 8 (+9)
        const __nv_bfloat16* c = Rb + (16 * s + 2 * t) * 32 + 8 * nt + g;
        bf[nt][s][0] = ldg_u16(c) | (ldg_u16(c + 32) << 16);
        bf[nt][s][1] = ldg_u16(c + 256) | (ldg_u16(c + 288) << 16);
      }
    }
}

// One warp task: 64 rows (four 16-row groups) x one 32-column block b; eight
// tasks per 256-thread CTA, consecutive tasks on consecutive blocks of the same
// rows. The warp copies the task's x columns into shared memory with 16-byte
// loads (4 KiB in flight), takes the A fragments from there with matrix
// loads, and stages the results the same way for 16-byte stores. The
// expert's R block, as B fragments, stays in registers while the rows'
// expert does not change; a group whose rows span several experts runs the
// MMAs once per expert and keeps each row's result from its own expert.
// TRANS = 0: out = x . R_e; 1: out = x . R_e^T. With rows (not NULL) the
// task's row p reads x[rows[p]] (the permuted rows are gathered from the token
// rows here, so they are never written out).
template <int TRANS>
__global__ void __launch_bounds__(256)
adapter_apply_kernel(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ rows,
                     const __nv_bfloat16* __restrict__ R,
                     const int32_t* __restrict__ offsets, int E, int M, int K,
                     __nv_bfloat16* __restrict__ out) {
  grid_dependency_wait();
  grid_dependents_launch();
  __shared__ __align__(16) uint16_t tile[8][16 * kApplyGroups][kStageLd];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int nb = K / 32;
  const int64_t task = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  const int64_t n_spans = (static_cast<int64_t>(M) + 16 * kApplyGroups - 1) / (16 * kApplyGroups);
  if (task >= n_spans * nb) return;
  const int b = static_cast<int>(task % nb);
  const int span0 = static_cast<int>(task / nb) * 16 * kApplyGroups;
  uint16_t (*tl)[kStageLd] = tile[warp];
  // 64 rows x 4 chunks of 16 bytes: eight per lane; rows past M read as zero.
  {
    uint4 v[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const int idx = lane + 32 * h, row = idx >> 2, ch = idx & 3;
      const int r = span0 + row;
      const int64_t src = (r < M) ? (rows ? __ldg(rows + r) : r) : 0;
      v[h] = (r < M) ? __ldg(reinterpret_cast<const uint4*>(x + src * K + 32 * b + 8 * ch))
                     : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const int idx = lane + 32 * h, row = idx >> 2, ch = idx & 3;
      *reinterpret_cast<uint4*>(&tl[row][8 * ch]) = v[h];
    }
  }
  __syncwarp();
  const uint32_t tl0 = smem_u32(&tl[0][0]);
  const int m = lane >> 3, mr = lane & 7;   // ldmatrix: matrix m, its row mr
  int cached = -1;
  // Expert of the task's first row (one search); the groups step forward from it.
  int e_run = expert_of_row(offsets, E, span0);
  uint32_t bf[4][2][2];
  for (int q = 0; q < kApplyGroups; ++q) {
    const int r0 = span0 + 16 * q;
    if (r0 >= M) break;
    // A fragments of the group: rows 16 q + (0-7 | 8-15), k 0-7 | 8-15 of step s.
    uint32_t a[2][4];
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int row = 16 * q + 8 * (m & 1) + mr, col = 16 * s + 8 * (m >> 1);
      ldsm_x4(tl0 + (row * kStageLd + col) * 2, a[s][0], a[s][1], a[s][2], a[s][3]);
    }
    const int ra = r0 + g, rb = ra + 8;
    const int e_first = expert_of_row_from(offsets, E, e_run, r0);
    const int e_last = expert_of_row_from(offsets, E, e_first, min(r0 + 15, M - 1));
    e_run = e_last;
    float res[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) res[nt][c] = 0.0f;
    for (int e = e_first; e <= e_last; ++e) {
      const int p0 = __ldg(offsets + e), p1 = __ldg(offsets + e + 1);
      if (p0 == p1) continue;
      if (e != cached) {
        load_r_frags<TRANS>(R + (static_cast<int64_t>(e) * nb + b) * 1024, g, t, bf);
        cached = e;
      }
      const bool ina = ra >= p0 && ra < p1, inb = rb >= p0 && rb < p1;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        mma16816(d, a[0], bf[nt][0][0], bf[nt][0][1]);
        mma16816(d, a[1], bf[nt][1][0], bf[nt][1][1]);
        if (ina) { res[nt][0] = d[0]; res[nt][1] = d[1]; }
        if (inb) { res[nt][2] = d[2]; res[nt][3] = d[3]; }
      }
    }
    // The group's rows of x are no longer needed: stage the results in their place.
    __syncwarp();
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      *reinterpret_cast<uint32_t*>(&tl[16 * q + g][8 * nt + 2 * t]) = pack_bf16x2(res[nt][0], res[nt][1]);
      *reinterpret_cast<uint32_t*>(&tl[16 * q + g + 8][8 * nt + 2 * t]) = pack_bf16x2(res[nt][2], res[nt][3]);
    }
  }
  __syncwarp();
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    const int idx = lane + 32 * h, row = idx >> 2, ch = idx & 3;
    const int r = span0 + row;
    if (r < M)
      *reinterpret_cast<uint4*>(out + static_cast<int64_t>(r) * K + 32 * b + 8 * ch) =
          *reinterpret_cast<const uint4*>(&tl[row][8 * ch]);
  }
}

constexpr int kGradWarps = 8;     // column blocks per CTA of the gradient kernel (one warp each)
constexpr int kGradRows = 32;     // rows staged per step

// Backward, fused: grid (E, ceil(K / 256)), 256 threads. Warp (e, b) walks the
// rows of expert e in ascending order, 32 at a time: it stages the rows' x and
// dx' columns of block b in shared memory and from them forms both
//   dR[e][b] += x^T . dx'   (A = x^T, B = dx', both through transposing matrix loads)
//   dx = dx' . R_e^T        (A = dx' through plain matrix loads, R_e^T's block as
//                            B fragments held in registers),
// so dx' is read from HBM once for both. dx is staged where the x rows were
// and written with 16-byte stores.
__global__ void __launch_bounds__(256)
adapter_bwd_kernel(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ rows,
                   const __nv_bfloat16* __restrict__ dxp,
                   const __nv_bfloat16* __restrict__ R, const int32_t* __restrict__ offsets,
                   int K, __nv_bfloat16* __restrict__ dx, float* __restrict__ dR) {
  grid_dependency_wait();
  grid_dependents_launch();
  __shared__ __align__(16) uint16_t xs[kGradWarps][kGradRows][kStageLd];
  __shared__ __align__(16) uint16_t gs[kGradWarps][kGradRows][kStageLd];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int e = blockIdx.x;
  const int b = blockIdx.y * kGradWarps + warp;
  const int nb = K / 32;
  if (b >= nb) return;                   // warp-uniform; the warps never sync with each other
  const int p0 = offsets[e], p1 = offsets[e + 1];
  float acc[2][4][4];                    // dR: [i tile][j tile][fragment]
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[mi][nt][c] = 0.0f;
  uint32_t bf[4][2][2];                  // R_e^T's block (e, b) as B fragments
  if (p1 > p0) load_r_frags<1>(R + (static_cast<int64_t>(e) * nb + b) * 1024, g, t, bf);
  const uint32_t xs0 = smem_u32(&xs[warp][0][0]);
  const uint32_t gs0 = smem_u32(&gs[warp][0][0]);
  const int m = lane >> 3, mr = lane & 7;   // ldmatrix: matrix m, its row mr
  for (int c0 = p0; c0 < p1; c0 += kGradRows) {
    // 32 rows x 4 chunks of 16 bytes per operand: four chunks per lane.
    uint4 vx[4], vg[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int idx = lane + 32 * h, row = idx >> 2, ch = idx & 3;
      const bool ok = c0 + row < p1;
      const int pr = ok ? c0 + row : p0;
      const int64_t gi = static_cast<int64_t>(pr) * K + 32 * b + 8 * ch;
      const int64_t xi = (rows ? static_cast<int64_t>(__ldg(rows + pr)) : pr) * K + 32 * b + 8 * ch;
      vx[h] = ok ? __ldg(reinterpret_cast<const uint4*>(x + xi)) : make_uint4(0, 0, 0, 0);
      // dx' is read once and dx written once: streaming (evict-first) hints
      // on both (measured at the training shape, 384 experts x 85 rows:
      // 446 -> 415 us)
      vg[h] = ok ? __ldcs(reinterpret_cast<const uint4*>(dxp + gi)) : make_uint4(0, 0, 0, 0);
    }
    __syncwarp();                        // the previous step's stores from xs are done
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int idx = lane + 32 * h, row = idx >> 2, ch = idx & 3;
      *reinterpret_cast<uint4*>(&xs[warp][row][8 * ch]) = vx[h];
      *reinterpret_cast<uint4*>(&gs[warp][row][8 * ch]) = vg[h];
    }
    __syncwarp();
    // dR += x^T . dx' over the 32 staged rows (zeros past the expert).
#pragma unroll
    for (int s = 0; s < kGradRows / 16; ++s) {
      uint32_t af[2][4];
#pragma unroll
      for (int mi = 0; mi < 2; ++mi) {
        const int krow = 16 * s + 8 * (m >> 1) + mr;
        const int icol = 16 * mi + 8 * (m & 1);
        ldsm_x4_trans(xs0 + (krow * kStageLd + icol) * 2, af[mi][0], af[mi][1], af[mi][2], af[mi][3]);
      }
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        const int krow = 16 * s + 8 * (m & 1) + mr;
        const int jcol = 8 * (2 * np + (m >> 1));
        uint32_t b00, b01, b10, b11;
        ldsm_x4_trans(gs0 + (krow * kStageLd + jcol) * 2, b00, b01, b10, b11);
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
          mma16816(acc[mi][2 * np], af[mi], b00, b01);
          mma16816(acc[mi][2 * np + 1], af[mi], b10, b11);
        }
      }
    }
    // dx = dx' . R_e^T for the two 16-row groups.
    float res[2][4][4];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t a[2][4];
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int row = 16 * q + 8 * (m & 1) + mr, col = 16 * s + 8 * (m >> 1);
        ldsm_x4(gs0 + (row * kStageLd + col) * 2, a[s][0], a[s][1], a[s][2], a[s][3]);
      }
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
        for (int c = 0; c < 4; ++c) res[q][nt][c] = 0.0f;
        mma16816(res[q][nt], a[0], bf[nt][0][0], bf[nt][0][1]);
        mma16816(res[q][nt], a[1], bf[nt][1][0], bf[nt][1][1]);
      }
    }
    __syncwarp();                        // every matrix load from xs is done: reuse it for dx
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        *reinterpret_cast<uint32_t*>(&xs[warp][16 * q + g][8 * nt + 2 * t]) =
            pack_bf16x2(res[q][nt][0], res[q][nt][1]);
        *reinterpret_cast<uint32_t*>(&xs[warp][16 * q + g + 8][8 * nt + 2 * t]) =
            pack_bf16x2(res[q][nt][2], res[q][nt][3]);
      }
    __syncwarp();
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int idx = lane + 32 * h, row = idx >> 2, ch = idx & 3;
      if (c0 + row < p1)
        __stcs(reinterpret_cast<uint4*>(dx + static_cast<int64_t>(c0 + row) * K + 32 * b + 8 * ch),
               *reinterpret_cast<const uint4*>(&xs[warp][row][8 * ch]));
    }
  }
  float* dst = dR + (static_cast<int64_t>(e) * nb + b) * 1024;
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int i = 16 * mi + g, j = 8 * nt + 2 * t;
      *reinterpret_cast<float2*>(dst + i * 32 + j) = make_float2(acc[mi][nt][0], acc[mi][nt][1]);
      *reinterpret_cast<float2*>(dst + (i + 8) * 32 + j) = make_float2(acc[mi][nt][2], acc[mi][nt][3]);
    }
}

}  // namespace

cudaError_t launch_adapter_apply(const void* x, const int32_t* rows, const void* R,
                                 const int32_t* offsets, int E, int M, int K, void* out,
                                 cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  const int nb = K / 32;
  const int64_t spans = (static_cast<int64_t>(M) + 16 * kApplyGroups - 1) / (16 * kApplyGroups);
  const int64_t ctas = (spans * nb + 7) / 8;
  if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
  return launch_pdl(adapter_apply_kernel<0>, dim3(static_cast<unsigned>(ctas)), dim3(256), 0, s,
                    static_cast<const __nv_bfloat16*>(x), rows, static_cast<const __nv_bfloat16*>(R),
                    offsets, E, M, K, static_cast<__nv_bfloat16*>(out));
}

cudaError_t launch_adapter_bwd(const void* x, const int32_t* rows, const void* dxp, const void* R,
                               const int32_t* offsets, int E, int K, void* dx, float* dR,
                               cudaStream_t s) {
  const int nb = K / 32;
  dim3 grid(E, (nb + kGradWarps - 1) / kGradWarps);
  return launch_pdl(adapter_bwd_kernel, grid, dim3(256), 0, s,
                    static_cast<const __nv_bfloat16*>(x), rows, static_cast<const __nv_bfloat16*>(dxp),
                    static_cast<const __nv_bfloat16*>(R), offsets, K,
                    static_cast<__nv_bfloat16*>(dx), dR);
}

}  // namespace moeq
