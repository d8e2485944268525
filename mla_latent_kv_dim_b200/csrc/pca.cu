// PCA reparameterisation of the latent: calibration statistics and the
// rotation x -> x U applied before TP slicing.
//
// The TPLA abstract and the feature request ("Directions under
// investigation") name PCA beside the Hadamard transform as the orthogonal
// change of basis applied to the latent before it is cut into shards; the
// pith.science review of the TPLA paper (referee report, comments on
// Sec. 4.3.2 and Eq. 25) places the PCA on the latent cache features with the
// position (rope) part excluded.  The basis U holds the covariance's
// eigenvectors; the eigensolve of the 512 x 512 matrix is offline work for
// the caller.  This file computes the statistics it needs over calibration
// rows and applies a given U to q or cache rows.
//
//  * latent_stats_kernel: C[i][j] += sum_r x_r[i] x_r[j] and s[i] += sum_r
//    x_r[i] over the 512 latent columns.  64 x 64 tiles of C per CTA, rows
//    streamed through shared memory in slices of 32, f32 FMA, one atomic add
//    per output at the end of a CTA's row chunk.  Calibration sets are small
//    (tens of thousands of rows), so plain FMA is enough.
//  * covariance_finalize_kernel: mean = s / n, cov = C / n - mean mean^T.
//  * rotation: the V-up kernel (the same contraction: the rows play the
//    requests of one head, U's two 256-column halves the V dimension) writes
//    x U in f32 to caller scratch; a store kernel rounds it to bf16 back into
//    the rows.  Both halves read every source row of a chunk before the store
//    of that chunk starts (stream order), so the rotation is in place.
#include <cuda_bf16.h>
#include <stdint.h>

#include "internal.h"

namespace tpla {
namespace {

constexpr int kStatTile = 64;     // C tile edge
constexpr int kStatSlice = 32;    // rows per shared-memory slice
constexpr int kStatChunk = 2048;  // rows per CTA
constexpr int kStatThreads = 256;

// Row r of a [B, H, >= 512] view (H = 1 for two-dimensional inputs).
__device__ __forceinline__ int64_t row_offset(int64_t r, int64_t H, int64_t sb, int64_t sh) {
  return (r / H) * sb + (r % H) * sh;
}

__global__ void __launch_bounds__(kStatThreads)
latent_stats_kernel(const __nv_bfloat16* __restrict__ x, int64_t nrows, int64_t H, int64_t sb,
                    int64_t sh, float* __restrict__ C, int64_t c_s0, float* __restrict__ s) {
  __shared__ float xi[kStatSlice][kStatTile];
  __shared__ float xj[kStatSlice][kStatTile];
  const int i0 = blockIdx.x * kStatTile, j0 = blockIdx.y * kStatTile;
  const int64_t r_begin = (int64_t)blockIdx.z * kStatChunk;
  const int64_t r_end = min(nrows, r_begin + kStatChunk);
  const int tid = threadIdx.x;
  const int ti = tid / 16, tj = tid % 16;  // 4 x 4 outputs each
  const bool sums = blockIdx.y == 0;       // one CTA column adds the column sums
  float acc[4][4] = {};
  float colsum = 0.f;
  for (int64_t r0 = r_begin; r0 < r_end; r0 += kStatSlice) {
    __syncthreads();
    // 32 rows x 64 columns per tile: 8 values of each tile per thread
    for (int e = tid; e < kStatSlice * kStatTile; e += kStatThreads) {
      const int rr = e / kStatTile, cc = e % kStatTile;
      const int64_t r = r0 + rr;
      float a = 0.f, b = 0.f;
      if (r < r_end) {
        const int64_t off = row_offset(r, H, sb, sh);
        a = __bfloat162float(x[off + i0 + cc]);
        b = __bfloat162float(x[off + j0 + cc]);
      }
      xi[rr][cc] = a;
      xj[rr][cc] = b;
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < kStatSlice; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = xi[k][4 * ti + u];
        b[u] = xj[k][4 * tj + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
    if (sums && tid < kStatTile) {
      for (int k = 0; k < kStatSlice; ++k) colsum += xi[k][tid];
    }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v)
      atomicAdd(&C[(int64_t)(i0 + 4 * ti + u) * c_s0 + j0 + 4 * tj + v], acc[u][v]);
  if (sums && tid < kStatTile) atomicAdd(&s[i0 + tid], colsum);
}

__global__ void covariance_finalize_kernel(const float* __restrict__ C, int64_t c_s0,
                                           const float* __restrict__ s, double n,
                                           float* __restrict__ cov, int64_t v_s0,
                                           float* __restrict__ mean) {
  const int i = blockIdx.x, j = threadIdx.x;  // 512 x 512
  const double mi = (double)s[i] / n, mj = (double)s[j] / n;
  cov[(int64_t)i * v_s0 + j] = (float)((double)C[(int64_t)i * c_s0 + j] / n - mi * mj);
  if (i == 0) mean[j] = (float)mj;
}

// dst rows [nb, H, >= 512] bf16 <- y [nb, H, 512] f32 (8 values per thread)
__global__ void store_rows_bf16_kernel(const float* __restrict__ y, int64_t nrows, int64_t H,
                                       __nv_bfloat16* __restrict__ dst, int64_t sb, int64_t sh) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t r = t / (kLatent / 8);
  const int c = 8 * (int)(t % (kLatent / 8));
  if (r >= nrows) return;
  const float4 a = *reinterpret_cast<const float4*>(y + r * kLatent + c);
  const float4 b = *reinterpret_cast<const float4*>(y + r * kLatent + c + 4);
  __nv_bfloat162 h[4] = {__floats2bfloat162_rn(a.x, a.y), __floats2bfloat162_rn(a.z, a.w),
                         __floats2bfloat162_rn(b.x, b.y), __floats2bfloat162_rn(b.z, b.w)};
  *reinterpret_cast<uint4*>(dst + row_offset(r, H, sb, sh) + c) = *reinterpret_cast<uint4*>(h);
}

}  // namespace

cudaError_t launch_latent_stats(const void* x, int64_t B, int64_t H, int64_t sb, int64_t sh,
                                float* C, int64_t c_s0, float* s, cudaStream_t stream) {
  const int64_t nrows = B * H;
  if (nrows == 0) return cudaSuccess;
  const int64_t chunks = (nrows + kStatChunk - 1) / kStatChunk;
  if (chunks > 65535) return cudaErrorInvalidValue;
  dim3 grid(kLatent / kStatTile, kLatent / kStatTile, (unsigned)chunks);
  latent_stats_kernel<<<grid, kStatThreads, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(x), nrows, H, sb, sh, C, c_s0, s);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_covariance_finalize(const float* C, int64_t c_s0, const float* s, int64_t n,
                                       float* cov, int64_t v_s0, float* mean,
                                       cudaStream_t stream) {
  if (n <= 0) return cudaErrorInvalidValue;
  covariance_finalize_kernel<<<kLatent, kLatent, 0, stream>>>(C, c_s0, s, (double)n, cov, v_s0,
                                                              mean);
  count_launch();
  return cudaGetLastError();
}

namespace {

// x U for rows [r0, r0 + n) of a uniformly strided row set (row r at
// x + r * rs), into scratch [n, 512] f32: the V-up kernel with one "head"
// whose rows are the requests, U's columns in two halves of 256.
cudaError_t rotate_rows_f32(const __nv_bfloat16* x, int64_t rs, int64_t n, const void* U,
                            float* scratch, cudaStream_t stream) {
  const __nv_bfloat16* u = reinterpret_cast<const __nv_bfloat16*>(U);
  for (int half = 0; half < 2; ++half) {
    cudaError_t e = launch_vup(x, 1, rs, rs, u + 256 * half, (int64_t)kLatent * kLatent,
                               kLatent, scratch + 256 * half, kLatent, kLatent, (int)n, 1, 256,
                               kLatent, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_rotate(void* x, int64_t B, int64_t H, int64_t sb, int64_t sh, const void* U,
                          float* scratch, int64_t chunk_b, cudaStream_t stream) {
  __nv_bfloat16* xb = reinterpret_cast<__nv_bfloat16*>(x);
  const bool uniform = H == 1 || sb == H * sh;  // rows evenly spaced across b
  const int64_t rs = H == 1 ? sb : sh;
  // one V-up launch covers at most 65535 tiles of 64 rows
  const int64_t max_rows = (int64_t)65535 * 64;
  for (int64_t b0 = 0; b0 < B; b0 += chunk_b) {
    const int64_t nb = B - b0 < chunk_b ? B - b0 : chunk_b;
    cudaError_t e = cudaSuccess;
    if (uniform) {
      for (int64_t r0 = 0; r0 < nb * H && e == cudaSuccess; r0 += max_rows) {
        const int64_t n = nb * H - r0 < max_rows ? nb * H - r0 : max_rows;
        e = rotate_rows_f32(xb + b0 * sb + r0 * rs, rs, n, U, scratch + r0 * kLatent, stream);
      }
    } else {
      for (int64_t b = 0; b < nb && e == cudaSuccess; ++b)
        e = rotate_rows_f32(xb + (b0 + b) * sb, sh, H, U, scratch + b * H * kLatent, stream);
    }
    if (e != cudaSuccess) return e;
    const int64_t threads = nb * H * (kLatent / 8);
    const int64_t blocks = (threads + 255) / 256;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    store_rows_bf16_kernel<<<(unsigned)blocks, 256, 0, stream>>>(scratch, nb * H, H, xb + b0 * sb,
                                                                  sb, sh);
    count_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace tpla
