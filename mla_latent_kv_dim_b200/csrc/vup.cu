// V up-projection combine: y[b, h, :] = sum_j out[b, h, j] W_uv[h, j, :].
//
// In TPLA the shard outputs are combined by the existing o_proj all-reduce
// (feature request "Bandwidth-optimal tensor-parallel sharding of MLA",
// section "Directions under investigation"); with the G shard outputs laid
// side by side in latent space, the sum over shards is exactly the
// contraction over j here, so this kernel stands in for that all-reduce.
//
// Per head h this is a small GEMM [B x 512] x [512 x Dv].  It is bound by
// reading W_uv (H * 512 * Dv bf16) and out (B * H * 512 f32) once.  Tensor
// cores (bf16 in, f32 accumulate); an f32 `out` is split into hi + lo bf16
// terms, so the result keeps about 16 mantissa bits of `out`.
#include <cuda_bf16.h>
#include <stdint.h>

#include "internal.h"

namespace tpla {
namespace {

constexpr int kWarps = 4;
constexpr int kMTile = 16 * kWarps;  // rows of B per CTA
constexpr int kKChunk = 32;
constexpr int kRowWords = kKChunk / 2 + 4;  // padded smem row, 32-bit words

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}

template <int NT, bool OUT_BF16>  // NT = Dv / 8 n-tiles per warp
__global__ void __launch_bounds__(kWarps * 32)
vup_kernel(const void* __restrict__ outp, int64_t o_sb, int64_t o_sh,
           const __nv_bfloat16* __restrict__ W, int64_t w_sh, int64_t w_sj,
           float* __restrict__ y, int64_t y_sb, int64_t y_sh, int B) {
  constexpr int Dv = NT * 8;
  __shared__ uint32_t a_hi[kMTile][kRowWords];
  __shared__ uint32_t a_lo[kMTile][kRowWords];
  __shared__ uint32_t w_t[Dv][kRowWords];  // W chunk transposed: [n][k]

  const int h = blockIdx.y;
  const int m0 = blockIdx.x * kMTile;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, t4 = lane & 3;

  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;

  for (int k0 = 0; k0 < kLatent; k0 += kKChunk) {
    __syncthreads();
    // A chunk: kMTile rows x 32 k, split into hi/lo bf16 pairs
    for (int i = tid; i < kMTile * (kKChunk / 2); i += kWarps * 32) {
      int r = i / (kKChunk / 2), kp = i % (kKChunk / 2);
      int b = m0 + r;
      float x0 = 0.f, x1 = 0.f;
      if (b < B) {
        int64_t off = (int64_t)b * o_sb + (int64_t)h * o_sh + k0 + 2 * kp;
        if (OUT_BF16) {
          const __nv_bfloat16* o = reinterpret_cast<const __nv_bfloat16*>(outp) + off;
          x0 = __bfloat162float(o[0]);
          x1 = __bfloat162float(o[1]);
        } else {
          const float* o = reinterpret_cast<const float*>(outp) + off;
          x0 = o[0];
          x1 = o[1];
        }
      }
      __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
      a_hi[r][kp] = pack_bf16(h0, h1);
      if (!OUT_BF16)
        a_lo[r][kp] = pack_bf16(__float2bfloat16_rn(x0 - __bfloat162float(h0)),
                                __float2bfloat16_rn(x1 - __bfloat162float(h1)));
    }
    // W chunk: 32 k rows x Dv, stored transposed as [n][k] pairs
    for (int i = tid; i < (kKChunk / 2) * Dv; i += kWarps * 32) {
      int kp = i / Dv, n = i % Dv;
      const __nv_bfloat16* wp = W + (int64_t)h * w_sh + (int64_t)(k0 + 2 * kp) * w_sj + n;
      w_t[n][kp] = pack_bf16(wp[0], wp[w_sj]);
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kKChunk / 2; kk += 8) {  // two k16 steps (8 words each)
      const int ra = warp * 16 + gid;
      uint32_t ah[4] = {a_hi[ra][kk + t4], a_hi[ra + 8][kk + t4],
                        a_hi[ra][kk + 4 + t4], a_hi[ra + 8][kk + 4 + t4]};
      uint32_t al[4];
      if (!OUT_BF16) {
        al[0] = a_lo[ra][kk + t4];
        al[1] = a_lo[ra + 8][kk + t4];
        al[2] = a_lo[ra][kk + 4 + t4];
        al[3] = a_lo[ra + 8][kk + 4 + t4];
      }
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        uint32_t b0 = w_t[n * 8 + gid][kk + t4];
        uint32_t b1 = w_t[n * 8 + gid][kk + 4 + t4];
        mma_bf16_16816(acc[n], ah, b0, b1);
        if (!OUT_BF16) mma_bf16_16816(acc[n], al, b0, b1);
      }
    }
  }
  const int r0 = m0 + warp * 16 + gid;
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    int c = n * 8 + 2 * t4;
    if (r0 < B) {
      float* yp = y + (int64_t)r0 * y_sb + (int64_t)h * y_sh + c;
      yp[0] = acc[n][0];
      yp[1] = acc[n][1];
    }
    if (r0 + 8 < B) {
      float* yp = y + (int64_t)(r0 + 8) * y_sb + (int64_t)h * y_sh + c;
      yp[0] = acc[n][2];
      yp[1] = acc[n][3];
    }
  }
}

template <int NT>
cudaError_t launch_nt(const void* o, int out_bf16, int64_t o_sb, int64_t o_sh,
                      const __nv_bfloat16* W, int64_t w_sh, int64_t w_sj, float* y,
                      int64_t y_sb, int64_t y_sh, int B, int H, cudaStream_t stream) {
  dim3 grid((B + kMTile - 1) / kMTile, H);
  if (out_bf16)
    vup_kernel<NT, true><<<grid, kWarps * 32, 0, stream>>>(o, o_sb, o_sh, W, w_sh, w_sj, y,
                                                           y_sb, y_sh, B);
  else
    vup_kernel<NT, false><<<grid, kWarps * 32, 0, stream>>>(o, o_sb, o_sh, W, w_sh, w_sj, y,
                                                            y_sb, y_sh, B);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_vup(const void* out_latent, int out_bf16, int64_t o_sb, int64_t o_sh,
                       const void* W, int64_t w_sh, int64_t w_sj, float* y,
                       int64_t y_sb, int64_t y_sh, int B, int H, int Dv,
                       cudaStream_t stream) {
  if (B == 0 || H == 0 || Dv == 0) return cudaSuccess;
  const __nv_bfloat16* w = reinterpret_cast<const __nv_bfloat16*>(W);
  switch (Dv) {
#define TPLA_VUP_CASE(D) \
  case D: return launch_nt<D / 8>(out_latent, out_bf16, o_sb, o_sh, w, w_sh, w_sj, y, y_sb, y_sh, B, H, stream);
    TPLA_VUP_CASE(16) TPLA_VUP_CASE(32) TPLA_VUP_CASE(48) TPLA_VUP_CASE(64)
    TPLA_VUP_CASE(80) TPLA_VUP_CASE(96) TPLA_VUP_CASE(112) TPLA_VUP_CASE(128)
    TPLA_VUP_CASE(144) TPLA_VUP_CASE(160) TPLA_VUP_CASE(176) TPLA_VUP_CASE(192)
    TPLA_VUP_CASE(208) TPLA_VUP_CASE(224) TPLA_VUP_CASE(240) TPLA_VUP_CASE(256)
#undef TPLA_VUP_CASE
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tpla
