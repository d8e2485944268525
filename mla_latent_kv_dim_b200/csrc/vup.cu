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
//
// The tiled kernel (16-byte aligned operands) gives every CTA a 64 x 64
// output tile of one head, streams K in chunks of 64 with the next chunk's
// global loads in flight while the current one is multiplied, and reads
// fragments with ldmatrix from padded (conflict-free) shared-memory rows.
// Other layouts take the element-wise kernel.
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

// ---------------------------------------------------------------- tiled kernel

constexpr int kTM = 64, kTN = 64, kTK = 64;  // CTA tile: rows of B, columns of Dv, K chunk
constexpr int kTRow = kTK + 8;               // padded smem row (bf16): 144 bytes

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

template <bool OUT_BF16>
__global__ void __launch_bounds__(128)
vup_tiled_kernel(const void* __restrict__ outp, int64_t o_sb, int64_t o_sh,
                 const __nv_bfloat16* __restrict__ W, int64_t w_sh, int64_t w_sj,
                 float* __restrict__ y, int64_t y_sb, int64_t y_sh, int B, int Dv) {
  __shared__ __align__(16) __nv_bfloat16 a_hi[kTM][kTRow];
  __shared__ __align__(16) __nv_bfloat16 a_lo[OUT_BF16 ? 1 : kTM][kTRow];
  __shared__ __align__(16) __nv_bfloat16 w_s[kTK][kTRow];  // [k][n]

  const int m0 = blockIdx.x * kTM, h = blockIdx.y, n0 = blockIdx.z * kTN;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, t4 = lane & 3;

  // per-thread share of one K chunk
  constexpr int kAVec = OUT_BF16 ? (kTM * kTK / 8) / 128 : (kTM * kTK / 4) / 128;  // 4 or 8
  constexpr int kWVec = (kTK * kTN / 8) / 128;                                      // 4
  uint4 ra[kAVec], rw[kWVec];

  auto load_chunk = [&](int k0) {
#pragma unroll
    for (int i = 0; i < kAVec; ++i) {
      const int idx = tid + 128 * i;
      const int row = OUT_BF16 ? idx / 8 : idx / 16;
      const int col = OUT_BF16 ? 8 * (idx % 8) : 4 * (idx % 16);
      const int b = m0 + row;
      ra[i] = make_uint4(0, 0, 0, 0);
      if (b < B) {
        const int64_t off = (int64_t)b * o_sb + (int64_t)h * o_sh + k0 + col;
        ra[i] = OUT_BF16 ? *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(outp) + off)
                         : *reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(outp) + off);
      }
    }
#pragma unroll
    for (int i = 0; i < kWVec; ++i) {
      const int idx = tid + 128 * i;
      const int kr = idx / 8, n = n0 + 8 * (idx % 8);
      rw[i] = make_uint4(0, 0, 0, 0);
      if (n < Dv)
        rw[i] = *reinterpret_cast<const uint4*>(W + (int64_t)h * w_sh + (int64_t)(k0 + kr) * w_sj + n);
    }
  };
  auto store_chunk = [&]() {
#pragma unroll
    for (int i = 0; i < kAVec; ++i) {
      const int idx = tid + 128 * i;
      if (OUT_BF16) {
        *reinterpret_cast<uint4*>(&a_hi[idx / 8][8 * (idx % 8)]) = ra[i];
      } else {
        const int row = idx / 16, col = 4 * (idx % 16);
        const float f[4] = {__uint_as_float(ra[i].x), __uint_as_float(ra[i].y),
                            __uint_as_float(ra[i].z), __uint_as_float(ra[i].w)};
        uint32_t hi[2], lo[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const __nv_bfloat16 h0 = __float2bfloat16_rn(f[2 * e]), h1 = __float2bfloat16_rn(f[2 * e + 1]);
          hi[e] = pack_bf16(h0, h1);
          lo[e] = pack_bf16(__float2bfloat16_rn(f[2 * e] - __bfloat162float(h0)),
                            __float2bfloat16_rn(f[2 * e + 1] - __bfloat162float(h1)));
        }
        *reinterpret_cast<uint2*>(&a_hi[row][col]) = make_uint2(hi[0], hi[1]);
        *reinterpret_cast<uint2*>(&a_lo[row][col]) = make_uint2(lo[0], lo[1]);
      }
    }
#pragma unroll
    for (int i = 0; i < kWVec; ++i) {
      const int idx = tid + 128 * i;
      *reinterpret_cast<uint4*>(&w_s[idx / 8][8 * (idx % 8)]) = rw[i];
    }
  };

  float acc[8][4];
#pragma unroll
  for (int n = 0; n < 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;

  load_chunk(0);
  for (int k0 = 0; k0 < kLatent; k0 += kTK) {
    __syncthreads();  // previous chunk's fragments are read
    store_chunk();
    __syncthreads();
    if (k0 + kTK < kLatent) load_chunk(k0 + kTK);  // in flight during the MMAs below
#pragma unroll
    for (int kk = 0; kk < kTK; kk += 16) {
      const int ar = 16 * warp + (lane & 15), ac = kk + 8 * (lane >> 4);
      uint32_t ah[4], al[4];
      ldsm_x4(smem_u32(&a_hi[ar][ac]), ah[0], ah[1], ah[2], ah[3]);
      if (!OUT_BF16) ldsm_x4(smem_u32(&a_lo[ar][ac]), al[0], al[1], al[2], al[3]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {  // two n-tiles of 8 per ldmatrix
        const int wr = kk + (lane & 7) + 8 * ((lane >> 3) & 1), wc = 16 * np + 8 * (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(&w_s[wr][wc]), b0, b1, b2, b3);
        mma_bf16_16816(acc[2 * np], ah, b0, b1);
        mma_bf16_16816(acc[2 * np + 1], ah, b2, b3);
        if (!OUT_BF16) {
          mma_bf16_16816(acc[2 * np], al, b0, b1);
          mma_bf16_16816(acc[2 * np + 1], al, b2, b3);
        }
      }
    }
  }
  const int r0 = m0 + 16 * warp + gid;
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    const int c = n0 + 8 * n + 2 * t4;
    if (c >= Dv) continue;
    if (r0 < B)
      *reinterpret_cast<float2*>(y + (int64_t)r0 * y_sb + (int64_t)h * y_sh + c) =
          make_float2(acc[n][0], acc[n][1]);
    if (r0 + 8 < B)
      *reinterpret_cast<float2*>(y + (int64_t)(r0 + 8) * y_sb + (int64_t)h * y_sh + c) =
          make_float2(acc[n][2], acc[n][3]);
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
  const int ovec = out_bf16 ? 8 : 4;  // elements per 16 bytes
  const bool tiled = (reinterpret_cast<uintptr_t>(out_latent) & 15u) == 0 &&
                     (reinterpret_cast<uintptr_t>(W) & 15u) == 0 &&
                     (reinterpret_cast<uintptr_t>(y) & 7u) == 0 && o_sb % ovec == 0 &&
                     o_sh % ovec == 0 && w_sh % 8 == 0 && w_sj % 8 == 0 && y_sb % 2 == 0 &&
                     y_sh % 2 == 0;
  if (tiled) {
    dim3 grid((B + kTM - 1) / kTM, H, (Dv + kTN - 1) / kTN);
    if (out_bf16)
      vup_tiled_kernel<true><<<grid, 128, 0, stream>>>(out_latent, o_sb, o_sh, w, w_sh, w_sj, y,
                                                       y_sb, y_sh, B, Dv);
    else
      vup_tiled_kernel<false><<<grid, 128, 0, stream>>>(out_latent, o_sb, o_sh, w, w_sh, w_sj, y,
                                                        y_sb, y_sh, B, Dv);
    count_launch();
    return cudaGetLastError();
  }
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
