// In-place orthonormal fast Walsh-Hadamard transform of row prefixes.
//
// The orthogonal reparameterisation applied to the latent before TPLA
// slicing (feature request "Bandwidth-optimal tensor-parallel sharding of
// MLA", section "Directions under investigation"; TPLA abstract: a Hadamard
// transform before TP slicing mitigates cross-shard interference).  The
// transform is the Sylvester (natural-order) matrix scaled by 1/sqrt(dim);
// it is symmetric and orthogonal, so applying it twice restores the input.
//
// One warp owns one row.  Lane l holds the E = dim/32 contiguous elements
// [l*E, l*E + E) in registers: butterflies with stride < E stay inside a
// lane, strides >= E pair lane l with lane l ^ (stride / E) via shuffles.
// The row is read and written exactly once (HBM-bound).
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"

namespace tpla {
namespace {

constexpr int kWarps = 8;

struct RowMap {
  int64_t rows;
  int64_t n1, n2;       // sizes of the two innermost row dimensions
  int64_t s0, s1, s2;   // strides of up to three row dimensions (outer..inner)
};

__device__ __forceinline__ int64_t row_offset(const RowMap& m, int64_t r) {
  int64_t i2 = r % m.n2;
  int64_t t = r / m.n2;
  int64_t i1 = t % m.n1;
  int64_t i0 = t / m.n1;
  return i0 * m.s0 + i1 * m.s1 + i2 * m.s2;
}

template <int E, bool BF16>
__global__ void __launch_bounds__(kWarps * 32)
hadamard_kernel(void* buf, RowMap m, float norm, bool vec_ok) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (r >= m.rows) return;
  const int64_t off = row_offset(m, r) + (int64_t)lane * E;
  float x[E];
  if (BF16) {
    __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(buf) + off;
    if (vec_ok && (E % 8) == 0) {
#pragma unroll
      for (int i = 0; i < E; i += 8) {
        uint4 v = *reinterpret_cast<const uint4*>(p + i);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float2 f = __bfloat1622float2(h2[j]);
          x[i + 2 * j] = f.x;
          x[i + 2 * j + 1] = f.y;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < E; ++i) x[i] = __bfloat162float(p[i]);
    }
  } else {
    float* p = reinterpret_cast<float*>(buf) + off;
    if (vec_ok && (E % 4) == 0) {
#pragma unroll
      for (int i = 0; i < E; i += 4) {
        float4 v = *reinterpret_cast<const float4*>(p + i);
        x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < E; ++i) x[i] = p[i];
    }
  }
  // in-lane butterflies
#pragma unroll
  for (int s = 1; s < E; s <<= 1) {
#pragma unroll
    for (int i = 0; i < E; ++i) {
      if ((i & s) == 0) {
        float a = x[i], c = x[i + s];
        x[i] = a + c;
        x[i + s] = a - c;
      }
    }
  }
  // cross-lane butterflies: stride s*E pairs lane with lane ^ s
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      float other = __shfl_xor_sync(0xffffffffu, x[i], s);
      x[i] = upper ? other - x[i] : x[i] + other;
    }
  }
  if (BF16) {
    __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(buf) + off;
    if (vec_ok && (E % 8) == 0) {
#pragma unroll
      for (int i = 0; i < E; i += 8) {
        uint4 v;
        __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          h2[j] = __floats2bfloat162_rn(x[i + 2 * j] * norm, x[i + 2 * j + 1] * norm);
        *reinterpret_cast<uint4*>(p + i) = v;
      }
    } else {
#pragma unroll
      for (int i = 0; i < E; ++i) p[i] = __float2bfloat16_rn(x[i] * norm);
    }
  } else {
    float* p = reinterpret_cast<float*>(buf) + off;
#pragma unroll
    for (int i = 0; i < E; ++i) p[i] = x[i] * norm;
  }
}

template <int E>
cudaError_t launch_e(void* buf, bool bf16, const RowMap& m, float norm, bool vec_ok,
                     cudaStream_t stream) {
  int64_t blocks = (m.rows + kWarps - 1) / kWarps;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (bf16)
    hadamard_kernel<E, true><<<(unsigned)blocks, kWarps * 32, 0, stream>>>(buf, m, norm, vec_ok);
  else
    hadamard_kernel<E, false><<<(unsigned)blocks, kWarps * 32, 0, stream>>>(buf, m, norm, vec_ok);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_hadamard(void* buf, int bf16, int ndim, const int64_t* shape,
                            const int64_t* stride, int dim, cudaStream_t stream) {
  RowMap m{};
  // row dimensions are all but the innermost; pad to three
  int64_t sz[3] = {1, 1, 1}, st[3] = {0, 0, 0};
  int nr = ndim - 1;
  for (int i = 0; i < nr; ++i) {
    sz[3 - nr + i] = shape[i];
    st[3 - nr + i] = stride[i];
  }
  m.rows = sz[0] * sz[1] * sz[2];
  m.n1 = sz[1];
  m.n2 = sz[2];
  m.s0 = st[0];
  m.s1 = st[1];
  m.s2 = st[2];
  if (m.rows == 0) return cudaSuccess;
  const int esize = bf16 ? 2 : 4;
  bool vec_ok = (reinterpret_cast<uintptr_t>(buf) % 16) == 0;
  for (int i = 0; i < 3; ++i)
    if (sz[i] > 1 && (st[i] * esize) % 16 != 0) vec_ok = false;
  if (((dim / 32) * esize) % 16 != 0) vec_ok = false;
  const float norm = (float)(1.0 / sqrt((double)dim));
  switch (dim) {
    case 32: return launch_e<1>(buf, bf16, m, norm, vec_ok, stream);
    case 64: return launch_e<2>(buf, bf16, m, norm, vec_ok, stream);
    case 128: return launch_e<4>(buf, bf16, m, norm, vec_ok, stream);
    case 256: return launch_e<8>(buf, bf16, m, norm, vec_ok, stream);
    case 512: return launch_e<16>(buf, bf16, m, norm, vec_ok, stream);
    case 1024: return launch_e<32>(buf, bf16, m, norm, vec_ok, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tpla
