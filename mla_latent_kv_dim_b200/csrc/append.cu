// Cache append: store each request's new token in the latent KV cache,
// normalised the way TPLA's shards read it.
//
// The stored latent is the RMS-normalised down-projection of the token (the
// norm's gain absorbed into the up-projections, like the orthogonal
// reparameterisation U; review of arXiv 2508.15881, key machinery).  With
// the latent cut into G tensor-parallel shards every rank normalises its own
// slice: Condition 1 of the review's key machinery asks the shard norms to
// be proportional to the global one, and a Hadamard rotation applied before
// slicing (feature request "Bandwidth-optimal tensor-parallel sharding of
// MLA", "Directions under investigation") spreads the energy evenly so that
// they nearly are.  Proposition 1 (RMSNorm commutes with an orthogonal
// transform) makes the one-group case with the rotation equal to the
// rotated exact-MLA row.
//
// One warp per request: lane l holds latent columns [16 l, 16 l + 16) in
// registers; the optional Walsh-Hadamard butterflies run in-lane and across
// lanes by shuffles (natural order, scaled by 1/sqrt(512)); each shard's
// sum of squares is a shuffle reduction over its 32/G lanes; the row is
// written once (bf16) at the request's position, the rope columns as given.
// Out-of-range positions or page ids are not written: the kernel records
// TPLA_ERR_DEVICE_BOUNDS in its status word.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"

namespace tpla {
namespace {

constexpr int kWarps = 8;
constexpr int kE = kLatent / 32;  // latent values per lane

__device__ int g_append_status;

struct AppendParams {
  const void* kv_new;
  int in_bf16;
  int64_t n_sb;
  const int* positions;  // nullptr: row b goes to position pos0 + b
  int pos0;
  const int* page_table;
  int64_t pt_sb;
  int max_pages;
  int64_t num_blocks;   // paged
  int64_t cap_rows;     // contiguous: rows per request
  __nv_bfloat16* cache;
  int64_t c_s0, c_s1;
  int B;
  int groups;
  int hadamard;
  float eps;
};

__global__ void __launch_bounds__(kWarps * 32) cache_append_kernel(const AppendParams p) {
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (b >= p.B) return;
  // destination row
  const int pos = p.positions ? p.positions[b] : p.pos0 + b;
  __nv_bfloat16* dst = nullptr;
  if (p.page_table) {
    if (pos >= 0 && pos < 64 * p.max_pages) {
      const int blk = p.page_table[(int64_t)b * p.pt_sb + pos / 64];
      if (blk >= 0 && blk < p.num_blocks)
        dst = p.cache + (int64_t)blk * p.c_s0 + (int64_t)(pos % 64) * p.c_s1;
    }
  } else if (pos >= 0 && pos < p.cap_rows) {
    dst = p.cache + (int64_t)b * p.c_s0 + (int64_t)pos * p.c_s1;
  }
  if (!dst) {
    if (lane == 0) atomicCAS(&g_append_status, 0, TPLA_ERR_DEVICE_BOUNDS);
    return;
  }
  // load: latent columns [16 lane, 16 lane + 16), rope columns 512 + 2 lane, + 1
  float x[kE], r[2];
  if (p.in_bf16) {
    const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(p.kv_new) + (int64_t)b * p.n_sb;
#pragma unroll
    for (int i = 0; i < kE; i += 8) {
      const uint4 v = *reinterpret_cast<const uint4*>(src + kE * lane + i);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(h[j]);
        x[i + 2 * j] = f.x;
        x[i + 2 * j + 1] = f.y;
      }
    }
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(src + kLatent + 2 * lane));
    r[0] = f.x;
    r[1] = f.y;
  } else {
    const float* src = reinterpret_cast<const float*>(p.kv_new) + (int64_t)b * p.n_sb;
#pragma unroll
    for (int i = 0; i < kE; i += 4) {
      const float4 v = *reinterpret_cast<const float4*>(src + kE * lane + i);
      x[i] = v.x;
      x[i + 1] = v.y;
      x[i + 2] = v.z;
      x[i + 3] = v.w;
    }
    const float2 v = *reinterpret_cast<const float2*>(src + kLatent + 2 * lane);
    r[0] = v.x;
    r[1] = v.y;
  }
  if (p.hadamard) {
    // butterflies of stride < 16 inside the lane, of stride 16 s across lanes l, l ^ s
#pragma unroll
    for (int s = 1; s < kE; s <<= 1) {
#pragma unroll
      for (int i = 0; i < kE; ++i) {
        if ((i & s) == 0) {
          const float a = x[i], c = x[i + s];
          x[i] = a + c;
          x[i + s] = a - c;
        }
      }
    }
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
      const bool upper = (lane & s) != 0;
#pragma unroll
      for (int i = 0; i < kE; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, x[i], s);
        x[i] = upper ? o - x[i] : x[i] + o;
      }
    }
    const float h = 0.044194173824159216f;  // 1 / sqrt(512)
#pragma unroll
    for (int i = 0; i < kE; ++i) x[i] *= h;
  }
  // mean square of this lane's shard: lanes [l - l % (32/G), + 32/G)
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kE; ++i) ss = fmaf(x[i], x[i], ss);
  const int span = 32 / p.groups;
  for (int o = 1; o < span; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float d = (float)(kLatent / p.groups);
  const float root = sqrtf(ss / d + p.eps);
  uint4 w[2];
  __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(w);
#pragma unroll
  for (int j = 0; j < kE / 2; ++j) h2[j] = __floats2bfloat162_rn(x[2 * j] / root, x[2 * j + 1] / root);
  *reinterpret_cast<uint4*>(dst + kE * lane) = w[0];
  *reinterpret_cast<uint4*>(dst + kE * lane + 8) = w[1];
  *reinterpret_cast<__nv_bfloat162*>(dst + kLatent + 2 * lane) = __floats2bfloat162_rn(r[0], r[1]);
}

}  // namespace

cudaError_t launch_cache_append(const void* kv_new, int in_bf16, int64_t n_sb, const int* positions,
                                int pos0, const int* page_table, int64_t pt_sb, int max_pages,
                                int64_t num_blocks, int64_t cap_rows, void* cache, int64_t c_s0,
                                int64_t c_s1, int B, int groups, int hadamard, float eps,
                                cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  AppendParams p{};
  p.kv_new = kv_new;
  p.in_bf16 = in_bf16;
  p.n_sb = n_sb;
  p.positions = positions;
  p.pos0 = pos0;
  p.page_table = page_table;
  p.pt_sb = pt_sb;
  p.max_pages = max_pages;
  p.num_blocks = num_blocks;
  p.cap_rows = cap_rows;
  p.cache = reinterpret_cast<__nv_bfloat16*>(cache);
  p.c_s0 = c_s0;
  p.c_s1 = c_s1;
  p.B = B;
  p.groups = groups;
  p.hadamard = hadamard;
  p.eps = eps;
  cache_append_kernel<<<(B + kWarps - 1) / kWarps, kWarps * 32, 0, stream>>>(p);
  count_launch();
  return cudaGetLastError();
}

cudaError_t status_read_clear_append(int* code) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_append_status, sizeof(int));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    int zero = 0;
    e = cudaMemcpyToSymbol(g_append_status, &zero, sizeof(int));
  }
  *code = v;
  return e;
}

}  // namespace tpla
