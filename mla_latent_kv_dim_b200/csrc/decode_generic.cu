// Portable CUDA-core MLA / TPLA decode kernel.
//
// One CTA computes, for one request b, one shard g, one group of 16 heads
// and one chunk of the request's tokens, the shard-local softmax attention
//   s_t = scale * (q[I_g] . c_t[I_g] + q[R_g] . c_t[R_g]),
//   out[I_g] = sum_t softmax(s)_t c_t[I_g],   lse = ln sum_t exp(s_t)
// (TPLA: per-shard softmax over the shard's latent slice plus its rope
// columns, as in the feature request "Bandwidth-optimal tensor-parallel
// sharding of MLA", section "Directions under investigation", and the
// review's description of Eq. 6 as an unscaled local softmax).  Tokens are
// streamed in tiles of 32 with the usual running-max / running-sum
// recurrence; chunks of a split request are merged afterwards by the
// log-sum-exp rule (tpla_lse_merge).
//
// This kernel covers every shape the API accepts (any G, either rope mode,
// one-shard mode, paged or contiguous caches); the tcgen05 kernel is the
// fast path for the shapes it supports.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"

namespace tpla {
namespace {

constexpr int kHG = 16;        // heads per CTA
constexpr int kTT = 32;        // tokens per tile
constexpr int kThreads = 256;
constexpr int kMaxK = kWidth;  // widest shard key (G = 1)

__device__ int g_status;       // first device-side error of this unit

__device__ __forceinline__ void set_status(int code) {
  atomicCAS(&g_status, 0, code);
}

__device__ __forceinline__ float ld_bf16(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

struct SmemGeneric {
  float q[kHG][kMaxK];
  float kv[kTT][kMaxK + 1];   // +1: conflict-free column access
  float s[kHG][kTT];
  float alpha[kHG];
  int valid[kTT];
};

__global__ void __launch_bounds__(kThreads)
decode_generic_kernel(DecodeProblem p, int splits, int chunk, float* o_part,
                      float* lse_part) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SmemGeneric& sm = *reinterpret_cast<SmemGeneric*>(smem_raw);

  const int tid = threadIdx.x;
  const int h0 = blockIdx.x * kHG;
  const int split = blockIdx.y;
  const int b = blockIdx.z / p.n_shards;
  const int k = blockIdx.z % p.n_shards;
  const int g = p.shard < 0 ? k : p.shard;

  const int d = kLatent / p.G;
  const int r = p.rope_mode == TPLA_ROPE_REPLICATE ? kRope : kRope / p.G;
  const int rope0 = p.rope_mode == TPLA_ROPE_REPLICATE ? kLatent : kLatent + g * r;
  const int lat0 = g * d;
  const int Kd = d + r;

  int L = p.seq_lens[b];
  int64_t cap = p.cache_rows;
  if (L < 0 || (int64_t)L > cap) {
    set_status(TPLA_ERR_DEVICE_BOUNDS);
    L = L < 0 ? 0 : (int)cap;
  }
  const int t_begin = split * chunk;
  const int t_end = min(L, t_begin + chunk);

  // query rows of this head group, shard columns only (f32)
  const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(p.q);
  for (int i = tid; i < kHG * Kd; i += kThreads) {
    int hh = i / Kd, c = i % Kd;
    int h = h0 + hh;
    int col = c < d ? lat0 + c : rope0 + (c - d);
    sm.q[hh][c] = h < p.H ? ld_bf16(qb + b * p.q_sb + (int64_t)h * p.q_sh + col) : 0.f;
  }

  // per-thread output slice: head oh, columns ocol + 16 j
  const int oh = tid / 16;
  const int ocol = tid % 16;
  const int nj = d / 16;
  float acc[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) acc[j] = 0.f;
  // per-warp softmax state for heads 2w, 2w + 1 (lane-replicated)
  const int warp = tid / 32, lane = tid % 32;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};

  const __nv_bfloat16* cb = reinterpret_cast<const __nv_bfloat16*>(p.cache);
  for (int t0 = t_begin; t0 < t_end; t0 += kTT) {
    __syncthreads();  // previous tile fully consumed
    if (tid < kTT) {
      int t = t0 + tid;
      int ok = t < t_end;
      if (ok && p.page_table) {
        int blk = p.page_table[b * p.pt_sb + t / kBlock];
        if (blk < 0 || blk >= p.num_blocks) {
          set_status(TPLA_ERR_DEVICE_BOUNDS);
          ok = 0;
        }
      }
      sm.valid[tid] = ok;
    }
    __syncthreads();
    for (int i = tid; i < kTT * Kd; i += kThreads) {
      int tt = i / Kd, c = i % Kd;
      int t = t0 + tt;
      float v = 0.f;
      if (sm.valid[tt]) {
        int col = c < d ? lat0 + c : rope0 + (c - d);
        const __nv_bfloat16* row;
        if (p.page_table) {
          int blk = p.page_table[b * p.pt_sb + t / kBlock];
          row = cb + (int64_t)blk * p.c_s0 + (int64_t)(t % kBlock) * p.c_s1;
        } else {
          row = cb + (int64_t)b * p.c_s0 + (int64_t)t * p.c_s1;
        }
        v = ld_bf16(row + col);
      }
      sm.kv[tt][c] = v;
    }
    __syncthreads();
    // scores: thread -> (token lane, heads warp and warp + 8)
    for (int hh = warp; hh < kHG; hh += kThreads / 32) {
      float sdot = 0.f;
      for (int c = 0; c < Kd; ++c) sdot = fmaf(sm.q[hh][c], sm.kv[lane][c], sdot);
      sm.s[hh][lane] = sm.valid[lane] ? sdot * p.scale : -INFINITY;
    }
    __syncthreads();
    // online softmax, warp w owns heads 2w, 2w + 1
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      int hh = 2 * warp + e;
      float sv = sm.s[hh][lane];
      float mt = sv;
      for (int o = 16; o; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
      float m_new = fmaxf(m_run[e], mt);
      float alpha, pv;
      if (m_new == -INFINITY) {
        alpha = 1.f;
        pv = 0.f;
      } else {
        alpha = expf(m_run[e] - m_new);
        pv = expf(sv - m_new);
      }
      float ps = pv;
      for (int o = 16; o; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      l_run[e] = l_run[e] * alpha + ps;
      m_run[e] = m_new;
      sm.s[hh][lane] = pv;
      if (lane == 0) sm.alpha[hh] = alpha;
    }
    __syncthreads();
    // O <- alpha O + P V (values: latent columns of the shard only)
    {
      float a = sm.alpha[oh];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j < nj) {
          int c = ocol + 16 * j;
          float sum = acc[j] * a;
          for (int tt = 0; tt < kTT; ++tt) sum = fmaf(sm.s[oh][tt], sm.kv[tt][c], sum);
          acc[j] = sum;
        }
      }
    }
  }
  __syncthreads();
  // publish per-head (m, l) from the softmax warps
  __shared__ float m_sh[kHG], l_sh[kHG];
  if (lane == 0) {
    m_sh[2 * warp] = m_run[0];
    m_sh[2 * warp + 1] = m_run[1];
    l_sh[2 * warp] = l_run[0];
    l_sh[2 * warp + 1] = l_run[1];
  }
  __syncthreads();
  const int h = h0 + oh;
  if (h >= p.H) return;
  const float lsum = l_sh[oh];
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
  const float lse_v = lsum > 0.f ? m_sh[oh] + logf(lsum) : -INFINITY;

  if (splits == 1) {
    const int cbase = p.shard < 0 ? lat0 : 0;
    for (int j = 0; j < nj; ++j) {
      int c = cbase + ocol + 16 * j;
      float v = acc[j] * inv;
      int64_t off = (int64_t)b * p.o_sb + (int64_t)h * p.o_sh + c;
      if (p.out_bf16)
        reinterpret_cast<__nv_bfloat16*>(p.out)[off] = __float2bfloat16_rn(v);
      else
        reinterpret_cast<float*>(p.out)[off] = v;
    }
    if (p.lse && ocol == 0) p.lse[(int64_t)b * p.l_sb + (int64_t)h * p.l_sh + k] = lse_v;
  } else {
    const int W = p.out_width;
    const int cbase = p.shard < 0 ? lat0 : 0;
    float* op = o_part + (((int64_t)split * p.B + b) * p.H + h) * W;
    for (int j = 0; j < nj; ++j) op[cbase + ocol + 16 * j] = acc[j] * inv;
    if (ocol == 0)
      lse_part[(((int64_t)split * p.B + b) * p.H + h) * p.n_shards + k] = lse_v;
  }
}

}  // namespace

size_t generic_workspace_bytes(const DecodeProblem& p, int splits) {
  if (splits <= 1) return 0;
  size_t o = (size_t)splits * p.B * p.H * p.out_width * sizeof(float);
  size_t l = (size_t)splits * p.B * p.H * p.n_shards * sizeof(float);
  return ((o + 255) / 256) * 256 + l;
}

cudaError_t launch_decode_generic(const DecodeProblem& p, int splits, void* ws,
                                  cudaStream_t stream) {
  if (p.B == 0 || p.H == 0) return cudaSuccess;
  if (splits < 1) splits = 1;
  int64_t cap = p.cache_rows;
  int64_t chunk = (cap + splits - 1) / splits;
  chunk = ((chunk + kTT - 1) / kTT) * kTT;
  if (chunk < kTT) chunk = kTT;
  float* o_part = nullptr;
  float* lse_part = nullptr;
  if (splits > 1) {
    size_t o = (size_t)splits * p.B * p.H * p.out_width * sizeof(float);
    o_part = reinterpret_cast<float*>(ws);
    lse_part = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + ((o + 255) / 256) * 256);
  }
  dim3 grid((p.H + kHG - 1) / kHG, splits, p.B * p.n_shards);
  size_t smem = sizeof(SmemGeneric);
  cudaError_t e = cudaFuncSetAttribute(decode_generic_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_generic_kernel<<<grid, kThreads, smem, stream>>>(p, splits, (int)chunk, o_part, lse_part);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess || splits == 1) return e;
  const int W = p.out_width;
  return launch_lse_merge(o_part, lse_part, splits,
                          (int64_t)p.B * p.H * W, (int64_t)p.B * p.H * p.n_shards,
                          p.B, p.H, W, p.n_shards,
                          (int64_t)p.H * W, W, (int64_t)p.H * p.n_shards, p.n_shards,
                          p.out, p.out_bf16, p.o_sb, p.o_sh, p.lse, p.l_sb, p.l_sh, stream);
}

cudaError_t status_read_clear_generic(int* code) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_status, sizeof(int));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    int zero = 0;
    e = cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
  }
  *code = v;
  return e;
}

}  // namespace tpla
