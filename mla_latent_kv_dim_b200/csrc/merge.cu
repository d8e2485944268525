// Log-sum-exp merge of split-KV partial results.
//
// The exact alternative of the feature request "Bandwidth-optimal
// tensor-parallel sharding of MLA" (section "Directions under
// investigation") that splits the sequence and combines the pieces by their
// log-sum-exp: chunk s of a request produced a normalised output o_s and
// lse_s, then
//   lse = M + ln sum_s exp(lse_s - M),  M = max_s lse_s
//   out = sum_s exp(lse_s - lse) o_s.
// Empty chunks carry lse = -inf and weigh nothing; a request whose chunks
// are all empty gets out = 0 and lse = -inf.  Each TPLA shard has its own
// lse and owns a contiguous block of Wd / Gs output columns.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"

namespace tpla {
namespace {

constexpr int kThreads = 128;
constexpr int kMaxParts = 1024;

__global__ void __launch_bounds__(kThreads)
lse_merge_kernel(const float* __restrict__ o_parts, const float* __restrict__ lse_parts,
                 int S, int64_t ps_o, int64_t ps_l, int H, int Wd, int Gs,
                 int64_t po_sb, int64_t po_sh, int64_t pl_sb, int64_t pl_sh,
                 void* out, int out_bf16, int64_t o_sb, int64_t o_sh,
                 float* lse, int64_t l_sb, int64_t l_sh) {
  __shared__ float w_sh[kMaxParts];
  const int b = blockIdx.x / H;
  const int h = blockIdx.x % H;
  const int cw = Wd / Gs;  // columns per shard
  for (int k = 0; k < Gs; ++k) {
    const float* lp = lse_parts + b * pl_sb + h * pl_sh + k;
    // max over parts (every thread computes it; S is small)
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, lp[s * ps_l]);
    float total;
    if (M == -INFINITY) {
      total = -INFINITY;
    } else {
      float z = 0.f;
      for (int s = 0; s < S; ++s) {
        float ls = lp[s * ps_l];
        z += ls == -INFINITY ? 0.f : expf(ls - M);
      }
      total = M + logf(z);
    }
    __syncthreads();
    for (int s = threadIdx.x; s < S; s += kThreads) {
      float ls = lp[s * ps_l];
      w_sh[s] = (total == -INFINITY || ls == -INFINITY) ? 0.f : expf(ls - total);
    }
    __syncthreads();
    for (int c = threadIdx.x; c < cw; c += kThreads) {
      int col = k * cw + c;
      float acc = 0.f;
      const float* op = o_parts + b * po_sb + h * po_sh + col;
      for (int s = 0; s < S; ++s) {
        float w = w_sh[s];
        if (w != 0.f) acc = fmaf(w, op[s * ps_o], acc);
      }
      int64_t off = (int64_t)b * o_sb + (int64_t)h * o_sh + col;
      if (out_bf16)
        reinterpret_cast<__nv_bfloat16*>(out)[off] = __float2bfloat16_rn(acc);
      else
        reinterpret_cast<float*>(out)[off] = acc;
    }
    if (lse && threadIdx.x == 0) lse[(int64_t)b * l_sb + (int64_t)h * l_sh + k] = total;
  }
}

}  // namespace

cudaError_t launch_lse_merge(const float* o_parts, const float* lse_parts, int S,
                             int64_t part_stride_o, int64_t part_stride_l,
                             int B, int H, int Wd, int Gs,
                             int64_t po_sb, int64_t po_sh, int64_t pl_sb, int64_t pl_sh,
                             void* out, int out_bf16, int64_t o_sb, int64_t o_sh,
                             float* lse, int64_t l_sb, int64_t l_sh,
                             cudaStream_t stream) {
  if (B == 0 || H == 0) return cudaSuccess;
  if (S > kMaxParts) return cudaErrorInvalidValue;
  lse_merge_kernel<<<B * H, kThreads, 0, stream>>>(
      o_parts, lse_parts, S, part_stride_o, part_stride_l, H, Wd, Gs,
      po_sb, po_sh, pl_sb, pl_sh, out, out_bf16, o_sb, o_sh, lse, l_sb, l_sh);
  count_launch();
  return cudaGetLastError();
}

}  // namespace tpla
