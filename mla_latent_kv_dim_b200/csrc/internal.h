// Host-side declarations shared by the libtpla translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "tpla.h"

namespace tpla {

constexpr int kLatent = 512;  // latent columns of a cache row
constexpr int kRope = 64;     // rope columns of a cache row
constexpr int kWidth = 576;   // values per cached token
constexpr int kBlock = 64;    // tokens per cache page

// One validated decode call, flattened to raw pointers and element strides.
struct DecodeProblem {
  const void* q;           // bf16 [B, H, 576]
  int64_t q_sb, q_sh;
  const void* cache;       // bf16 paged [NB, 64, 576] or contiguous [B, Lmax, 576]
  int64_t c_s0, c_s1;      // paged: block, row strides; contiguous: batch, row
  int64_t num_blocks;      // paged only
  int64_t cache_rows;      // contiguous: Lmax;  paged: max_pages * 64
  const int* seq_lens;     // [B], or nullptr: request b holds causal_base + b + 1 tokens
  int causal_base;
  const int* page_table;   // [B, max_pages] or nullptr (contiguous)
  int64_t pt_sb;
  int max_pages;
  int B, H, G, rope_mode, shard;  // shard -1 = all shards
  int n_shards;            // shards computed by this call: G or 1
  int out_width;           // 512 (all shards) or 512 / G (one shard)
  float scale;
  void* out;               // [B, H, out_width]
  int out_bf16;
  int64_t o_sb, o_sh;
  float* lse;              // [B, H, n_shards] or nullptr
  int64_t l_sb, l_sh;
};

// Per-launch description of split partial results kept in the workspace.
struct SplitParts {
  float* o;     // [S, B, H, out_width]
  float* lse;   // [S, B, H, n_shards]
  int S;
};

// ---------------------------------------------------------------- generic path
size_t generic_workspace_bytes(const DecodeProblem& p, int splits);
cudaError_t launch_decode_generic(const DecodeProblem& p, int splits, void* ws,
                                  cudaStream_t stream);

// ---------------------------------------------------------------- sm100 path
// cuTensorMapEncodeTiled (as void*), or nullptr when the driver lacks it.
void* tensor_map_encoder();
// True when `device` is an sm_100 GPU the tcgen05 kernels can run on.
bool sm100_device(int device);
// Returns true when the tcgen05 kernel can run this problem on this device.
bool sm100_supported(const DecodeProblem& p, int device);
size_t sm100_workspace_bytes(const DecodeProblem& p, int num_splits, int device);
cudaError_t launch_decode_sm100(const DecodeProblem& p, int num_splits, void* ws,
                                size_t ws_bytes, cudaStream_t stream);

// ---------------------------------------------------------------- merge
// out[b,h,:] / lse[b,h,:] from S partials laid out as SplitParts.
cudaError_t launch_lse_merge(const float* o_parts, const float* lse_parts, int S,
                             int64_t part_stride_o, int64_t part_stride_l,
                             int B, int H, int Wd, int Gs,
                             int64_t po_sb, int64_t po_sh, int64_t pl_sb, int64_t pl_sh,
                             void* out, int out_bf16, int64_t o_sb, int64_t o_sh,
                             float* lse, int64_t l_sb, int64_t l_sh,
                             cudaStream_t stream);

// ---------------------------------------------------------------- hadamard / vup
cudaError_t launch_hadamard(void* buf, int bf16, int ndim, const int64_t* shape,
                            const int64_t* stride, int dim, cudaStream_t stream);
// True when the V-up kernel takes these layouts (TMA: 16-byte aligned bases
// and row strides).
bool vup_supported(const void* out_latent, int out_bf16, int64_t o_sb, int64_t o_sh,
                   const void* W, int64_t w_sh, int64_t w_sj);
cudaError_t launch_vup(const void* out_latent, int out_bf16, int64_t o_sb, int64_t o_sh,
                       const void* W, int64_t w_sh, int64_t w_sj, float* y,
                       int64_t y_sb, int64_t y_sh, int B, int H, int Dv, int K,
                       cudaStream_t stream);

// ---------------------------------------------------------------- PCA reparameterisation
// Rows are the first 512 columns of a [B, H, >= 512] bf16 view (element
// strides sb, sh; innermost contiguous).
cudaError_t launch_latent_stats(const void* x, int64_t B, int64_t H, int64_t sb, int64_t sh,
                                float* C, int64_t c_s0, float* s, cudaStream_t stream);
cudaError_t launch_covariance_finalize(const float* C, int64_t c_s0, const float* s, int64_t n,
                                       float* cov, int64_t v_s0, float* mean,
                                       cudaStream_t stream);
cudaError_t launch_rotate(void* x, int64_t B, int64_t H, int64_t sb, int64_t sh, const void* U,
                          float* scratch, int64_t chunk_b, cudaStream_t stream);

// ---------------------------------------------------------------- cache append
// positions == nullptr: row b goes to position pos0 + b.
cudaError_t launch_cache_append(const void* kv_new, int in_bf16, int64_t n_sb, const int* positions,
                                int pos0, const int* page_table, int64_t pt_sb, int max_pages,
                                int64_t num_blocks, int64_t cap_rows, void* cache, int64_t c_s0,
                                int64_t c_s1, int B, int groups, int hadamard, float eps,
                                cudaStream_t stream);

// ---------------------------------------------------------------- launch counter
// Called once per kernel launch by every launcher.
void count_launch(int n = 1);

// ---------------------------------------------------------------- device status
// Each translation unit that launches kernels owns a device status word;
// these read and clear it (after the caller synchronised the stream).
cudaError_t status_read_clear_generic(int* code);
cudaError_t status_read_clear_sm100(int* code);
cudaError_t status_read_clear_vup(int* code);
cudaError_t status_read_clear_append(int* code);
cudaError_t launch_wait_timeout_selftest(long long cycles, cudaStream_t stream);

}  // namespace tpla
