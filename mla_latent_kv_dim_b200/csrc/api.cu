// libtpla C ABI: argument validation, kernel selection, errors, status.
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <atomic>

#include "internal.h"
#include "tpla.h"

namespace tpla {
namespace {

thread_local int t_last_cuda_error = 0;
std::atomic<int64_t> g_launches{0};

int cuda_fail(cudaError_t e) {
  t_last_cuda_error = (int)e;
  return TPLA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch-geometry limits the entry points check before any launch.
constexpr int kMaxSplits = 65535;                     // a grid dimension of the generic kernel
constexpr int64_t kMaxRequestHeads = 1LL << 30;       // B * H: merge blocks, 32-bit grid
constexpr int64_t kMaxRequestSplits = 1LL << 24;      // B * num_splits: 2x that many slots
constexpr int64_t kMaxGenericRequestShards = 65535;   // B * shards: the generic grid's z

bool check_tensor(const tpla_tensor* t, int dtype, int ndim) {
  if (!t || t->dtype != dtype || t->ndim != ndim) return false;
  for (int i = 0; i < ndim; ++i) {
    if (t->shape[i] < 0) return false;
    if (t->stride[i] < 0) return false;
  }
  if (ndim > 0 && t->shape[ndim - 1] > 1 && t->stride[ndim - 1] != 1) return false;
  bool empty = false;
  for (int i = 0; i < ndim; ++i) empty |= t->shape[i] == 0;
  if (!empty && !t->data) return false;
  return true;
}

int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev;
}

// Flatten and validate a decode call.
int build_problem(const tpla_tensor* q, const tpla_tensor* kv, const tpla_tensor* seq,
                  const tpla_tensor* pt, int G, int rope_mode, float scale,
                  const tpla_tensor* out, const tpla_tensor* lse,
                  const tpla_decode_opts* opts, DecodeProblem* p) {
  if (!q || !kv || !seq || !out) return TPLA_ERR_INVALID_ARG;
  if (!(G == 1 || G == 2 || G == 4 || G == 8)) return TPLA_ERR_INVALID_ARG;
  if (rope_mode != TPLA_ROPE_REPLICATE && rope_mode != TPLA_ROPE_SPLIT) return TPLA_ERR_INVALID_ARG;
  if (!isfinite(scale)) return TPLA_ERR_INVALID_ARG;
  int shard = opts ? opts->shard : -1;
  if (shard < -1 || shard >= G) return TPLA_ERR_INVALID_ARG;
  if (opts && (opts->reserved != 0 || opts->num_splits < 0)) return TPLA_ERR_INVALID_ARG;
  if (opts && opts->num_splits > kMaxSplits) return TPLA_ERR_UNSUPPORTED;
  if (opts && (opts->kernel < TPLA_KERNEL_AUTO || opts->kernel > TPLA_KERNEL_SM100))
    return TPLA_ERR_INVALID_ARG;

  if (!check_tensor(q, TPLA_BF16, 3) || q->shape[2] != kWidth) return TPLA_ERR_INVALID_ARG;
  const int64_t B = q->shape[0], H = q->shape[1];
  if (B > (1 << 20) || H > 4096) return TPLA_ERR_UNSUPPORTED;
  // (request, head) pairs index one merge block each; explicit splits index
  // 2 * B * num_splits partial slots
  if (B * H > kMaxRequestHeads) return TPLA_ERR_UNSUPPORTED;
  if (opts && B * opts->num_splits > kMaxRequestSplits) return TPLA_ERR_UNSUPPORTED;
  if (!check_tensor(seq, TPLA_I32, 1) || seq->shape[0] != B) return TPLA_ERR_INVALID_ARG;
  if (!check_tensor(kv, TPLA_BF16, 3) || kv->shape[2] != kWidth) return TPLA_ERR_INVALID_ARG;
  const bool paged = pt != nullptr;
  if (paged) {
    if (!check_tensor(pt, TPLA_I32, 2) || pt->shape[0] != B) return TPLA_ERR_INVALID_ARG;
    if (kv->shape[1] != kBlock) return TPLA_ERR_UNSUPPORTED;  // 64-token pages only
    if (pt->shape[1] < 1 && B > 0) return TPLA_ERR_INVALID_ARG;
    if (pt->shape[1] > (1 << 24)) return TPLA_ERR_UNSUPPORTED;
  } else {
    if (kv->shape[0] != B) return TPLA_ERR_INVALID_ARG;
  }
  // 16-byte rows (TMA and vector loads)
  if (B > 0 && H > 0) {
    if (!aligned16(q->data) || (q->stride[1] % 8) || (q->stride[0] % 8)) return TPLA_ERR_INVALID_ARG;
  }
  if (kv->shape[0] > 0 && kv->shape[1] > 0) {
    if (!aligned16(kv->data) || (kv->stride[1] % 8) || (kv->stride[0] % 8)) return TPLA_ERR_INVALID_ARG;
  }

  const int n_shards = shard < 0 ? G : 1;
  const int width = shard < 0 ? kLatent : kLatent / G;
  if (!out || (out->dtype != TPLA_F32 && out->dtype != TPLA_BF16)) return TPLA_ERR_INVALID_ARG;
  if (!check_tensor(out, out->dtype, 3) || out->shape[0] != B || out->shape[1] != H ||
      out->shape[2] != width)
    return TPLA_ERR_INVALID_ARG;
  if (lse) {
    if (!check_tensor(lse, TPLA_F32, 3) || lse->shape[0] != B || lse->shape[1] != H ||
        lse->shape[2] != n_shards)
      return TPLA_ERR_INVALID_ARG;
  }

  memset(p, 0, sizeof(*p));
  p->q = q->data;
  p->q_sb = q->stride[0];
  p->q_sh = q->stride[1];
  p->cache = kv->data;
  p->c_s0 = kv->stride[0];
  p->c_s1 = kv->stride[1];
  p->seq_lens = reinterpret_cast<const int*>(seq->data);
  if (paged) {
    p->page_table = reinterpret_cast<const int*>(pt->data);
    p->pt_sb = pt->stride[0];
    p->max_pages = (int)pt->shape[1];
    p->num_blocks = kv->shape[0];
    p->cache_rows = (int64_t)pt->shape[1] * kBlock;
  } else {
    p->page_table = nullptr;
    p->num_blocks = 0;
    p->cache_rows = kv->shape[1];
  }
  p->B = (int)B;
  p->H = (int)H;
  p->G = G;
  p->rope_mode = rope_mode;
  p->shard = shard;
  p->n_shards = n_shards;
  p->out_width = width;
  p->scale = scale;
  p->out = out->data;
  p->out_bf16 = out->dtype == TPLA_BF16;
  p->o_sb = out->stride[0];
  p->o_sh = out->stride[1];
  p->lse = lse ? reinterpret_cast<float*>(lse->data) : nullptr;
  p->l_sb = lse ? lse->stride[0] : 0;
  p->l_sh = lse ? lse->stride[1] : 0;
  return TPLA_OK;
}

enum class Path { Generic, Sm100 };

int choose_path(const DecodeProblem& p, const tpla_decode_opts* opts, Path* path) {
  int choice = opts ? opts->kernel : TPLA_KERNEL_AUTO;
  int dev = current_device();
  bool fast = sm100_supported(p, dev);
  if (choice == TPLA_KERNEL_GENERIC) {
    *path = Path::Generic;
  } else if (choice == TPLA_KERNEL_SM100) {
    if (!fast) return TPLA_ERR_UNSUPPORTED;
    *path = Path::Sm100;
  } else {
    // the automatic choice is the tcgen05 kernel; the portable kernel runs
    // only when the caller names it
    if (!fast) return TPLA_ERR_UNSUPPORTED;
    *path = Path::Sm100;
  }
  if (*path == Path::Generic && (int64_t)p.B * p.n_shards > kMaxGenericRequestShards)
    return TPLA_ERR_UNSUPPORTED;
  return TPLA_OK;
}

// Generic-path split count: the caller's, else enough CTAs to fill the GPU.
int generic_splits(const DecodeProblem& p, const tpla_decode_opts* opts) {
  int s = opts ? opts->num_splits : 0;
  if (s >= 1) return s;
  int64_t ctas = (int64_t)((p.H + 15) / 16) * p.B * p.n_shards;
  int64_t want = (2 * 148 + ctas - 1) / (ctas > 0 ? ctas : 1);
  int64_t tiles = (p.cache_rows + 255) / 256;  // at least 256 tokens per chunk
  if (want > tiles) want = tiles;
  if (want < 1) want = 1;
  if (want > 64) want = 64;
  return (int)want;
}

int workspace_needed(const DecodeProblem& p, const tpla_decode_opts* opts, Path path,
                     size_t* bytes) {
  if (path == Path::Generic) {
    *bytes = generic_workspace_bytes(p, generic_splits(p, opts));
  } else {
    *bytes = sm100_workspace_bytes(p, opts ? opts->num_splits : 0, current_device());
  }
  return TPLA_OK;
}

int run_decode(const DecodeProblem& p, const tpla_decode_opts* opts, Path path, void* ws,
               size_t ws_bytes, cudaStream_t stream) {
  cudaError_t e;
  if (path == Path::Generic) {
    e = launch_decode_generic(p, generic_splits(p, opts), ws, stream);
  } else {
    e = launch_decode_sm100(p, opts ? opts->num_splits : 0, ws, ws_bytes, stream);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  return TPLA_OK;
}

// A validated prefill call: the exact-MLA attention of its prompt rows as a
// decode problem with one query row per prompt token, causal lengths and the
// request's page-table row shared by every query row (row stride 0).
struct PrefillCall {
  DecodeProblem p;
};

int build_prefill(const tpla_tensor* q, const tpla_tensor* kv_new, int start,
                  const tpla_tensor* page_row, const tpla_tensor* kv, int norm_groups,
                  int hadamard, float eps, float scale, const tpla_tensor* out,
                  const tpla_tensor* lse, PrefillCall* c) {
  memset(c, 0, sizeof(*c));
  if (!check_tensor(q, TPLA_BF16, 3) || q->shape[2] != kWidth) return TPLA_ERR_INVALID_ARG;
  const int64_t T = q->shape[0], H = q->shape[1];
  if (T > (1 << 20) || H > 4096) return TPLA_ERR_UNSUPPORTED;
  if (T * H > kMaxRequestHeads) return TPLA_ERR_UNSUPPORTED;
  if (T > 0 && H > 0 && (!aligned16(q->data) || (q->stride[1] % 8) || (q->stride[0] % 8)))
    return TPLA_ERR_INVALID_ARG;
  c->p.B = (int)T;
  c->p.H = (int)H;
  c->p.G = 1;
  c->p.shard = -1;
  c->p.n_shards = 1;
  c->p.out_width = kLatent;
  if (!kv_new) return TPLA_OK;  // workspace-size query: q alone fixes it
  if (kv_new->dtype != TPLA_BF16 && kv_new->dtype != TPLA_F32) return TPLA_ERR_INVALID_ARG;
  if (!check_tensor(kv_new, kv_new->dtype, 2) || kv_new->shape[0] != T ||
      kv_new->shape[1] != kWidth)
    return TPLA_ERR_INVALID_ARG;
  const int64_t esz = kv_new->dtype == TPLA_BF16 ? 2 : 4;
  if (T > 0 && (!aligned16(kv_new->data) || (kv_new->stride[0] * esz) % 16))
    return TPLA_ERR_INVALID_ARG;
  if (start < 0) return TPLA_ERR_INVALID_ARG;
  if (!(norm_groups == 1 || norm_groups == 2 || norm_groups == 4 || norm_groups == 8))
    return TPLA_ERR_INVALID_ARG;
  if (!(hadamard == 0 || hadamard == 1) || !isfinite(eps) || eps < 0.f)
    return TPLA_ERR_INVALID_ARG;
  if (!kv || !check_tensor(kv, TPLA_BF16, 3) || kv->shape[2] != kWidth)
    return TPLA_ERR_INVALID_ARG;
  if (kv->shape[1] != kBlock) return TPLA_ERR_UNSUPPORTED;  // 64-token pages only
  if (!aligned16(kv->data) || kv->stride[0] % 8 || kv->stride[1] % 8)
    return TPLA_ERR_INVALID_ARG;
  if (!check_tensor(page_row, TPLA_I32, 1) || page_row->shape[0] < 1) return TPLA_ERR_INVALID_ARG;
  if (page_row->shape[0] > (1 << 24)) return TPLA_ERR_UNSUPPORTED;
  if ((int64_t)start + T > page_row->shape[0] * kBlock) return TPLA_ERR_INVALID_ARG;
  // the attention half is a decode problem: query row i holds start + i + 1
  // tokens, every row reads the request's page-table row
  tpla_tensor pt = *page_row;
  pt.ndim = 2;
  pt.shape[0] = T;
  pt.shape[1] = page_row->shape[0];
  pt.stride[0] = 0;
  pt.stride[1] = 1;
  int placeholder = 0;  // stands for a lengths array that is never read
  tpla_tensor seq;
  memset(&seq, 0, sizeof(seq));
  seq.data = &placeholder;
  seq.dtype = TPLA_I32;
  seq.ndim = 1;
  seq.shape[0] = T;
  seq.stride[0] = 1;
  int rc = build_problem(q, kv, &seq, &pt, 1, TPLA_ROPE_REPLICATE, scale, out, lse, nullptr,
                         &c->p);
  if (rc != TPLA_OK) return rc;
  c->p.seq_lens = nullptr;
  c->p.causal_base = start;
  if (c->p.B > 0 && c->p.H > 0 && !sm100_supported(c->p, current_device()))
    return TPLA_ERR_UNSUPPORTED;
  return TPLA_OK;
}

}  // namespace

void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

}  // namespace tpla

using namespace tpla;

extern "C" {

int tpla_decode_workspace_size(const tpla_tensor* q, const tpla_tensor* kv_cache,
                               const tpla_tensor* seq_lens, const tpla_tensor* page_table,
                               int G, int rope_mode, const tpla_tensor* out,
                               const tpla_decode_opts* opts, size_t* bytes) {
  if (!bytes) return TPLA_ERR_INVALID_ARG;
  DecodeProblem p;
  int rc = build_problem(q, kv_cache, seq_lens, page_table, G, rope_mode, 1.0f, out, nullptr,
                         opts, &p);
  if (rc != TPLA_OK) return rc;
  Path path;
  rc = choose_path(p, opts, &path);
  if (rc != TPLA_OK) return rc;
  return workspace_needed(p, opts, path, bytes);
}

int tpla_decode_ex(const tpla_tensor* q, const tpla_tensor* kv_cache,
                   const tpla_tensor* seq_lens, const tpla_tensor* page_table, int G,
                   int rope_mode, float scale, tpla_tensor* out, tpla_tensor* lse,
                   const tpla_decode_opts* opts, tpla_stream_t stream) {
  DecodeProblem p;
  int rc = build_problem(q, kv_cache, seq_lens, page_table, G, rope_mode, scale, out, lse,
                         opts, &p);
  if (rc != TPLA_OK) return rc;
  if (p.B == 0 || p.H == 0) return TPLA_OK;
  Path path;
  rc = choose_path(p, opts, &path);
  if (rc != TPLA_OK) return rc;
  size_t need = 0;
  workspace_needed(p, opts, path, &need);
  void* ws = opts ? opts->workspace : nullptr;
  size_t have = opts ? opts->workspace_bytes : 0;
  if (need > 0 && (!ws || have < need || !aligned16(ws))) return TPLA_ERR_WORKSPACE;
  return run_decode(p, opts, path, ws, have, reinterpret_cast<cudaStream_t>(stream));
}

int tpla_decode(const tpla_tensor* q, const tpla_tensor* kv_cache, const tpla_tensor* seq_lens,
                const tpla_tensor* page_table, int G, int rope_mode, float scale,
                tpla_tensor* out, tpla_tensor* lse, tpla_stream_t stream) {
  DecodeProblem p;
  int rc = build_problem(q, kv_cache, seq_lens, page_table, G, rope_mode, scale, out, lse,
                         nullptr, &p);
  if (rc != TPLA_OK) return rc;
  if (p.B == 0 || p.H == 0) return TPLA_OK;
  Path path;
  rc = choose_path(p, nullptr, &path);
  if (rc != TPLA_OK) return rc;
  size_t need = 0;
  workspace_needed(p, nullptr, path, &need);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  if (need > 0) {
    cudaError_t e = cudaMallocAsync(&ws, need, s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  rc = run_decode(p, nullptr, path, ws, need, s);
  if (ws) {
    cudaError_t e = cudaFreeAsync(ws, s);
    if (rc == TPLA_OK && e != cudaSuccess) rc = cuda_fail(e);
  }
  return rc;
}

int tpla_lse_merge(const tpla_tensor* o_parts, const tpla_tensor* lse_parts, tpla_tensor* out,
                   tpla_tensor* lse, tpla_stream_t stream) {
  if (!check_tensor(o_parts, TPLA_F32, 4) || !check_tensor(lse_parts, TPLA_F32, 4))
    return TPLA_ERR_INVALID_ARG;
  const int64_t S = o_parts->shape[0], B = o_parts->shape[1], H = o_parts->shape[2],
                Wd = o_parts->shape[3];
  const int64_t Gs = lse_parts->shape[3];
  if (lse_parts->shape[0] != S || lse_parts->shape[1] != B || lse_parts->shape[2] != H)
    return TPLA_ERR_INVALID_ARG;
  if (Gs < 1 || Wd % Gs != 0 || S < 1) return TPLA_ERR_INVALID_ARG;
  if (S > 1024 || B * H > kMaxRequestHeads || Wd > (1 << 20)) return TPLA_ERR_UNSUPPORTED;
  if (!out || (out->dtype != TPLA_F32 && out->dtype != TPLA_BF16) ||
      !check_tensor(out, out->dtype, 3) || out->shape[0] != B || out->shape[1] != H ||
      out->shape[2] != Wd)
    return TPLA_ERR_INVALID_ARG;
  if (lse && (!check_tensor(lse, TPLA_F32, 3) || lse->shape[0] != B || lse->shape[1] != H ||
              lse->shape[2] != Gs))
    return TPLA_ERR_INVALID_ARG;
  cudaError_t e = launch_lse_merge(
      reinterpret_cast<const float*>(o_parts->data),
      reinterpret_cast<const float*>(lse_parts->data), (int)S, o_parts->stride[0],
      lse_parts->stride[0], (int)B, (int)H, (int)Wd, (int)Gs, o_parts->stride[1],
      o_parts->stride[2], lse_parts->stride[1], lse_parts->stride[2], out->data,
      out->dtype == TPLA_BF16, out->stride[0], out->stride[1],
      lse ? reinterpret_cast<float*>(lse->data) : nullptr, lse ? lse->stride[0] : 0,
      lse ? lse->stride[1] : 0, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TPLA_OK : cuda_fail(e);
}

int tpla_hadamard_apply(tpla_tensor* buf, int dim, tpla_stream_t stream) {
  if (!buf || (buf->dtype != TPLA_BF16 && buf->dtype != TPLA_F32)) return TPLA_ERR_INVALID_ARG;
  if (buf->ndim < 1 || buf->ndim > 4 || !check_tensor(buf, buf->dtype, buf->ndim))
    return TPLA_ERR_INVALID_ARG;
  if (dim < 32 || dim > 1024 || (dim & (dim - 1))) return TPLA_ERR_UNSUPPORTED;
  if (buf->shape[buf->ndim - 1] < dim) return TPLA_ERR_INVALID_ARG;
  if (buf->ndim > 4) return TPLA_ERR_UNSUPPORTED;
  // rows may be described by at most three dimensions
  cudaError_t e = launch_hadamard(buf->data, buf->dtype == TPLA_BF16, buf->ndim, buf->shape,
                                  buf->stride, dim, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TPLA_OK : cuda_fail(e);
}

int tpla_vup_combine(const tpla_tensor* out_latent, const tpla_tensor* W_uv, tpla_tensor* y,
                     tpla_stream_t stream) {
  if (!out_latent || (out_latent->dtype != TPLA_F32 && out_latent->dtype != TPLA_BF16))
    return TPLA_ERR_INVALID_ARG;
  if (!check_tensor(out_latent, out_latent->dtype, 3)) return TPLA_ERR_INVALID_ARG;
  // K latent columns: 512, or one shard's 512 / G (a rank's partial product)
  const int64_t B = out_latent->shape[0], H = out_latent->shape[1], K = out_latent->shape[2];
  if (K < 64 || K > kLatent || K % 64) return TPLA_ERR_INVALID_ARG;
  if (!check_tensor(W_uv, TPLA_BF16, 3) || W_uv->shape[0] != H || W_uv->shape[1] != K)
    return TPLA_ERR_INVALID_ARG;
  const int64_t Dv = W_uv->shape[2];
  if (Dv % 16 != 0 || Dv < 16 || Dv > 256) return TPLA_ERR_UNSUPPORTED;
  if (!check_tensor(y, TPLA_F32, 3) || y->shape[0] != B || y->shape[1] != H || y->shape[2] != Dv)
    return TPLA_ERR_INVALID_ARG;
  if (H > 65535 || (B + 63) / 64 > 65535) return TPLA_ERR_UNSUPPORTED;
  if (!vup_supported(out_latent->data, out_latent->dtype == TPLA_BF16, out_latent->stride[0],
                     out_latent->stride[1], W_uv->data, W_uv->stride[0], W_uv->stride[1]))
    return TPLA_ERR_UNSUPPORTED;
  cudaError_t e = launch_vup(out_latent->data, out_latent->dtype == TPLA_BF16,
                             out_latent->stride[0], out_latent->stride[1], W_uv->data,
                             W_uv->stride[0], W_uv->stride[1],
                             reinterpret_cast<float*>(y->data), y->stride[0], y->stride[1],
                             (int)B, (int)H, (int)Dv, (int)K, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TPLA_OK : cuda_fail(e);
}

namespace {
// [N, >= 512] or [B, H, >= 512] bf16 rows, innermost contiguous, 16-byte rows.
bool latent_rows(const tpla_tensor* t, int64_t* B, int64_t* H, int64_t* sb, int64_t* sh) {
  if (!t || t->dtype != TPLA_BF16 || (t->ndim != 2 && t->ndim != 3)) return false;
  if (!check_tensor(t, TPLA_BF16, t->ndim) || t->shape[t->ndim - 1] < kLatent) return false;
  if (t->ndim == 2) {
    *B = t->shape[0];
    *H = 1;
    *sb = t->stride[0];
    *sh = 0;
  } else {
    *B = t->shape[0];
    *H = t->shape[1];
    *sb = t->stride[0];
    *sh = t->stride[1];
  }
  if (*B * *H > 0 && (!aligned16(t->data) || *sb % 8 || *sh % 8)) return false;
  return true;
}
}  // namespace

int tpla_latent_covariance(const tpla_tensor* rows, tpla_tensor* C, tpla_tensor* s,
                           tpla_stream_t stream) {
  int64_t B, H, sb, sh;
  if (!latent_rows(rows, &B, &H, &sb, &sh)) return TPLA_ERR_INVALID_ARG;
  if (!check_tensor(C, TPLA_F32, 2) || C->shape[0] != kLatent || C->shape[1] != kLatent ||
      !check_tensor(s, TPLA_F32, 1) || s->shape[0] != kLatent)
    return TPLA_ERR_INVALID_ARG;
  if (B * H > (int64_t)65535 * 2048 || H > (1 << 30)) return TPLA_ERR_UNSUPPORTED;
  cudaError_t e = launch_latent_stats(rows->data, B, H, sb, sh, reinterpret_cast<float*>(C->data),
                                      C->stride[0], reinterpret_cast<float*>(s->data),
                                      reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TPLA_OK : cuda_fail(e);
}

int tpla_covariance_finalize(const tpla_tensor* C, const tpla_tensor* s, int64_t n,
                             tpla_tensor* cov, tpla_tensor* mean, tpla_stream_t stream) {
  if (n <= 0) return TPLA_ERR_INVALID_ARG;
  for (const tpla_tensor* m : {C, static_cast<const tpla_tensor*>(cov)})
    if (!check_tensor(m, TPLA_F32, 2) || m->shape[0] != kLatent || m->shape[1] != kLatent)
      return TPLA_ERR_INVALID_ARG;
  for (const tpla_tensor* v : {s, static_cast<const tpla_tensor*>(mean)})
    if (!check_tensor(v, TPLA_F32, 1) || v->shape[0] != kLatent) return TPLA_ERR_INVALID_ARG;
  cudaError_t e = launch_covariance_finalize(
      reinterpret_cast<const float*>(C->data), C->stride[0],
      reinterpret_cast<const float*>(s->data), n, reinterpret_cast<float*>(cov->data),
      cov->stride[0], reinterpret_cast<float*>(mean->data), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TPLA_OK : cuda_fail(e);
}

int tpla_rotate_apply(tpla_tensor* buf, const tpla_tensor* U, void* scratch,
                      size_t scratch_bytes, tpla_stream_t stream) {
  int64_t B, H, sb, sh;
  if (!latent_rows(buf, &B, &H, &sb, &sh)) return TPLA_ERR_INVALID_ARG;
  if (!check_tensor(U, TPLA_BF16, 2) || U->shape[0] != kLatent || U->shape[1] != kLatent ||
      U->stride[0] != kLatent || !aligned16(U->data))
    return TPLA_ERR_INVALID_ARG;
  if (B * H == 0) return TPLA_OK;
  if (H > 65535 || B > (1LL << 31) - 1) return TPLA_ERR_UNSUPPORTED;
  const size_t per_b = (size_t)H * kLatent * sizeof(float);
  if (!scratch || !aligned16(scratch) || scratch_bytes < per_b) return TPLA_ERR_WORKSPACE;
  int64_t chunk = (int64_t)(scratch_bytes / per_b);
  if (chunk > B) chunk = B;
  if (chunk > (1 << 24)) chunk = 1 << 24;
  if (chunk * H > (1LL << 30)) chunk = (1LL << 30) / H;  // store grid stays below 2^31 blocks
  cudaError_t e = launch_rotate(buf->data, B, H, sb, sh, U->data, reinterpret_cast<float*>(scratch),
                                chunk, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TPLA_OK : cuda_fail(e);
}

int tpla_cache_append(const tpla_tensor* kv_new, const tpla_tensor* positions,
                      const tpla_tensor* page_table, tpla_tensor* kv_cache, int norm_groups,
                      int hadamard, float eps, tpla_stream_t stream) {
  if (!kv_new || (kv_new->dtype != TPLA_BF16 && kv_new->dtype != TPLA_F32))
    return TPLA_ERR_INVALID_ARG;
  if (!check_tensor(kv_new, kv_new->dtype, 2) || kv_new->shape[1] != kWidth)
    return TPLA_ERR_INVALID_ARG;
  const int64_t B = kv_new->shape[0];
  const int64_t esz = kv_new->dtype == TPLA_BF16 ? 2 : 4;
  if (B > 0 && (!aligned16(kv_new->data) || (kv_new->stride[0] * esz) % 16))
    return TPLA_ERR_INVALID_ARG;
  if (!check_tensor(positions, TPLA_I32, 1) || positions->shape[0] != B)
    return TPLA_ERR_INVALID_ARG;
  if (!(norm_groups == 1 || norm_groups == 2 || norm_groups == 4 || norm_groups == 8))
    return TPLA_ERR_INVALID_ARG;
  if (!(hadamard == 0 || hadamard == 1) || !isfinite(eps) || eps < 0.f)
    return TPLA_ERR_INVALID_ARG;
  if (!check_tensor(kv_cache, TPLA_BF16, 3) || kv_cache->shape[2] != kWidth)
    return TPLA_ERR_INVALID_ARG;
  if (!aligned16(kv_cache->data) || kv_cache->stride[0] % 8 || kv_cache->stride[1] % 8)
    return TPLA_ERR_INVALID_ARG;
  int max_pages = 0;
  if (page_table) {
    if (!check_tensor(page_table, TPLA_I32, 2) || page_table->shape[0] != B)
      return TPLA_ERR_INVALID_ARG;
    if (kv_cache->shape[1] != kBlock) return TPLA_ERR_UNSUPPORTED;
    if (page_table->shape[1] > (1 << 24)) return TPLA_ERR_UNSUPPORTED;
    max_pages = (int)page_table->shape[1];
  } else if (kv_cache->shape[0] != B) {
    return TPLA_ERR_INVALID_ARG;
  }
  if (B > (1 << 20)) return TPLA_ERR_UNSUPPORTED;
  if (B == 0) return TPLA_OK;
  cudaError_t e = launch_cache_append(
      kv_new->data, kv_new->dtype == TPLA_BF16, kv_new->stride[0],
      reinterpret_cast<const int*>(positions->data), 0,
      page_table ? reinterpret_cast<const int*>(page_table->data) : nullptr,
      page_table ? page_table->stride[0] : 0, max_pages, kv_cache->shape[0], kv_cache->shape[1],
      kv_cache->data, kv_cache->stride[0], kv_cache->stride[1], (int)B, norm_groups, hadamard,
      eps, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TPLA_OK : cuda_fail(e);
}

int tpla_prefill_workspace_size(const tpla_tensor* q, size_t* bytes) {
  if (!bytes) return TPLA_ERR_INVALID_ARG;
  PrefillCall c;
  int rc = build_prefill(q, nullptr, 0, nullptr, nullptr, 1, 0, 0.f, 1.0f, nullptr, nullptr, &c);
  if (rc != TPLA_OK) return rc;
  *bytes = c.p.H > 0 ? sm100_workspace_bytes(c.p, 0, current_device()) : 0;
  return TPLA_OK;
}

int tpla_prefill(const tpla_tensor* q, const tpla_tensor* kv_new, int start,
                 const tpla_tensor* page_row, tpla_tensor* kv_cache, int norm_groups,
                 int hadamard, float eps, float scale, tpla_tensor* out, tpla_tensor* lse,
                 void* workspace, size_t workspace_bytes, tpla_stream_t stream) {
  PrefillCall c;
  int rc = build_prefill(q, kv_new, start, page_row, kv_cache, norm_groups, hadamard, eps, scale,
                         out, lse, &c);
  if (rc != TPLA_OK) return rc;
  const DecodeProblem& p = c.p;
  if (p.B == 0) return TPLA_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  size_t need = p.H > 0 ? sm100_workspace_bytes(p, 0, current_device()) : 0;
  if (workspace && (workspace_bytes < need || !aligned16(workspace))) return TPLA_ERR_WORKSPACE;
  // 1. the prompt rows into the cache (row b at position start + b)
  cudaError_t e = launch_cache_append(
      kv_new->data, kv_new->dtype == TPLA_BF16, kv_new->stride[0], nullptr, start,
      reinterpret_cast<const int*>(page_row->data), 0, (int)page_row->shape[0],
      kv_cache->shape[0], 0, kv_cache->data, kv_cache->stride[0], kv_cache->stride[1], p.B,
      norm_groups, hadamard, eps, s);
  if (e != cudaSuccess) return cuda_fail(e);
  if (p.H == 0) return TPLA_OK;
  // 2. exact MLA of every prompt token over its causal prefix
  void* ws = workspace;
  bool owned = false;
  if (!ws && need > 0) {
    e = cudaMallocAsync(&ws, need, s);
    if (e != cudaSuccess) return cuda_fail(e);
    owned = true;
  }
  e = launch_decode_sm100(p, 0, ws, need, s);
  rc = e == cudaSuccess ? TPLA_OK : cuda_fail(e);
  if (owned) {
    e = cudaFreeAsync(ws, s);
    if (rc == TPLA_OK && e != cudaSuccess) rc = cuda_fail(e);
  }
  return rc;
}

const char* tpla_error_string(int status) {
  switch (status) {
    case TPLA_OK: return "ok";
    case TPLA_ERR_INVALID_ARG: return "invalid argument";
    case TPLA_ERR_UNSUPPORTED: return "unsupported by the library";
    case TPLA_ERR_CUDA: return "CUDA error";
    case TPLA_ERR_WORKSPACE: return "workspace missing or too small";
    case TPLA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case TPLA_ERR_DEVICE_BOUNDS: return "page id or sequence length out of range";
    default: return "unknown status";
  }
}

int tpla_last_cuda_error(void) { return t_last_cuda_error; }

int tpla_get_device_status(tpla_stream_t stream, int* status) {
  if (!status) return TPLA_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  int a = 0, b = 0;
  e = status_read_clear_generic(&a);
  if (e != cudaSuccess) return cuda_fail(e);
  e = status_read_clear_sm100(&b);
  if (e != cudaSuccess) return cuda_fail(e);
  int c = 0, d = 0;
  e = status_read_clear_vup(&c);
  if (e != cudaSuccess) return cuda_fail(e);
  e = status_read_clear_append(&d);
  if (e != cudaSuccess) return cuda_fail(e);
  *status = a != 0 ? a : (b != 0 ? b : (c != 0 ? c : d));
  return TPLA_OK;
}

int tpla_selftest_wait_timeout(int microseconds, tpla_stream_t stream) {
  if (microseconds < 1 || microseconds > 1000000) return TPLA_ERR_INVALID_ARG;
  int dev = current_device();
  int khz = 0;
  if (cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev) != cudaSuccess || khz <= 0) {
    cudaGetLastError();
    khz = 2000000;
  }
  const long long cycles = (long long)microseconds * (khz / 1000);
  cudaError_t e = launch_wait_timeout_selftest(cycles, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TPLA_OK : cuda_fail(e);
}

int tpla_version(void) { return TPLA_VERSION; }

int64_t tpla_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
