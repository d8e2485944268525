/*
 * tpla.h -- C ABI of libtpla: single-token MLA decode attention over the
 * compressed latent KV cache (absorbed form) and its TPLA variant, on
 * NVIDIA B200 (sm_100a).
 *
 * What is computed (sources: the GitHub feature request "Bandwidth-optimal
 * tensor-parallel sharding of MLA (latent-cache sharding / TPLA)", sections
 * "Background / problem" and "Directions under investigation"; the TPLA
 * abstract; the pith.science review of arXiv 2508.15881, key machinery and
 * skeptic critique of Eq. 6):
 *
 *   Each cached token holds 576 values: 512 latent (c_KV) + 64 rope key.
 *   For request b, head h and shard g (G shards; d = 512 / G):
 *     s_t   = scale * ( q[b,h,I_g] . c_t[I_g]  +  q[b,h,R_g] . c_t[R_g] )
 *     out[b,h,I_g] = sum_t softmax_t(s) * c_t[I_g]
 *     lse[b,h,g]   = ln sum_t exp(s_t)
 *   I_g = [g*d, (g+1)*d).  R_g = all 64 rope columns (rope_mode REPLICATE)
 *   or the contiguous slice [512 + g*64/G, 512 + (g+1)*64/G) (SPLIT).
 *   G = 1 is exact MLA decode.  G > 1 is TPLA: every shard runs its own,
 *   unscaled softmax; shard outputs are laid side by side in latent space
 *   and later summed through the V up-projection (tpla_vup_combine), which
 *   stands in for the tensor-parallel all-reduce.
 *
 * Conventions for every entry point:
 *   - Tensors are described by tpla_tensor: data pointer, dtype, rank and
 *     per-dimension sizes and strides (strides in ELEMENTS).  The innermost
 *     dimension must be contiguous (stride 1).
 *   - All tensor data lives in device memory of the current CUDA device and
 *     is owned by the caller.  The library never frees or retains pointers.
 *   - Every call is asynchronous on `stream` (NULL = legacy default stream)
 *     and performs no host synchronisation, except tpla_get_device_status.
 *   - Inputs are never modified, except the buffer of tpla_hadamard_apply
 *     and the cache of tpla_cache_append / tpla_prefill.
 *   - Some kernels after the first of a call (the split-KV merge, the V
 *     up-projection) are launched as programmatic dependents of the kernel
 *     before them in the stream: they start their set-up early and read
 *     nothing before that kernel has finished and its writes are visible.
 *     Stream order, as the caller sees it, is unchanged.
 *   - Return value: TPLA_OK (0) or a negative tpla_status.  Arguments are
 *     validated before anything is launched; on an argument error nothing is
 *     launched and no memory is touched.  No C++ exception crosses the ABI.
 */
#ifndef TPLA_H
#define TPLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TPLA_VERSION 100

#if defined(__GNUC__)
#define TPLA_API __attribute__((visibility("default")))
#else
#define TPLA_API
#endif

/* cudaStream_t without including CUDA headers. */
typedef struct CUstream_st* tpla_stream_t;

enum tpla_dtype { TPLA_BF16 = 1, TPLA_F32 = 2, TPLA_I32 = 3 };

enum tpla_status {
  TPLA_OK = 0,
  TPLA_ERR_INVALID_ARG = -1,   /* null pointer, shape/stride/dtype mismatch  */
  TPLA_ERR_UNSUPPORTED = -2,   /* valid request the library cannot run       */
  TPLA_ERR_CUDA = -3,          /* a CUDA call failed; see tpla_last_cuda_error */
  TPLA_ERR_WORKSPACE = -4,     /* workspace missing or too small             */
  TPLA_ERR_DEVICE_TIMEOUT = -5,/* a kernel gave up waiting (device status)   */
  TPLA_ERR_DEVICE_BOUNDS = -6  /* a kernel met an out-of-range page id or
                                  sequence length (device status)            */
};

enum tpla_rope_mode { TPLA_ROPE_REPLICATE = 0, TPLA_ROPE_SPLIT = 1 };

enum tpla_kernel_choice {
  TPLA_KERNEL_AUTO = 0,     /* the tcgen05/TMA kernel (same as SM100)          */
  TPLA_KERNEL_GENERIC = 1,  /* portable CUDA-core kernel, only when named: a   */
                            /* reference point and the path for G = 8          */
  TPLA_KERNEL_SM100 = 2     /* tcgen05/TMA kernel; UNSUPPORTED if it cannot   */
};

typedef struct {
  void* data;
  int32_t dtype;     /* enum tpla_dtype */
  int32_t ndim;      /* 1..4 */
  int64_t shape[4];
  int64_t stride[4]; /* elements */
} tpla_tensor;

typedef struct {
  /* 0 = automatic split of the KV sequence (balanced over the GPU's SMs);
     k >= 1 = cut every request's tokens into k equal chunks and merge them
     with the log-sum-exp rule.  1 = no split. */
  int32_t num_splits;
  /* -1 = compute all G shards.  s in [0, G) = one-shard mode: read only the
     columns shard s needs (the bytes one tensor-parallel rank reads) and
     write out [B, H, d], lse [B, H, 1]. */
  int32_t shard;
  int32_t kernel;    /* enum tpla_kernel_choice */
  int32_t reserved;  /* must be 0 */
  /* Device scratch for split partial results; see
     tpla_decode_workspace_size.  May be NULL when the size is 0. */
  void* workspace;
  size_t workspace_bytes;
} tpla_decode_opts;

/*
 * tpla_decode_ex -- latent-KV decode attention, MLA (G = 1) or TPLA (G > 1).
 *
 *   q          [B, H, 576] bf16.  Query in absorbed form (q_nope already
 *              multiplied by W_UK, then rope query).  Rows must start on
 *              16-byte boundaries (stride[1] % 8 == 0, data 16-byte aligned).
 *   kv_cache   paged:      [num_blocks, 64, 576] bf16 (64-token pages),
 *              contiguous: [B, Lmax, 576] bf16 when page_table is NULL.
 *              stride[1] % 8 == 0, stride[0] % 8 == 0, 16-byte aligned.
 *   seq_lens   [B] int32: tokens of each request (0 allowed).
 *   page_table [B, max_pages] int32 or NULL.  Entry p of row b is the
 *              physical block holding tokens [64p, 64p + 64) of request b;
 *              only entries p < ceil(seq_lens[b] / 64) are read.
 *   G          1, 2, 4 or 8 latent shards.
 *   rope_mode  TPLA_ROPE_REPLICATE or TPLA_ROPE_SPLIT.
 *   scale      softmax scale applied to the dot products (finite).
 *   out        [B, H, 512] (or [B, H, d] in one-shard mode), f32 or bf16.
 *   lse        NULL or [B, H, G] (one-shard: [B, H, 1]) f32, natural log.
 *   opts       NULL = defaults {0, -1, AUTO, 0, NULL, 0}.
 *
 * A request with seq_lens = 0 gets out = 0 and lse = -inf.  Page ids outside
 * [0, num_blocks) or seq_lens larger than the cache can hold are not read;
 * the kernel records TPLA_ERR_DEVICE_BOUNDS in the device status word
 * (tpla_get_device_status) and treats the missing tokens as absent.
 *
 * Precondition: the rows of a request's last page (contiguous mode: of its
 * last 64-row block inside the cache) past seq_lens[b] must hold finite
 * values.  The tensor-core path reads whole pages and gives those rows zero
 * weight after the softmax, and 0 * NaN is NaN.
 *
 * Kernel choice (opts->kernel = AUTO or SM100): the tcgen05 kernel, which
 * needs an sm_100 device, G of 1, 2 or 4 and out rows on 16-byte boundaries
 * (data 16-byte aligned, stride[0] and stride[1] multiples of 16 bytes);
 * otherwise TPLA_ERR_UNSUPPORTED before any launch.  Any finite scale
 * (negative and zero included) and any H (one launch per group of 128
 * heads) are taken.  The portable kernel (opts->kernel = GENERIC) computes
 * the same function and runs only when named.
 *
 * Size limits (TPLA_ERR_UNSUPPORTED beyond them, nothing launched):
 * B <= 2^20, H <= 4096, B * H <= 2^30, num_splits <= 65535,
 * B * num_splits <= 2^24, and on the portable kernel B * shards <= 65535.
 */
TPLA_API int tpla_decode_ex(const tpla_tensor* q, const tpla_tensor* kv_cache,
                   const tpla_tensor* seq_lens, const tpla_tensor* page_table,
                   int G, int rope_mode, float scale,
                   tpla_tensor* out, tpla_tensor* lse,
                   const tpla_decode_opts* opts, tpla_stream_t stream);

/*
 * tpla_decode_workspace_size -- bytes of device workspace tpla_decode_ex
 * needs for these arguments and options (0 when no split is used).  Same
 * validation as tpla_decode_ex; writes the size to *bytes.
 */
TPLA_API int tpla_decode_workspace_size(const tpla_tensor* q, const tpla_tensor* kv_cache,
                               const tpla_tensor* seq_lens,
                               const tpla_tensor* page_table, int G,
                               int rope_mode, const tpla_tensor* out,
                               const tpla_decode_opts* opts, size_t* bytes);

/*
 * tpla_decode -- tpla_decode_ex with default options.  When a split is used
 * the workspace comes from the stream-ordered allocator (cudaMallocAsync /
 * cudaFreeAsync on `stream`), so this convenience call allocates; callers
 * that manage memory themselves use tpla_decode_ex.
 */
TPLA_API int tpla_decode(const tpla_tensor* q, const tpla_tensor* kv_cache,
                const tpla_tensor* seq_lens, const tpla_tensor* page_table,
                int G, int rope_mode, float scale, tpla_tensor* out,
                tpla_tensor* lse, tpla_stream_t stream);

/*
 * tpla_decode_noalloc -- tpla_decode_ex for callers that cannot allocate
 * device memory while they decode (a caller whose memory pool or arena owns
 * the whole GPU, a runtime whose allocator must not be re-entered from the
 * decode call, code paths where cudaMalloc is not allowed).  The source
 * pages have no counterpart; this is a library convenience.
 *
 * Same arguments and results as tpla_decode_ex with opts = {num_splits,
 * shard, TPLA_KERNEL_AUTO}; there is no workspace argument.  Split-KV
 * partial results go to one fixed scratch buffer of
 * TPLA_NOALLOC_SCRATCH_BYTES bytes that the library reserves in device
 * memory on every GPU where it is loaded and keeps until the process exits.
 * This call never calls cudaMalloc, cudaFree or any allocating routine.
 *   - A problem whose workspace (tpla_decode_workspace_size) exceeds that
 *     capacity is rejected with TPLA_ERR_WORKSPACE before any launch.
 *   - The first valid call on a device is its set-up call: it looks up the
 *     buffer's device address (cudaGetSymbolAddress, once per device, with
 *     that device current).  Under CUDA's lazy module loading (the default)
 *     that lookup is also what loads the buffer, so the first call may
 *     reserve TPLA_NOALLOC_SCRATCH_BYTES of device memory.  Make one call
 *     on each device before handing its memory to an arena or pool and
 *     before capturing a stream; later calls reserve nothing.
 *   - The address is kept for the life of the process: do not use the
 *     library on a device after cudaDeviceReset on it.
 *   - All calls on a device share the one buffer and it keeps the previous
 *     call's contents (nothing needs clearing: every entry read is written
 *     earlier in the same call).  Calls whose kernels overlap on the GPU,
 *     e.g. on two streams without ordering, race on the buffer; order them.
 */
#define TPLA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
TPLA_API int tpla_decode_noalloc(const tpla_tensor* q, const tpla_tensor* kv_cache,
                                 const tpla_tensor* seq_lens, const tpla_tensor* page_table,
                                 int G, int rope_mode, float scale, tpla_tensor* out,
                                 tpla_tensor* lse, int num_splits, int shard,
                                 tpla_stream_t stream);

/*
 * tpla_lse_merge -- exact merge of S partial attention results over disjoint
 * key chunks (the log-sum-exp rule of the sequence-split alternative in the
 * feature request's "Directions under investigation").
 *   o_parts   [S, B, H, Wd] f32, each chunk's normalised output.
 *   lse_parts [S, B, H, Gs] f32; Wd must be a multiple of Gs and shard k of
 *             a row owns columns [k*Wd/Gs, (k+1)*Wd/Gs).
 *   out       [B, H, Wd] f32 or bf16;  lse NULL or [B, H, Gs] f32.
 * lse = ln sum_s exp(lse_s); out = sum_s exp(lse_s - lse) o_s.  Chunks with
 * lse = -inf contribute nothing; if every chunk is -inf, out = 0, lse = -inf.
 * Limits (TPLA_ERR_UNSUPPORTED): S <= 1024, B * H <= 2^30, Wd <= 2^20.
 */
TPLA_API int tpla_lse_merge(const tpla_tensor* o_parts, const tpla_tensor* lse_parts,
                   tpla_tensor* out, tpla_tensor* lse, tpla_stream_t stream);

/*
 * tpla_hadamard_apply -- in-place orthonormal Walsh-Hadamard transform of
 * the first `dim` columns of every row of `buf` (Sylvester / natural order,
 * entries (-1)^popcount(i & j) / sqrt(dim)); other columns are untouched.
 * The transform is its own inverse.  The orthogonal reparameterisation
 * applied before slicing (feature request, "Directions under investigation";
 * TPLA abstract).
 *   buf  bf16 or f32, ndim 1..4, innermost dimension >= dim and contiguous;
 *        every other dimension indexes rows.
 *   dim  power of two in [32, 1024].
 * Arithmetic is f32; bf16 rows are rounded once on store.
 */
TPLA_API int tpla_hadamard_apply(tpla_tensor* buf, int dim, tpla_stream_t stream);

/*
 * tpla_vup_combine -- y[b, h, :] = sum_j out_latent[b, h, j] * W_uv[h, j, :].
 * The V up-projection; with shard outputs laid side by side in latent space,
 * the contraction over j is the sum over shards that the tensor-parallel
 * all-reduce performs (feature request, "Directions under investigation").
 *   out_latent [B, H, K] f32 or bf16;  W_uv [H, K, Dv] bf16, Dv a multiple
 *   of 16 and <= 256;  y [B, H, Dv] f32.  K = 512 (the whole latent) or any
 *   multiple of 64 up to 512: with K = 512 / G, the one-shard output of
 *   rank g (tpla_decode_ex with opts->shard = g) and the rows I_g of W_uv
 *   give that rank's partial product, which the all-reduce sums.
 * Accumulation is f32 on tensor cores; an f32 out_latent is split into two
 * bf16 terms (hi + lo) so that its rounding does not limit accuracy.
 */
TPLA_API int tpla_vup_combine(const tpla_tensor* out_latent, const tpla_tensor* W_uv,
                     tpla_tensor* y, tpla_stream_t stream);

/*
 * PCA reparameterisation (TPLA abstract; feature request, "Directions under
 * investigation": PCA beside the Hadamard transform as the orthogonal change
 * of basis applied before slicing; the TPLA review's referee comments on
 * Sec. 4.3.2 / Eq. 25: PCA of the latent cache features, rope excluded).
 * The library computes the calibration statistics and applies a basis; the
 * 512 x 512 eigensolve that turns the covariance into U is the caller's,
 * offline.
 *
 * tpla_latent_covariance -- accumulates, over the first 512 columns x of every
 * row of `rows` ([N, >= 512] or [B, H, >= 512] bf16, innermost contiguous,
 * 16-byte aligned rows):  C[i][j] += sum x_i x_j  and  s[i] += sum x_i.
 *   C [512, 512] f32 and s [512] f32, zeroed by the caller before the first
 *   call; several calls accumulate.  f32 arithmetic, atomic adds (the sum
 *   order is not fixed).
 * tpla_covariance_finalize -- mean = s / n, cov = C / n - mean mean^T
 *   (n = rows accumulated), both f32; cov [512, 512], mean [512].
 * tpla_rotate_apply -- in place, x <- x U on the first 512 columns of every row
 *   of `buf` (same layouts as `rows` above); other columns untouched.
 *   U [512, 512] bf16, row-major and contiguous (U[j][n] multiplies x_j into
 *   output n).  `scratch` is caller device memory of at least
 *   H * 512 * 4 bytes (H = 1 for two-dimensional buf); larger scratch lets
 *   the rows go through in fewer, longer passes.  Tensor-core bf16 products,
 *   f32 accumulation, one bf16 rounding on store.
 * Errors: TPLA_ERR_INVALID_ARG for shapes, dtypes, strides or alignment;
 * TPLA_ERR_WORKSPACE for missing or short scratch.
 */
TPLA_API int tpla_latent_covariance(const tpla_tensor* rows, tpla_tensor* C, tpla_tensor* s,
                                    tpla_stream_t stream);
TPLA_API int tpla_covariance_finalize(const tpla_tensor* C, const tpla_tensor* s, int64_t n,
                                      tpla_tensor* cov, tpla_tensor* mean,
                                      tpla_stream_t stream);
TPLA_API int tpla_rotate_apply(tpla_tensor* buf, const tpla_tensor* U, void* scratch,
                               size_t scratch_bytes, tpla_stream_t stream);

/*
 * tpla_cache_append -- store each request's new token in the latent cache,
 * normalised the way the shards read it.  The review of arXiv 2508.15881
 * (key machinery): the stored latent is the RMS-normalised down-projection
 * (its gain absorbed into the up-projections, like the rotation U), and in
 * TPLA every rank normalises its own slice, which Condition 1 asks to track
 * the global norm; its referee report calls Proposition 1 (RMSNorm commutes
 * with an orthogonal transform) correct.  The feature request ("Directions
 * under investigation") applies the Hadamard reparameterisation on this
 * path (kv_a_layernorm).
 *   kv_new      [B, 576] bf16 or f32, rows 16-byte aligned: columns 0..511
 *               the token's latent before normalisation, 512..575 its
 *               position-encoded rope key (stored as given).
 *   positions   [B] int32: token index each request writes (its length
 *               before this token, for appending).
 *   page_table  [B, max_pages] int32 (paged cache) or NULL (contiguous).
 *   kv_cache    paged [num_blocks, 64, 576] or contiguous [B, Lmax, 576]
 *               bf16, the layout tpla_decode_ex reads; 16-byte aligned rows.
 *   norm_groups 1: one RMS over all 512 latent columns (exact MLA); 2, 4 or
 *               8: each contiguous shard of 512 / norm_groups columns
 *               divided by its own RMS (one TPLA rank per shard).
 *   hadamard    1: rotate the latent by the orthonormal Walsh-Hadamard matrix
 *               (tpla_hadamard_apply's) before the norm; 0: no rotation.
 *   eps         >= 0, added to each mean square.
 * Stored row: latent x (rotated if asked), each shard x_g / sqrt(mean(x_g^2)
 * + eps), f32 arithmetic, rounded once to bf16; rope copied.  A position
 * outside the cache or a page id outside [0, num_blocks) is not written: the
 * kernel records TPLA_ERR_DEVICE_BOUNDS (tpla_get_device_status).  Nothing
 * else of the cache is touched.  Asynchronous on `stream`; allocates nothing.
 * Errors before any launch: TPLA_ERR_INVALID_ARG (shapes, dtypes, strides,
 * alignment, norm_groups, hadamard, eps); TPLA_ERR_UNSUPPORTED (B > 2^20,
 * paged cache with pages other than 64 tokens).
 */
TPLA_API int tpla_cache_append(const tpla_tensor* kv_new, const tpla_tensor* positions,
                               const tpla_tensor* page_table, tpla_tensor* kv_cache,
                               int norm_groups, int hadamard, float eps,
                               tpla_stream_t stream);

/*
 * tpla_prefill -- the prefill half of prefill/decode separation, for T prompt
 * tokens of one request.  The TPLA abstract: models pre-trained with MLA keep
 * MLA-style prefilling and decode tensor-parallel; the TPLA review (referee
 * report, major comment on Table 2 and the abstract; forward implications):
 * the separated variant runs exact MLA in the compute-bound prefill and TPLA
 * only in decode.  Two steps, in stream order on `stream`:
 *  1. row i of kv_new is stored at position start + i of the request,
 *     exactly as tpla_cache_append stores a row (optional Hadamard rotation,
 *     RMS norm over norm_groups slices, one bf16 rounding);
 *  2. prompt token i gets exact MLA attention -- one softmax over all 576
 *     values of each token, absorbed form, G = 1 -- over the request's stored
 *     rows 0 .. start + i (causal): out[i] and lse[i].  The tcgen05 kernel of
 *     tpla_decode_ex runs it with one query row per prompt token, the
 *     lengths start + i + 1 computed in the kernel and the page-table row
 *     shared by every query row; the split-KV merge follows.
 * A later tpla_decode_ex of the request (any G) reads the same stored rows.
 *   q         [T, H, 576] bf16: the prompt tokens' absorbed queries (the
 *             layout of tpla_decode_ex's q; 16-byte aligned rows).
 *   kv_new    [T, 576] bf16 or f32: tpla_cache_append's row layout.
 *   start     >= 0: tokens of the request already in the cache.
 *   page_row  [max_pages] int32, contiguous: the request's page-table row;
 *             start + T <= 64 * max_pages.  Page ids must lie in
 *             [0, num_blocks): others are not written or read, and the
 *             kernels record TPLA_ERR_DEVICE_BOUNDS.
 *   kv_cache  [num_blocks, 64, 576] bf16, the paged layout (16-byte aligned
 *             rows); updated in place.
 *   norm_groups, hadamard, eps: as in tpla_cache_append.
 *   scale     softmax scale, any finite value (as in tpla_decode_ex).
 *   out       [T, H, 512] f32 or bf16 (16-byte aligned rows); lse [T, H, 1]
 *             f32 or NULL.
 *   workspace split scratch of at least tpla_prefill_workspace_size bytes,
 *             16-byte aligned, or NULL: the call then takes it from the
 *             stream-ordered allocator (cudaMallocAsync / cudaFreeAsync on
 *             `stream`), as tpla_decode does.
 * Errors before any launch: TPLA_ERR_INVALID_ARG (shapes, dtypes, strides,
 * alignment, start, a page row too short for start + T, norm_groups,
 * hadamard, eps, scale); TPLA_ERR_UNSUPPORTED (T > 2^20, H > 4096,
 * T * H > 2^30, pages other than 64 tokens, no sm_100 GPU);
 * TPLA_ERR_WORKSPACE (a workspace that is short or misaligned).
 */
TPLA_API int tpla_prefill(const tpla_tensor* q, const tpla_tensor* kv_new, int start,
                          const tpla_tensor* page_row, tpla_tensor* kv_cache, int norm_groups,
                          int hadamard, float eps, float scale, tpla_tensor* out,
                          tpla_tensor* lse, void* workspace, size_t workspace_bytes,
                          tpla_stream_t stream);

/* tpla_prefill_workspace_size -- bytes of workspace tpla_prefill needs for
 * queries q ([T, H, 576] bf16) on the current device. */
TPLA_API int tpla_prefill_workspace_size(const tpla_tensor* q, size_t* bytes);

/* Human-readable name of a tpla_status code (static string). */
TPLA_API const char* tpla_error_string(int status);

/* The cudaError_t of the most recent TPLA_ERR_CUDA on this host thread. */
TPLA_API int tpla_last_cuda_error(void);

/*
 * tpla_get_device_status -- synchronise `stream`, then read and clear the
 * status word the kernels of this library set on the current device
 * (TPLA_OK, TPLA_ERR_DEVICE_BOUNDS or TPLA_ERR_DEVICE_TIMEOUT).
 */
TPLA_API int tpla_get_device_status(tpla_stream_t stream, int* status);

/* Number of CUDA kernels this library has launched in this process (all
 * devices, all host threads).  Lets a caller count the library's launches
 * inside a timed region. */
TPLA_API int64_t tpla_launch_count(void);

/*
 * tpla_selftest_wait_timeout -- test support for the device failure path;
 * the pages have no counterpart.  Launches one thread that waits, through
 * the same bounded barrier wait the decode kernels use, on a barrier that
 * nothing completes.  After about `microseconds` (1 .. 1e6) of SM clock the
 * wait gives up, records TPLA_ERR_DEVICE_TIMEOUT in the device status word
 * and the kernel returns; the context stays usable.  Read the status with
 * tpla_get_device_status.  Asynchronous on `stream`.
 */
TPLA_API int tpla_selftest_wait_timeout(int microseconds, tpla_stream_t stream);

/* TPLA_VERSION of the loaded library. */
TPLA_API int tpla_version(void);

#ifdef __cplusplus
}
#endif
#endif /* TPLA_H */
