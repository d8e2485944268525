// tpla_decode_noalloc: decode with a fixed, library-owned scratch buffer.
//
// Some callers cannot allocate device memory at the time they decode: code
// running inside a memory pool or arena that owns every byte of the GPU,
// embedded runtimes whose allocator must not be re-entered from a decode
// callback, and host code that runs where cudaMalloc is forbidden or too
// slow.  For them this entry point takes no workspace argument and never
// allocates: the split-KV partial results live in one file-scope __device__
// array, reserved when the library's code is loaded on a device and kept
// there until the process exits.  Under CUDA's lazy module loading that
// load happens at the first call on a device (the symbol lookup below), so
// the first call is the set-up call: it may reserve the buffer; later calls
// reserve nothing.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "tpla.h"

namespace tpla {
namespace {

// Fixed scratch capacity; every device that loads this library holds it.
constexpr size_t kScratchBytes = TPLA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code
// the symbol itself is only a handle; cudaGetSymbolAddress turns it into a
// pointer kernels may use.  Looked up once per device and cached; the cached
// address belongs to the device's current context, so the library must not
// be used across cudaDeviceReset (the buffer may be placed elsewhere after).
int scratch_for_current_device(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return TPLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TPLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return TPLA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return TPLA_OK;
}

}  // namespace
}  // namespace tpla

extern "C" int tpla_decode_noalloc(const tpla_tensor* q, const tpla_tensor* kv_cache,
                                   const tpla_tensor* seq_lens, const tpla_tensor* page_table,
                                   int G, int rope_mode, float scale, tpla_tensor* out,
                                   tpla_tensor* lse, int num_splits, int shard,
                                   tpla_stream_t stream) {
  tpla_decode_opts opts;
  opts.num_splits = num_splits;
  opts.shard = shard;
  opts.kernel = TPLA_KERNEL_AUTO;
  opts.reserved = 0;
  opts.workspace = nullptr;
  opts.workspace_bytes = 0;
  size_t need = 0;
  int rc = tpla_decode_workspace_size(q, kv_cache, seq_lens, page_table, G, rope_mode, out,
                                      &opts, &need);
  if (rc != TPLA_OK) return rc;
  if (need > tpla::kScratchBytes) return TPLA_ERR_WORKSPACE;  // beyond the fixed capacity
  // The set-up (symbol lookup, which also loads the buffer) runs on the first
  // valid call on a device whether or not that call needs scratch, so that
  // "make one call first" is enough for every later call.
  void* ws = nullptr;
  rc = tpla::scratch_for_current_device(&ws);
  if (rc != TPLA_OK) return rc;
  if (need > 0) {
    opts.workspace = ws;
    opts.workspace_bytes = tpla::kScratchBytes;
  }
  // Every scratch entry the kernels read is written earlier in the same
  // call, so nothing has to be cleared between calls.
  return tpla_decode_ex(q, kv_cache, seq_lens, page_table, G, rope_mode, scale, out, lse,
                        &opts, stream);
}
