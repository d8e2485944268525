// tcgen05 / TMA MLA decode kernel for sm_100a (in progress: not yet enabled).
#include "internal.h"

namespace tpla {
namespace {
__device__ int g_status;
}

bool sm100_supported(const DecodeProblem&, int) { return false; }
size_t sm100_workspace_bytes(const DecodeProblem&, int, int) { return 0; }
cudaError_t launch_decode_sm100(const DecodeProblem&, int, void*, size_t, cudaStream_t) {
  return cudaErrorNotSupported;
}

cudaError_t status_read_clear_sm100(int* code) {
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
