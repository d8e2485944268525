// V up-projection combine: y[b, h, :] = sum_j out[b, h, j] W_uv[h, j, :],
// over j < K (K = 512 for the whole latent; K = 512 / G for one rank's
// shard, whose partial product the tensor-parallel all-reduce sums).
//
// In TPLA the shard outputs are combined by the existing o_proj all-reduce
// (feature request "Bandwidth-optimal tensor-parallel sharding of MLA",
// section "Directions under investigation"); with the G shard outputs laid
// side by side in latent space, the sum over shards is exactly the
// contraction over j here, so this kernel stands in for that all-reduce.
//
// Per head h this is a small GEMM, computed transposed on the 5th-generation
// tensor core:  Y_h^T [Dv x B] = W_h^T [Dv x 512] . out_h^T [512 x B], so the
// MMA's M is the V dimension (128 per accumulator, two accumulators for
// Dv > 128) and N the batch tile (up to 64 requests).  The op reads W_uv
// (H * 512 * Dv bf16) and out (B * H * 512, f32 or bf16) once and is bound by
// HBM; what matters is many bytes in flight per SM:
//  * one CTA per (head, batch tile); W and out arrive by TMA (no multicast)
//    in 64-column K chunks through a ring of up to 8 stages (~160 KB in
//    flight per SM);
//  * W lands MN-major in the 128-byte swizzle the MMA reads directly; a bf16
//    `out` lands K-major the same way; an f32 `out` lands as plain rows and
//    four converter warps split it into hi + lo bf16 tiles (out = hi + lo to
//    about 16 mantissa bits), each multiplied by the same W tile;
//  * one thread issues the tcgen05 MMAs into TMEM; the converter warps read
//    the accumulators back and store y.
// Every barrier wait is bounded; on timeout the kernel records
// TPLA_ERR_DEVICE_TIMEOUT in its status word and stops.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace tpla {
namespace {

using namespace ptx;

constexpr int kKC = 64;                   // latent columns per K chunk
constexpr int kMaxKChunks = kLatent / kKC;  // 8
constexpr int kMaxN = 64;                 // batch rows per CTA (MMA N)
constexpr int kWBox = 8192;               // one [64 j][64 v] bf16 tile
constexpr int kConvStages = 2;
constexpr int kMaxRaw = 8;
constexpr int kThreads = 192;             // warp 0 TMA, warp 1 MMA, warps 2-5 convert + store
constexpr int kSmemBudget = 200 * 1024;
constexpr long long kTimeoutCycles = 4000000000LL;  // about 2 s at full clock

__device__ int g_vup_status;

struct VupParams {
  float* y;
  int64_t y_sb, y_sh;
  int B, H, Dv;
  int kc;          // K chunks of 64 latent columns (K / 64, 1 .. 8)
  int mh;          // 128-row halves of Dv (1 or 2)
  int nt;          // batch rows per tile (MMA N), multiple of 16, <= 64
  int out_bf16;
  int raw_stages;
  uint32_t raw_bytes;  // per stage: mh * 2 W tiles, then the out tile (1 KB aligned)
  uint32_t tx_bytes;   // bytes the TMA copies of one stage deliver
  uint32_t o_bytes;    // out tile bytes (nt rows of 64 values)
  uint32_t off_conv, off_bar;
};

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      :
      : "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      :
      : "r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Bounded wait; false on timeout (status recorded) or when another role
// already gave up.
__device__ bool wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_sleep(bar, parity, 20000)) return true;
    if ((i & 15) == 0) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kTimeoutCycles) {
        atomicCAS(&g_vup_status, 0, TPLA_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ uint32_t bf16_bits(float x) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__global__ void __launch_bounds__(kThreads, 1)
vup_sm100_kernel(const __grid_constant__ CUtensorMap wmap,
                 const __grid_constant__ CUtensorMap omap, const VupParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x;
  const int b0 = blockIdx.y * p.nt;
  const int R = p.raw_stages;
  const uint32_t bar0 = sbase + p.off_bar;
  auto raw_full = [&](int s) { return bar0 + 8 * s; };
  auto raw_empty = [&](int s) { return bar0 + 8 * (kMaxRaw + s); };
  auto conv_full = [&](int c) { return bar0 + 8 * (2 * kMaxRaw + c); };
  auto conv_empty = [&](int c) { return bar0 + 8 * (2 * kMaxRaw + kConvStages + c); };
  const uint32_t acc_full = bar0 + 8 * (2 * kMaxRaw + 2 * kConvStages);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + p.off_bar + 8 * (2 * kMaxRaw + 2 * kConvStages + 1));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < R; ++s) {
      mbar_init(raw_full(s), 1);
      mbar_init(raw_empty(s), 1);
    }
    for (int c = 0; c < kConvStages; ++c) {
      mbar_init(conv_full(c), 4);  // one arrival per converter warp
      mbar_init(conv_empty(c), 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {  // accumulators: mh blocks of 64 columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(p.mh == 2 ? 128u : 64u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  // launched as a programmatic dependent of the kernel before it (the merge
  // or the decode that wrote `out`): the set-up above overlaps its end, and
  // nothing is read before that grid and its writes are complete
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // One SM's bulk copies from a single issuing thread complete one after
    // another, so the boxes of a stage go out from different lanes: box i
    // (W tiles, then the out tile) of stage s from lane nbox * s + i (the
    // launcher keeps nbox * stages <= 32).
    const int nbox = 2 * p.mh + 1;
    if (lane == 0) {
      tma_prefetch(&wmap);
      tma_prefetch(&omap);
    }
    int issued = 0;
    for (int k = 0; k < p.kc; ++k) {
      const int s = k % R;
      int ok = 1;
      if (lane == 0) {
        if (k >= R) ok = wait(raw_empty(s), ((k / R) - 1) & 1, abort_flag);
        if (ok) mbar_arrive_expect_tx(raw_full(s), p.tx_bytes);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const int i = lane - nbox * s;
      if (i >= 0 && i < nbox) {
        const uint32_t st = sbase + (uint32_t)s * p.raw_bytes;
        if (i < 2 * p.mh)
          tma_load_3d(st + (uint32_t)i * kWBox, &wmap, 64 * i, kKC * k, h, raw_full(s));
        else
          tma_load_3d(st + (uint32_t)(2 * p.mh) * kWBox, &omap, kKC * k, h, b0, raw_full(s));
      }
      issued = k + 1;
    }
    // copies still in flight after an abort land before the CTA exits
    if (lane == 0)
      for (int k = issued - R < 0 ? 0 : issued - R; k < issued && *abort_flag; ++k) {
        const long long t0 = clock64();
        while (!mbar_try_wait(raw_full(k % R), (k / R) & 1) && clock64() - t0 < kTimeoutCycles) {
        }
      }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, p.nt, true, false);
      bool ok = true;
      for (int k = 0; k < p.kc && ok; ++k) {
        const int s = k % R, c = k % kConvStages;
        ok = wait(raw_full(s), (k / R) & 1, abort_flag);
        if (ok && !p.out_bf16) ok = wait(conv_full(c), (k / kConvStages) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t st = sbase + (uint32_t)s * p.raw_bytes;
        // out^T operands: K-major [nt rows][64 j]; f32 out gives hi and lo
        const uint32_t o0 = p.out_bf16 ? st + (uint32_t)(2 * p.mh) * kWBox
                                       : sbase + p.off_conv + (uint32_t)c * 2 * p.o_bytes;
        const int nterms = p.out_bf16 ? 1 : 2;
        for (int m = 0; m < p.mh; ++m) {
          const uint64_t a0 = sw128_desc(st + (uint32_t)(2 * m) * kWBox, kWBox, 1024);
          for (int t = 0; t < nterms; ++t) {
            const uint64_t bd = sw128_desc(o0 + (uint32_t)t * p.o_bytes, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // K-steps of 16: A +2 KB (MN-major), B +32 B
              mma_f16(tmem + 64 * m, a0 + (uint64_t)(kk * 128), bd + (uint64_t)(kk * 2), idesc,
                      (k | kk | t) != 0);
          }
        }
        mma_commit(raw_empty(s));
        if (!p.out_bf16) mma_commit(conv_empty(c));
      }
      mma_commit(acc_full);
      if (!ok) {  // let issued MMAs finish before the accumulators are freed
        const long long t0 = clock64();
        while (!mbar_try_wait(acc_full, 0) && clock64() - t0 < kTimeoutCycles) {
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- converters + epilogue
    const int ct = threadIdx.x - 64;  // 0..127
    bool ok = true;
    if (!p.out_bf16) {
      const int items = p.nt * 8;  // (row, 8-column group) per chunk
      for (int k = 0; k < p.kc && ok; ++k) {
        const int s = k % R, c = k % kConvStages;
        ok = wait(raw_full(s), (k / R) & 1, abort_flag);
        if (ok && k >= kConvStages) ok = wait(conv_empty(c), ((k / kConvStages) - 1) & 1, abort_flag);
        if (!ok) break;
        const uint8_t* stage = smem + (size_t)s * p.raw_bytes + (size_t)(2 * p.mh) * kWBox;
        const uint32_t hi = sbase + p.off_conv + (uint32_t)c * 2 * p.o_bytes;
        const uint32_t lo = hi + p.o_bytes;
        for (int i = ct; i < items; i += 128) {
          const int r = i >> 3, g = i & 7;
          const float4 x0 = *reinterpret_cast<const float4*>(stage + r * 256 + g * 32);
          const float4 x1 = *reinterpret_cast<const float4*>(stage + r * 256 + g * 32 + 16);
          const float v[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          uint32_t ph[4], pl[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t h0 = bf16_bits(v[2 * e]), h1 = bf16_bits(v[2 * e + 1]);
            const float r0 = v[2 * e] - __uint_as_float(h0 << 16);
            const float r1 = v[2 * e + 1] - __uint_as_float(h1 << 16);
            ph[e] = h0 | (h1 << 16);
            pl[e] = bf16_bits(r0) | (bf16_bits(r1) << 16);
          }
          const uint32_t off = (uint32_t)r * 128 + ((uint32_t)(g ^ (r & 7)) << 4);
          st_shared_v4(hi + off, ph[0], ph[1], ph[2], ph[3]);
          st_shared_v4(lo + off, pl[0], pl[1], pl[2], pl[3]);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(conv_full(c));
      }
    }
    if (ok) ok = wait(acc_full, 0, abort_flag) && !*abort_flag;
    if (ok) {
      tc_fence_after();
      const int q = warp & 3;  // TMEM lanes 32q .. 32q + 31
      for (int m = 0; m < p.mh; ++m) {
        const int v = 128 * m + 32 * q + lane;
        for (int c0 = 0; c0 < p.nt; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + 64 * m + c0, r);
          tmem_wait_ld();
          if (v < p.Dv) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int b = b0 + c0 + i;
              if (c0 + i < p.nt && b < p.B)
                p.y[(int64_t)b * p.y_sb + (int64_t)h * p.y_sh + v] = __uint_as_float(r[i]);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(p.mh == 2 ? 128u : 64u)
                 : "memory");
  }
}

std::mutex g_vup_mu;
bool g_vup_attr[64] = {};

}  // namespace

bool vup_supported(const void* out_latent, int out_bf16, int64_t o_sb, int64_t o_sh,
                   const void* W, int64_t w_sh, int64_t w_sj) {
  const int64_t esz = out_bf16 ? 2 : 4;
  auto a16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; };
  return a16(out_latent) && a16(W) && (o_sb * esz) % 16 == 0 && (o_sh * esz) % 16 == 0 &&
         (w_sh * 2) % 16 == 0 && (w_sj * 2) % 16 == 0;
}

cudaError_t launch_vup(const void* out_latent, int out_bf16, int64_t o_sb, int64_t o_sh,
                       const void* W, int64_t w_sh, int64_t w_sj, float* y, int64_t y_sb,
                       int64_t y_sh, int B, int H, int Dv, int K, cudaStream_t stream) {
  if (B == 0 || H == 0 || Dv == 0) return cudaSuccess;
  if (!vup_supported(out_latent, out_bf16, o_sb, o_sh, W, w_sh, w_sj) || Dv > 256 || Dv % 16 ||
      K < kKC || K > kLatent || K % kKC)
    return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!sm100_device(dev)) return cudaErrorNotSupported;
  auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!encode) return cudaErrorNotSupported;

  VupParams p{};
  p.y = y;
  p.y_sb = y_sb;
  p.y_sh = y_sh;
  p.B = B;
  p.H = H;
  p.Dv = Dv;
  p.kc = K / kKC;
  p.mh = Dv > 128 ? 2 : 1;
  p.nt = B >= kMaxN ? kMaxN : ((B + 15) / 16) * 16;
  p.out_bf16 = out_bf16;
  p.o_bytes = (uint32_t)p.nt * (out_bf16 ? 128u : 256u);
  const uint32_t conv_tile = (uint32_t)p.nt * 128u;  // one bf16 K-major tile
  p.tx_bytes = (uint32_t)(2 * p.mh) * kWBox + p.o_bytes;
  p.raw_bytes = (p.tx_bytes + 1023u) & ~1023u;
  const uint32_t conv_bytes = out_bf16 ? 0u : ((kConvStages * 2 * conv_tile + 1023u) & ~1023u);
  int R = (int)((kSmemBudget - conv_bytes) / p.raw_bytes);
  p.raw_stages = R > kMaxRaw ? kMaxRaw : R;
  while (p.raw_stages * (2 * p.mh + 1) > 32) --p.raw_stages;  // one issuing lane per box
  p.off_conv = (uint32_t)p.raw_stages * p.raw_bytes;
  p.o_bytes = out_bf16 ? p.o_bytes : conv_tile;  // the MMA reads hi/lo tiles of nt x 128 B
  p.off_bar = p.off_conv + conv_bytes;
  const uint32_t smem = p.off_bar + 8 * (2 * kMaxRaw + 2 * kConvStages + 1) + 16 + 1024;

  // W as [H][K][Dv] (v innermost): boxes of 64 v x 64 j, MN-major for the MMA
  CUtensorMap wmap, omap;
  {
    cuuint64_t dims[3] = {(cuuint64_t)Dv, (cuuint64_t)K, (cuuint64_t)H};
    cuuint64_t strides[2] = {(cuuint64_t)w_sj * 2, (cuuint64_t)w_sh * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kKC, 1};
    cuuint32_t es[3] = {1, 1, 1};
    if (encode(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(W), dims, strides,
               box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // out as [B][H][K] (j innermost): boxes of 64 j x 1 head x nt requests
  {
    const uint64_t esz = out_bf16 ? 2 : 4;
    cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)H, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)o_sh * esz, (cuuint64_t)o_sb * esz};
    cuuint32_t box[3] = {(cuuint32_t)kKC, 1, (cuuint32_t)p.nt};
    cuuint32_t es[3] = {1, 1, 1};
    if (encode(&omap,
               out_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
               const_cast<void*>(out_latent), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE,
               out_bf16 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    std::lock_guard<std::mutex> lock(g_vup_mu);
    if (!g_vup_attr[dev & 63]) {
      cudaError_t e = cudaFuncSetAttribute(vup_sm100_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kSmemBudget + 4096);
      if (e != cudaSuccess) return e;
      g_vup_attr[dev & 63] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(H, (B + p.nt - 1) / p.nt);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, vup_sm100_kernel, wmap, omap, p);
  count_launch();
  return e;
}

cudaError_t status_read_clear_vup(int* code) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_vup_status, sizeof(int));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    int zero = 0;
    e = cudaMemcpyToSymbol(g_vup_status, &zero, sizeof(int));
  }
  *code = v;
  return e;
}

}  // namespace tpla
