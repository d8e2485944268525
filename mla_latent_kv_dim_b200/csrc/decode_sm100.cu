// MLA / TPLA latent-KV decode on the 5th-generation tensor cores (sm_100a).
//
// What it computes (feature request "Bandwidth-optimal tensor-parallel
// sharding of MLA", sections "Background / problem" and "Directions under
// investigation"; TPLA abstract; review of arXiv 2508.15881, key machinery
// and the skeptic's description of Eq. 6 as an unscaled local softmax):
// for every request b, head h and shard g,
//   s_t = scale * (q[I_g] . c_t[I_g] + q[R_g] . c_t[R_g])
//   out[I_g] = softmax_t(s) c_t[I_g],  lse_g = ln sum_t exp(s_t).
// All heads share one latent row per token, so per request this is a dense
// [heads x tokens] GEMM (QK^T) followed by a dense [heads x latent] GEMM (PV).
//
// Design (B200):
//  * A CTA pair (cluster of 2, tcgen05 cta_group::2) owns one stream of
//    256-token tiles (four pages; CTA r holds pages 2r, 2r + 1 for QK^T).
//    MMA M = 128 heads: CTA r holds heads [64r, 64r + 64) of Q in shared
//    memory and the rows of S, P and O for those heads in its tensor memory.
//    QK^T and PV both use N = 256 (tokens / latent columns, half from each
//    CTA), the widest pair MMA: each MMA keeps the SM's tensor pipe busy for
//    64 cycles, longer than one thread needs to issue it.
//  * Tiles are staged by TMA (no multicast) into seven 16 KB slots, split
//    into a QK^T ring and a PV ring with two producer warps each.  A 4-D
//    view of the cache (column, row, 64-column chunk, page) lands [64 rows]
//    [64 bf16] chunk tiles with the 128-byte swizzle the MMA reads directly:
//    K-major for QK^T, the same bytes MN-major for PV.  A copy takes ~2 us
//    to land under load, so the ring depth (bytes in flight per SM) sets the
//    bandwidth.  The PV columns are fetched again (mostly from L2) because
//    the pair splits QK^T by tokens and PV by latent columns.
//  * TMEM per CTA: two S buffers (128 columns each) and O (256 columns).
//    Softmax warps read S with tcgen05.ld, keep a running max per shard and
//    rescale O in TMEM only when the max grows by more than 2^8 (so P stays
//    below 256 and bf16); P goes to shared memory for the PV MMA.
//  * TPLA shards are independent attention problems sharing the cache rows:
//    a (tile, shard) "unit" is one QK^T, one softmax and one PV.  S is
//    double-buffered in TMEM; P has one shared-memory buffer (the ring gets
//    the space).  Three issuing threads: QK^T of even units, QK^T of odd
//    units, PV.  Two softmax warpgroups split each unit's tokens.
//  * The issuing threads share their SM sub-partitions with softmax warps
//    and lose issue slots to them; the MMA issue code is kept short and the
//    issuers run on the lowest warp ids.
//  * Split-KV: a persistent grid of one pair per two SMs walks a balanced
//    range of the concatenated (request, tile) sequence; requests cut by a
//    range boundary leave normalised partials + lse in the workspace and
//    the merge kernel combines them with the log-sum-exp rule (the exact
//    sequence-split path of the feature request).  Explicit `num_splits`
//    cuts every request into equal chunks instead.
//  * Every wait is bounded (about 2 s); on timeout the kernel records
//    TPLA_ERR_DEVICE_TIMEOUT, stops issuing work and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace tpla {
namespace {

using namespace ptx;

constexpr int kTileTok = 256;      // tokens per tile (four pages, two per CTA)
constexpr int kChunkBytes = 8192;  // one [64 rows][64 bf16] chunk tile
constexpr int kSlotChunks = 2;     // 8 KB chunk tiles per ring slot
constexpr int kSlotBytes = kSlotChunks * kChunkBytes;
constexpr int kRingSlots = 7;      // slots shared by the QK^T ring and the PV ring
constexpr int kProducers = 4;      // two producer warps per ring
constexpr int kPBufs = 1;          // P tiles in shared memory
constexpr int kQChunks = 9;        // 576 / 64 column chunks of q
constexpr int kRopeChunk = 8;      // chunk index of the 64 rope columns
constexpr int kRoles = 3;          // MMA issuers: QK^T of even units, of odd units, PV
constexpr int kSoftmaxWarps = 8;   // two warpgroups
// Warps 0-2 issue MMAs, 3-6 produce, 7-14 run the softmax.  The issuers take
// the lowest warp ids, which the warp schedulers favour when several warps
// of a sub-partition are ready; warp w reaches TMEM lanes 32 (w % 4) + [0, 32).
constexpr int kWarpIssuer0 = 0;
constexpr int kWarpProducer0 = kWarpIssuer0 + kRoles;
constexpr int kWarpSoftmax0 = kWarpProducer0 + kProducers;
constexpr int kThreads = 32 * (kWarpSoftmax0 + kSoftmaxWarps);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // S buffers: [0, 128), [128, 256)
constexpr uint32_t kColO = 256;    // O: [256, 512)
constexpr long long kTimeoutCycles = 4000000000LL;  // about 2 s at full clock
constexpr uint32_t kWaitSleepNs = 100000;  // suspend hint of one barrier poll
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

constexpr int kOffQ = 0;
constexpr int kOffP = kOffQ + kQChunks * kChunkBytes;
constexpr int kPTileBytes = 4 * kChunkBytes;  // P: 64 heads x 256 tokens, one [64][64] tile per page
constexpr int kOffRing = kOffP + kPBufs * kPTileBytes;  // QK^T slots, then PV slots
constexpr int kOffBar = kOffRing + kRingSlots * kSlotBytes;
constexpr int kNumBars = 5 * kRingSlots + 10;
constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr int kOffAbort = kOffTmemSlot + 4;
constexpr int kOffXbuf = kOffAbort + 12;              // float [2][2][128]
constexpr int kOffLbuf = kOffXbuf + 2 * 2 * 128 * 4;  // float [2][128][4]
constexpr int kSmemUsed = kOffLbuf + 2 * 128 * 4 * 4;
constexpr int kSmemBytes = kSmemUsed + 1024;       // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffRing % 1024 == 0 && kSlotBytes % 1024 == 0, "swizzled tiles need 1 KB alignment");

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 256, false, false);
constexpr uint32_t kIdescPV256 = idesc_bf16_f32(128, 256, false, true);
constexpr uint32_t kIdescPV128 = idesc_bf16_f32(128, 128, false, true);

__device__ int g_status;

__device__ __forceinline__ void set_status(int code) { atomicCAS(&g_status, 0, code); }

struct Params {
  const int* seq_lens;  // [B], or nullptr: request b holds causal_base + b + 1 tokens
  int causal_base;      // (the query rows of a prompt, each seeing its causal prefix)
  const int* page_table;
  int64_t pt_sb;
  int num_blocks;   // paged: physical blocks (block index num_blocks reads as zeros)
  int cap_tokens;   // tokens one request's cache can hold
  int paged;
  int B, H, G, split_rope, shard, nsh, d;
  int dq;    // latent 64-column chunks per shard (d / 64)
  int NB;    // PV block width: min(256, d) latent columns per MMA
  int nblk;  // PV blocks per shard (d / NB)
  int qk_slots, pv_slots;  // ring split (sum kRingSlots)
  float scale_log2;  // |softmax scale| * log2(e) (> 0; see the launcher)
  int negate;        // scale < 0: the scores are negated before the softmax
  void* out;
  int out_bf16;
  int64_t o_sb, o_sh;
  float* lse;
  int64_t l_sb, l_sh;
  float* part_o;  // [slots, H, W]
  float* part_l;  // [slots, H, nsh]
  int W;
  int tile_tok;  // tokens per schedule tile: 256 (pair kernel) or 128 (shard kernel)
  int seg_cost;  // schedule cost of a segment's fixed work, in tiles
  int ring;      // shard kernel: ring slots
  int nS;        // shard kernel: S / P buffers in TMEM (2 or 3: 128 nS + d <= 512)
  int mode;  // 0 = balanced persistent ranges, 1 = explicit equal splits
  int P;     // clusters
  int S;     // explicit splits
};

// ---------------------------------------------------------------- schedule

__device__ __forceinline__ int req_len(const Params& p, int b) {
  int L = p.seq_lens ? p.seq_lens[b] : p.causal_base + b + 1;
  if (L < 0 || L > p.cap_tokens) {
    set_status(TPLA_ERR_DEVICE_BOUNDS);
    L = L < 0 ? 0 : p.cap_tokens;
  }
  return L;
}

__device__ __forceinline__ int req_tiles(const Params& p, int b) {
  return (req_len(p, b) + p.tile_tok - 1) / p.tile_tok;
}

// Causal lengths: sum over n = 1 .. N of ceil(n / tile_tok), in closed form.
__device__ __forceinline__ long long causal_tile_sum(const Params& p, long long N) {
  const long long tt = p.tile_tok, q = N / tt, r = N % tt;
  return tt * q * (q + 1) / 2 + r * (q + 1);
}

// Schedule cost of a request: its tiles plus seg_cost for the fixed work of
// a segment (loading q, the epilogue), so that a range of many short
// requests is not overloaded.  An empty request costs nothing.
__device__ __forceinline__ long long req_cost(const Params& p, int b) {
  const int nt = req_tiles(p, b);
  return nt > 0 ? (long long)nt + p.seg_cost : 0;
}

// Cost of requests [0, b).  Lengths from seq_lens are summed one by one;
// causal lengths (start + 1, start + 2, ...; never empty; the host keeps them
// inside the cache) in closed form.
__device__ __forceinline__ long long cost_before(const Params& p, int b) {
  if (!p.seq_lens)
    return causal_tile_sum(p, (long long)p.causal_base + b) - causal_tile_sum(p, p.causal_base) +
           (long long)p.seg_cost * b;
  long long t = 0;
  for (int i = 0; i < b; ++i) t += req_cost(p, i);
  return t;
}

struct Segment {
  int b, t_lo, t_hi, L;
  int complete;
  int slot;
};

struct Cursor {
  int b;
  long long pre, cur, end;
  int idx;
};

__device__ void seg_begin(const Params& p, int cl, Cursor& c) {
  c.idx = 0;
  if (p.mode == 0) {
    // range cl covers the cost positions [cl C / P, (cl + 1) C / P); with a
    // smaller total cost than clusters only the first C clusters get work
    const long long T = cost_before(p, p.B);
    const long long P = min((long long)p.P, T);
    if (cl >= P) {
      c.cur = c.end = 0;
    } else {
      c.cur = (long long)cl * T / P;
      c.end = (long long)(cl + 1) * T / P;
    }
    c.b = 0;
    c.pre = 0;
    if (!p.seq_lens && c.cur > 0) {
      // causal lengths: the last request starting at or before position
      // c.cur, by bisection instead of a walk over all earlier requests
      int lo = 0, hi = p.B - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (cost_before(p, mid) <= c.cur) lo = mid; else hi = mid - 1;
      }
      c.b = lo;
      c.pre = cost_before(p, lo);
    }
  } else {
    c.b = cl / p.S;
    c.pre = c.cur = c.end = 0;
  }
}

__device__ bool seg_next(const Params& p, int cl, Cursor& c, Segment& s) {
  if (p.mode == 0) {
    if (c.cur >= c.end) return false;
    while (c.b < p.B && c.pre + req_cost(p, c.b) <= c.cur) {
      c.pre += req_cost(p, c.b);
      ++c.b;
    }
    if (c.b >= p.B) return false;
    // request c.b: its fixed cost, then its tiles at positions t0, t0 + 1, ...
    const int nt = req_tiles(p, c.b);
    const long long t0 = c.pre + p.seg_cost;
    const long long lo = max(c.cur, t0), hi = min(c.end, t0 + nt);
    if (lo >= hi) {  // the range ends inside the request's fixed cost
      c.cur = c.end;
      return false;
    }
    s.b = c.b;
    s.L = req_len(p, c.b);
    s.t_lo = (int)(lo - t0);
    s.t_hi = (int)(hi - t0);
    s.complete = (s.t_lo == 0 && s.t_hi == nt);
    // a range's first segment writes partials to slot 2 cl, the others
    // (only its last can be partial) to 2 cl + 1
    s.slot = 2 * cl + (c.idx == 0 ? 0 : 1);
    c.cur = hi;
    ++c.idx;
    return true;
  }
  if (c.idx > 0) return false;
  const int b = cl / p.S, sp = cl % p.S;
  const int nt = req_tiles(p, b);
  const int chunk = (nt + p.S - 1) / p.S;
  s.b = b;
  s.L = req_len(p, b);
  s.t_lo = min(nt, sp * chunk);
  s.t_hi = min(nt, (sp + 1) * chunk);
  s.complete = p.S == 1;
  s.slot = 2 * cl;
  ++c.idx;
  return true;
}

// Columns of shard g: latent 64-column chunks [g d/64, (g+1) d/64) and the
// rope chunk (index 8).  K-steps (16 columns) of the rope chunk this shard
// uses: all four (replicate) or its own slice (split).
__device__ __forceinline__ int shard_of(const Params& p, int i) { return p.shard < 0 ? i : p.shard; }

__device__ __forceinline__ void rope_steps(const Params& p, int g, int& k0, int& k1) {
  if (!p.split_rope) {
    k0 = 0;
    k1 = 4;
  } else {
    const int per = 4 / p.G;  // 16-column steps per shard (G <= 4)
    k0 = g * per;
    k1 = k0 + per;
  }
}

// Stage plan of one unit (tile t, shard g), shared by producers and issuers
// so that both walk the same stage sequence.  A tile is four pages; CTA r
// holds pages 2r and 2r + 1 for QK^T.
//  QK^T: one stage per item (the shard's latent chunks g*dq .. g*dq + dq - 1,
//        then the rope chunk): chunk c of this CTA's two pages, the second
//        page's [64][64] tile right after the first, so that one descriptor
//        with an 8-row stride covers the CTA's 128 tokens.
//  PV:   items (block j, page pg), j-major over pages 0..3 of the tile.  An
//        item is this CTA's half of latent block j (NB/128 chunks) for the
//        64 tokens of page pg; one item per stage when NB = 256, two pages
//        per stage when NB = 128.
__device__ __forceinline__ int qk_nstages(const Params& p) { return p.dq + 1; }
__device__ __forceinline__ int qk_item_chunk(const Params& p, int g, int item) {
  return item < p.dq ? g * p.dq + item : kRopeChunk;
}
__device__ __forceinline__ int pv_items_per_stage(const Params& p) { return p.NB == 256 ? 1 : 2; }
__device__ __forceinline__ int pv_nstages(const Params& p) {
  return 4 * p.nblk / pv_items_per_stage(p);
}
// first chunk of CTA `rank`'s half of latent block j of shard g
__device__ __forceinline__ int pv_chunk(const Params& p, int g, int j, uint32_t rank) {
  return g * p.dq + j * (p.NB / 64) + (int)rank * (p.NB / 128);
}

// ---------------------------------------------------------------- waits

// Bounded wait.  The bound uses the SM cycle counter: reading %globaltimer
// costs about half a microsecond, which would throttle every pipeline
// hand-off that has to wait.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         long long limit = kTimeoutCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
    if ((i & 15) == 0) {
      if (*abort_flag) return false;
      if (clock64() - t0 > limit) {
        set_status(TPLA_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Warp-uniform variant: lane 0 polls, the result is broadcast.
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity,
                                              volatile int* abort_flag) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, abort_flag);
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Ring "full" barriers exist per (slot, consuming issuer).  A barrier phase
// wait only tells phases apart by parity, so a waiter must never be two
// phases away from the barrier; one shared full barrier per slot breaks that
// when an issuer skips the other issuers' stages and runs ahead.  With one
// full barrier per (slot, issuer) every barrier has a single consumer that
// takes its phases strictly in order.
struct Bars {
  static constexpr int kX = 5 * kRingSlots;
  uint32_t base;
  // QK^T ring: one full barrier per (slot, QK issuer), see above
  __device__ uint32_t qk_full(int s, int role) const { return base + 8 * (role * kRingSlots + s); }
  __device__ uint32_t qk_empty(int s) const { return base + 8 * (2 * kRingSlots + s); }
  __device__ uint32_t pv_full(int s) const { return base + 8 * (3 * kRingSlots + s); }
  __device__ uint32_t pv_empty(int s) const { return base + 8 * (4 * kRingSlots + s); }
  __device__ uint32_t q_full() const { return base + 8 * kX; }
  __device__ uint32_t q_empty() const { return base + 8 * (kX + 1); }
  __device__ uint32_t s_full(int i) const { return base + 8 * (kX + 2 + i); }
  __device__ uint32_t p_full(int i) const { return base + 8 * (kX + 4 + i); }
  __device__ uint32_t p_empty(int i) const { return base + 8 * (kX + 6 + i); }
  __device__ uint32_t s_free(int i) const { return base + 8 * (kX + 8 + i); }
};

// ---------------------------------------------------------------- producer

// Physical block ids of one request, 32 pages per window.  Each lane of the
// producer warp holds one entry of three consecutive windows (prev, cur,
// next): stages of the previous tile still hit after the window advanced,
// and advancing issues the load of the window after next, which is not read
// until the producer gets there 32 pages later.  So TMA issue never waits
// on a page-table load except at the start of a request.
struct PageWindow {
  int b = -1, base = 0;
  int prev = 0, cur = 0, next = 0;

  __device__ static int raw(const Params& p, const Segment& s, int pg, int npages) {
    return (pg >= 0 && pg < npages) ? p.page_table[(int64_t)s.b * p.pt_sb + pg] : p.num_blocks;
  }

  __device__ int get(const Params& p, const Segment& s, int page, int lane) {
    const int npages = (s.L + 63) / 64;
    if (page >= npages) return p.num_blocks;  // beyond the request: reads as zeros
    const int wb = page & ~31;
    if (s.b != b || wb < base - 32 || wb > base + 32) {
      b = s.b;
      base = wb;
      prev = raw(p, s, base - 32 + lane, npages);
      cur = raw(p, s, base + lane, npages);
      next = raw(p, s, base + 32 + lane, npages);
    } else if (wb == base + 32) {
      prev = cur;
      cur = next;
      base = wb;
      next = raw(p, s, base + 32 + lane, npages);
    }
    // wb is now base or base - 32; `next` is not touched, so its load stays in flight
    int blk = __shfl_sync(0xffffffffu, wb == base ? cur : prev, page & 31);
    if (blk < 0 || blk >= p.num_blocks) {
      set_status(TPLA_ERR_DEVICE_BOUNDS);
      blk = p.num_blocks;
    }
    return blk;
  }
};

// Runs on all 32 lanes of the producer warp (uniform control flow); lane 0
// issues the barrier arrivals and TMA copies.
//
// Two rings: QK^T stages and PV stages, each of kRingSlots slots with two
// producer warps (slot s of a ring is filled by that ring's warp s % 2, which
// therefore takes the phases of its slots' empty barriers in order).  With
// separate rings, PV stages waiting for their softmax never hold up the
// loads of later QK^T stages.
__device__ void producer(const Params& p, const CUtensorMap* qmap, const CUtensorMap* kv1,
                         const CUtensorMap* kv2, int cl, int pid, uint32_t rank, uint32_t sbase,
                         const Bars& bars, volatile int* abort_flag) {
  const int lane = threadIdx.x & 31;
  const bool leader_lane = lane == 0;
  const bool qk_ring = pid < 2;
  const uint32_t rpid = (uint32_t)(pid & 1);
  Cursor cur;
  seg_begin(p, cl, cur);
  Segment s;
  PageWindow win;
  uint32_t n = 0, qloads = 0, U0 = 0;
  const uint32_t q_full_c = mapa(bars.q_full(), 0);
  const int nq = qk_nstages(p), np = pv_nstages(p), ipst = pv_items_per_stage(p);
  const int pv_k = p.NB / 128;  // chunks per PV item
  const uint32_t nslots = (uint32_t)(qk_ring ? p.qk_slots : p.pv_slots);
  const uint32_t ring_base = sbase + kOffRing + (qk_ring ? 0u : (uint32_t)p.qk_slots * kSlotBytes);

  // Claims stage n of this warp's ring.  Returns 1 when this warp loads it
  // (slot free, the leader CTA's full barrier of consumer `owner` armed for
  // `bytes` per CTA), 0 when the ring's other producer does, -1 on abort.
  // Warp-uniform.
  auto next_slot = [&](uint32_t& slot, uint32_t& full_c, int owner, uint32_t bytes) -> int {
    const uint32_t me = n++;
    slot = me % nslots;
    if ((slot & 1u) != rpid) return 0;
    if (me >= nslots) {
      const uint32_t eb = qk_ring ? bars.qk_empty(slot) : bars.pv_empty(slot);
      if (!wait_bar_warp(eb, ((me / nslots) - 1) & 1, abort_flag)) return -1;
    }
    const uint32_t fb = qk_ring ? bars.qk_full(slot, owner) : bars.pv_full(slot);
    full_c = mapa(fb, 0);
    if (rank == 0 && leader_lane) mbar_arrive_expect_tx(fb, 2 * bytes);
    return 1;
  };
  // k consecutive chunk tiles from `chunk` of page pg (0..3) of tile t
  auto load = [&](uint32_t dst, uint32_t full_c, int chunk, int k, int t, int pg) {
    const CUtensorMap* map = k == 1 ? kv1 : kv2;
    if (p.paged) {
      const int blk = win.get(p, s, 4 * t + pg, lane);
      if (leader_lane) tma_load_4d_pair(dst, map, 0, 0, chunk, blk, full_c);
    } else if (leader_lane) {
      tma_load_4d_pair(dst, map, 0, kTileTok * t + 64 * pg, chunk, s.b, full_c);
    }
  };

  while (seg_next(p, cl, cur, s)) {
    const int nunits = (s.t_hi - s.t_lo) * p.nsh;
    if (nunits == 0) continue;
    if (pid == 0) {  // q of this segment, once its previous user is done
      if (qloads > 0 && !wait_bar_warp(bars.q_empty(), (qloads - 1) & 1, abort_flag)) return;
      const int nqc = p.shard < 0 ? kQChunks : p.dq + 1;
      if (leader_lane) {
        if (rank == 0) mbar_arrive_expect_tx(bars.q_full(), 2 * nqc * kChunkBytes);
        for (int i = 0; i < nqc; ++i) {
          const int c = p.shard < 0 ? i : qk_item_chunk(p, p.shard, i);
          tma_load_3d_pair(sbase + kOffQ + c * kChunkBytes, qmap, 64 * c, 64 * (int)rank, s.b,
                           q_full_c);
        }
      }
    }
    ++qloads;
    for (int j = 0; j < nunits; ++j) {
      const int t = s.t_lo + j / p.nsh;
      const int g = shard_of(p, j % p.nsh);
      if (qk_ring) {  // QK^T stages of unit j: this CTA's page, shard columns + rope
        const int owner = (int)((U0 + j) & 1);
        for (int st = 0; st < nq; ++st) {
          uint32_t slot, full_c;
          const int r = next_slot(slot, full_c, owner, 2 * kChunkBytes);
          if (r < 0) return;
          if (r == 0) continue;
          const uint32_t base = ring_base + slot * kSlotBytes;
          const int c = qk_item_chunk(p, g, st);
          load(base, full_c, c, 1, t, 2 * (int)rank);
          load(base + kChunkBytes, full_c, c, 1, t, 2 * (int)rank + 1);
        }
      } else {  // PV stages of unit j: both pages, this CTA's latent half
        for (int st = 0; st < np; ++st) {
          uint32_t slot, full_c;
          const int r = next_slot(slot, full_c, 0, (uint32_t)(ipst * pv_k) * kChunkBytes);
          if (r < 0) return;
          if (r == 0) continue;
          const uint32_t base = ring_base + slot * kSlotBytes;
          for (int i = 0; i < ipst; ++i) {
            const int it = st * ipst + i;
            load(base + i * pv_k * kChunkBytes, full_c, pv_chunk(p, g, it >> 2, rank), pv_k, t,
                 it & 3);
          }
        }
      }
    }
    U0 += nunits;
  }
}

// ---------------------------------------------------------------- MMA issuers
//
// One thread can issue a tcgen05.mma about every 55 cycles, while a
// 128 x 128 x 16 pair MMA (QK^T) keeps the tensor pipe busy for only 32
// cycles per SM; a 128 x 256 x 16 one (PV) for 64.  So three threads of the
// leader CTA issue MMAs into independent accumulators: role 0/1 = QK^T of
// even/odd units (S buffer Ug & 1), role 2 = PV.  Every issuer walks the
// producers' stage sequence and consumes (waits for, multiplies, releases)
// only its own ring stages; a commit tracks only the issuing thread's MMAs,
// so each issuer releases its own slots and signals its own barriers.

__device__ void mma_issuer(const Params& p, int cl, int role, uint32_t sbase, uint32_t tmem,
                           const Bars& bars, volatile int* abort_flag) {
  Cursor cur;
  seg_begin(p, cl, cur);
  Segment s;
  uint32_t n = 0, qloads = 0, U0 = 0;
  const bool qk = role < 2;
  const int nq = qk_nstages(p), np = pv_nstages(p), ipst = pv_items_per_stage(p);
  const int g0 = p.shard < 0 ? 0 : p.shard;
  const uint32_t idesc_pv = p.NB == 256 ? kIdescPV256 : kIdescPV128;
  const uint32_t pv_item_desc = (uint32_t)((p.NB / 128) * kChunkBytes) >> 4;
  // Descriptor templates; an operand at byte offset `o` from a region start
  // is template + (o >> 4) (shared memory is below 256 KB, so the 14-bit
  // start-address field never overflows).
  const uint64_t dQ = sw128_desc(sbase + kOffQ, 16, 1024);               // K-major q
  const uint32_t nslots = (uint32_t)(qk ? p.qk_slots : p.pv_slots);
  const uint32_t off_pv = kOffRing + (uint32_t)p.qk_slots * kSlotBytes;
  const uint64_t dRk = sw128_desc(sbase + kOffRing, 16, 1024);        // K-major QK^T ring
  const uint64_t dRm = sw128_desc(sbase + off_pv, kChunkBytes, 1024);  // MN-major PV ring
  const uint64_t dP = sw128_desc(sbase + kOffP, 16, 1024);               // K-major P
  constexpr uint32_t kChunkDesc = kChunkBytes >> 4;
  constexpr uint32_t kSlotDesc = kSlotBytes >> 4;
  // 32-bit halves: adding an in-range offset to the low half never carries
  const uint32_t q_lo = (uint32_t)dQ, q_hi = (uint32_t)(dQ >> 32);
  const uint32_t rk_lo = (uint32_t)dRk, rk_hi = (uint32_t)(dRk >> 32);
  const uint32_t rm_lo = (uint32_t)dRm, rm_hi = (uint32_t)(dRm >> 32);
  const uint32_t p_lo = (uint32_t)dP, p_hi = (uint32_t)(dP >> 32);

  // A ring slot is filled by TMA, whose completion the barrier itself orders
  // before the MMA's shared-memory reads: no tcgen05 fence is needed here.
  // full_parity bit s = parity of this issuer's next phase on slot s
  uint32_t full_parity = 0;
  auto take = [&](uint32_t slot) -> bool {
    const uint32_t fb = qk ? bars.qk_full(slot, role) : bars.pv_full(slot);
    const bool ok = wait_bar(fb, (full_parity >> slot) & 1u, abort_flag);
    full_parity ^= 1u << slot;
    return ok;
  };

  while (seg_next(p, cl, cur, s)) {
    const int nunits = (s.t_hi - s.t_lo) * p.nsh;
    if (nunits == 0) continue;
    if (qk) {
      if (!wait_bar(bars.q_full(), qloads & 1, abort_flag)) return;
      tc_fence_after();
    }
    ++qloads;
    for (int j = 0; j <= nunits; ++j) {
      if (j < nunits) {  // QK^T(j)
        const uint32_t Ug = U0 + j;
        if (qk && (Ug & 1) == (uint32_t)role) {
          const int g = shard_of(p, j % p.nsh);
          // S[Ug & 1] is free once the softmax of unit Ug - 2 has read it
          if (Ug >= 2 && !wait_bar(bars.s_free(Ug & 1), ((Ug - 2) >> 1) & 1, abort_flag)) return;
          tc_fence_after();
          const uint32_t dS = tmem + kColS + 128 * (Ug & 1);
          int rk0, rk1;
          rope_steps(p, g, rk0, rk1);
          uint32_t acc = 0;
          for (int st = 0; st < nq; ++st) {
            const uint32_t slot = (n + st) % nslots;
            if (!take(slot)) return;
            {
              const int i = st;
              const uint32_t a = q_lo + (uint32_t)qk_item_chunk(p, g, i) * kChunkDesc;
              const uint32_t b = rk_lo + slot * kSlotDesc;
              if (i < p.dq) {  // latent chunk: four K-steps of 16 columns
                mma_pair_f16_lh(dS, a, q_hi, b, rk_hi, kIdescQK, acc);
                mma_pair_f16_lh(dS, a + 2, q_hi, b + 2, rk_hi, kIdescQK, 1u);
                mma_pair_f16_lh(dS, a + 4, q_hi, b + 4, rk_hi, kIdescQK, 1u);
                mma_pair_f16_lh(dS, a + 6, q_hi, b + 6, rk_hi, kIdescQK, 1u);
                acc = 1;
              } else {  // rope chunk: this shard's K-steps
                for (int kk = rk0; kk < rk1; ++kk) {
                  mma_pair_f16_lh(dS, a + 2 * kk, q_hi, b + 2 * kk, rk_hi, kIdescQK, acc);
                  acc = 1;
                }
              }
            }
            mma_commit_pair(bars.qk_empty(slot), 0x3);
          }
          mma_commit_pair(bars.s_full(Ug & 1), 0x3);
        }
        if (qk) n += nq;
      }
      if (j >= 1) {  // PV(j - 1)
        const int k = j - 1;
        const uint32_t Ug = U0 + k;
        if (!qk) {
          const int g = shard_of(p, k % p.nsh);
          const uint32_t first = k < p.nsh ? 1u : 0u;  // first tile of this shard here
          if (!wait_bar(bars.p_full(Ug % kPBufs), (Ug / kPBufs) & 1, abort_flag)) return;
          tc_fence_after();
          const uint32_t pa = p_lo + (Ug % kPBufs) * (kPTileBytes >> 4);
          for (int st = 0; st < np; ++st) {
            const uint32_t slot = (n + st) % nslots;
            if (!take(slot)) return;
            for (int i = 0; i < ipst; ++i) {
              const int it = st * ipst + i;
              const int jb = it >> 2, pg = it & 3;
              const uint32_t dO = tmem + kColO + ((g - g0) * p.nblk + jb) * (p.NB / 2);
              const uint32_t a = pa + (uint32_t)pg * kChunkDesc;
              const uint32_t b = rm_lo + slot * kSlotDesc + (uint32_t)i * pv_item_desc;
              const uint32_t acc0 = pg == 0 ? (first ^ 1u) : 1u;
              mma_pair_f16_lh(dO, a, p_hi, b, rm_hi, idesc_pv, acc0);
              mma_pair_f16_lh(dO, a + 2, p_hi, b + 128, rm_hi, idesc_pv, 1u);
              mma_pair_f16_lh(dO, a + 4, p_hi, b + 256, rm_hi, idesc_pv, 1u);
              mma_pair_f16_lh(dO, a + 6, p_hi, b + 384, rm_hi, idesc_pv, 1u);
            }
            mma_commit_pair(bars.pv_empty(slot), 0x3);
          }
          // P[Ug % kPBufs] free and O up to date
          mma_commit_pair(bars.p_empty(Ug % kPBufs), 0x3);
        }
        if (!qk) n += np;
      }
    }
    // both QK roles arrive on q_empty (count 2) once their QKs of this
    // segment have completed
    if (qk) mma_commit_pair(bars.q_empty(), 0x3);
    U0 += nunits;
  }
}

// ---------------------------------------------------------------- softmax + epilogue

// Four per-shard floats kept in registers: a runtime index into a local
// array would put it in (slow) local memory.
struct Reg4 {
  float v0, v1, v2, v3;
  __device__ explicit Reg4(float x) : v0(x), v1(x), v2(x), v3(x) {}
  __device__ float get(int i) const { return i == 0 ? v0 : (i == 1 ? v1 : (i == 2 ? v2 : v3)); }
  __device__ void set(int i, float x) {
    v0 = i == 0 ? x : v0;
    v1 = i == 1 ? x : v1;
    v2 = i == 2 ? x : v2;
    v3 = i == 3 ? x : v3;
  }
};

// Packed two-lane float arithmetic (sm_100): one instruction for two
// values halves the softmax's issue slots for these steps, and those issue
// slots are shared with the MMA-issuing threads of the same sub-partition.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// (lo, hi) rounded to a bf16 pair, lo in the low half
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void write_out_row(const Params& p, const Segment& s, int head,
                                              int col0, const float* v, float inv) {
  if (head >= p.H) return;
  if (s.complete) {
    const int64_t off = (int64_t)s.b * p.o_sb + (int64_t)head * p.o_sh + col0;
    if (p.out_bf16) {
      __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + off;
#pragma unroll
      for (int j = 0; j < 32; j += 8) {
        uint4 w;
        __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) h2[e] = __floats2bfloat162_rn(v[j + 2 * e] * inv, v[j + 2 * e + 1] * inv);
        *reinterpret_cast<uint4*>(o + j) = w;
      }
    } else {
      float* o = reinterpret_cast<float*>(p.out) + off;
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4*>(o + j) =
            make_float4(v[j] * inv, v[j + 1] * inv, v[j + 2] * inv, v[j + 3] * inv);
    }
  } else {
    float* o = p.part_o + ((int64_t)s.slot * p.H + head) * p.W + col0;
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      *reinterpret_cast<float4*>(o + j) =
          make_float4(v[j] * inv, v[j + 1] * inv, v[j + 2] * inv, v[j + 3] * inv);
  }
}

__device__ __forceinline__ void write_lse(const Params& p, const Segment& s, int head, int i,
                                          float v) {
  if (head >= p.H) return;
  if (s.complete) {
    if (p.lse) p.lse[(int64_t)s.b * p.l_sb + (int64_t)head * p.l_sh + i] = v;
  } else {
    p.part_l[((int64_t)s.slot * p.H + head) * p.nsh + i] = v;
  }
}

// Two warpgroups share each unit: thread (wg, lane) holds TMEM lane `lane`
// (head 64*rank + lane % 64, token half lane / 64) and tokens
// [32 wg, 32 wg + 32) of that half.  Both warpgroups keep the same running
// max (they exchange partial maxima every unit) and each its partial sum;
// they split the O columns for rescaling and the epilogue.
__device__ void softmax_warps(const Params& p, int cl, uint32_t rank, uint32_t sbase,
                              uint8_t* smem, uint32_t tmem, const Bars& bars,
                              volatile int* abort_flag) {
  // tid = 128 * warpgroup + TMEM lane (a warp's lanes are fixed by warp % 4)
  const int w = (int)(threadIdx.x >> 5);
  const int tid = ((w - kWarpSoftmax0) >> 2) * 128 + 32 * (w & 3) + (int)(threadIdx.x & 31);
  const int wg = tid >> 7, lt = tid & 127;
  const int half = lt >> 6, hl = lt & 63;
  const int head = 64 * (int)rank + hl;
  const uint32_t lane_base = (uint32_t)(32 * ((tid >> 5) & 3)) << 16;
  float* xbuf = reinterpret_cast<float*>(smem + kOffXbuf);  // [2 buffers][2 wg][128]
  float* lbuf = reinterpret_cast<float*>(smem + kOffLbuf);  // [2 wg][128][4]
  const uint32_t pf_c[2] = {mapa(bars.p_full(0), 0), mapa(bars.p_full(1), 0)};
  const uint32_t sf_c[2] = {mapa(bars.s_free(0), 0), mapa(bars.s_free(1), 0)};
  // O of shard g, block jb: TMEM columns o_col(g, jb) + [0, NB/2); lanes
  // 0-63 hold latent columns jb*NB + [0, NB/2) of the shard, lanes 64-127
  // the next NB/2 (the pair MMA's accumulator layout for M = 128).  Pieces
  // of 32 columns alternate between the warpgroups.
  const int g0 = p.shard < 0 ? 0 : p.shard;
  const int npiece = p.NB / 64;  // 32-column pieces per lane and block
  auto o_col = [&](int g, int jb) -> uint32_t {
    return kColO + (uint32_t)(((g - g0) * p.nblk + jb) * (p.NB / 2));
  };
  auto out_col = [&](int g, int jb) -> int {
    return (p.shard < 0 ? g * p.d : 0) + jb * p.NB + half * (p.NB / 2);
  };

  Cursor cur;
  seg_begin(p, cl, cur);
  Segment s;
  uint32_t U = 0;
  while (seg_next(p, cl, cur, s)) {
    const int nunits = (s.t_hi - s.t_lo) * p.nsh;
    if (nunits == 0) {  // empty chunk: out 0, lse -inf
      float z[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) z[j] = 0.f;
      for (int i = 0; i < p.nsh; ++i) {
        const int g = shard_of(p, i);
        for (int pc = wg; pc < p.nblk * npiece; pc += 2)
          write_out_row(p, s, head, out_col(g, pc / npiece) + 32 * (pc % npiece), z, 0.f);
        if (half == 0 && wg == 0) write_lse(p, s, head, i, -INFINITY);
      }
      continue;
    }
    Reg4 m(-INFINITY), l(0.f);
    for (int k = 0; k < nunits; ++k) {
      const uint32_t Ug = U + k;
      const int i = k % p.nsh;
      const int g = shard_of(p, i);
      const int t = s.t_lo + k / p.nsh;
      if (!wait_bar(bars.s_full(Ug & 1), (Ug >> 1) & 1, abort_flag)) return;
      tc_fence_after();
      // this thread's 64 tokens: page 2 * half + wg of the tile
      uint32_t r0[32], r1[32];
      tmem_ld32(tmem + lane_base + kColS + 128 * (Ug & 1) + 64 * wg, r0);
      tmem_ld32(tmem + lane_base + kColS + 128 * (Ug & 1) + 64 * wg + 32, r1);
      tmem_wait_ld();
      // S[Ug & 1] is in registers: let QK^T of unit Ug + 2 overwrite it
      tc_fence_before();
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive_remote(sf_c[Ug & 1]);
      // raw scores; |scale| is applied inside the exponent, a negative
      // scale's sign here (uniform branch, not taken for the usual scale > 0)
      const int nv = max(0, min(64, s.L - (kTileTok * t + 128 * half + 64 * wg)));
      float x[64];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        x[j] = __uint_as_float(r0[j]);
        x[j + 32] = __uint_as_float(r1[j]);
      }
      if (p.negate) {
#pragma unroll
        for (int j = 0; j < 64; ++j) x[j] = -x[j];
      }
      if (nv < 64) {  // warp-uniform: a warp covers one 64-token range
#pragma unroll
        for (int j = 0; j < 64; ++j) x[j] = j < nv ? x[j] : -INFINITY;
      }
      float mx0 = fmaxf(x[0], x[1]), mx1 = fmaxf(x[2], x[3]);
#pragma unroll
      for (int j = 4; j < 64; j += 4) {
        mx0 = fmaxf(mx0, fmaxf(x[j], x[j + 1]));
        mx1 = fmaxf(mx1, fmaxf(x[j + 2], x[j + 3]));
      }
      float mx = fmaxf(mx0, mx1) * p.scale_log2;
      float* xb = xbuf + (Ug & 1) * 256;
      xb[wg * 128 + lt] = mx;
      named_bar_sync(1, 256);
      mx = fmaxf(fmaxf(xb[lt], xb[128 + lt]), fmaxf(xb[lt ^ 64], xb[128 + (lt ^ 64)]));
      float mi = m.get(i);
      float factor = 1.f;
      int resc = 0;
      if (mi == -INFINITY) {
        mi = mx;
      } else if (mx > mi + kRescaleThreshold) {
        factor = ex2(mi - mx);
        mi = mx;
        resc = 1;
      }
      m.set(i, mi);
      l.set(i, l.get(i) * factor);
      if (__any_sync(0xffffffffu, resc)) {
        // O of this shard was last written by an earlier PV: wait for all
        // issued PVs (up to unit Ug - 1), then rescale this warpgroup's pieces
        if (!wait_bar(bars.p_empty((Ug - 1) % kPBufs), ((Ug - 1) / kPBufs) & 1, abort_flag)) return;
        tc_fence_after();
        for (int pc = wg; pc < p.nblk * npiece; pc += 2) {
          const uint32_t ta = tmem + lane_base + o_col(g, pc / npiece) + 32 * (pc % npiece);
          uint32_t o[32];
          tmem_ld32(ta, o);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * factor);
          tmem_st32(ta, o);
        }
        tmem_wait_st();
      }
      // P = 2^(x - m) in bf16 (masked tokens give 0); l sums the rounded values
      uint32_t pk[32];
      const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nm2 = f2_pack(-mi, -mi);
      uint64_t ls2 = f2_pack(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float e0, e1;
        f2_unpack(f2_fma(f2_pack(x[2 * j], x[2 * j + 1]), sc2, nm2), e0, e1);
        const uint32_t u = cvt_bf16x2(ex2(e0), ex2(e1));
        ls2 = f2_add(ls2, f2_pack(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u)));
        pk[j] = u;
      }
      float ls0, ls1;
      f2_unpack(ls2, ls0, ls1);
      l.set(i, l.get(i) + (ls0 + ls1));
      if (Ug >= (uint32_t)kPBufs) {  // P[Ug % kPBufs] was read by PV of unit Ug - kPBufs
        if (!wait_bar(bars.p_empty(Ug % kPBufs), ((Ug - kPBufs) / kPBufs) & 1, abort_flag)) return;
      }
      // P tile of page 2 * half + wg: row hl, all eight 16-byte chunks, swizzled
      const uint32_t prow = sbase + kOffP + (Ug % kPBufs) * kPTileBytes +
                            (2 * half + wg) * kChunkBytes + hl * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        st_shared_v4(prow + ((c ^ (hl & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                     pk[4 * c + 3]);
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive_remote(pf_c[Ug % kPBufs]);
    }
    U += nunits;
    // epilogue: all PVs of the segment done
    if (!wait_bar(bars.p_empty((U - 1) % kPBufs), ((U - 1) / kPBufs) & 1, abort_flag)) return;
    tc_fence_after();
    for (int i = 0; i < p.nsh; ++i) lbuf[(wg * 128 + lt) * 4 + i] = l.get(i);
    named_bar_sync(1, 256);
    for (int i = 0; i < p.nsh; ++i) {
      const int g = shard_of(p, i);
      const float lt_sum = (lbuf[lt * 4 + i] + lbuf[(128 + lt) * 4 + i]) +
                           (lbuf[(lt ^ 64) * 4 + i] + lbuf[(128 + (lt ^ 64)) * 4 + i]);
      const float inv = lt_sum > 0.f ? 1.f / lt_sum : 0.f;
      const float lse = lt_sum > 0.f ? (m.get(i) + log2f(lt_sum)) * kLn2 : -INFINITY;
      for (int pc = wg; pc < p.nblk * npiece; pc += 2) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + o_col(g, pc / npiece) + 32 * (pc % npiece), o);
        tmem_wait_ld();
        write_out_row(p, s, head, out_col(g, pc / npiece) + 32 * (pc % npiece),
                      reinterpret_cast<const float*>(o), inv);
      }
      if (half == 0 && wg == 0) write_lse(p, s, head, i, lse);
    }
    tc_fence_before();
    named_bar_sync(1, 256);
  }
}

// ---------------------------------------------------------------- kernel

__global__ void __launch_bounds__(kThreads, 1)
tpla_decode_sm100_kernel(const __grid_constant__ CUtensorMap qmap,
                         const __grid_constant__ CUtensorMap kv1,
                         const __grid_constant__ CUtensorMap kv2, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cl = (int)cluster_id_x();
  Bars bars{sbase + kOffBar};
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRingSlots; ++s) {
      mbar_init(bars.qk_full(s, 0), 1);
      mbar_init(bars.qk_full(s, 1), 1);
      mbar_init(bars.qk_empty(s), 1);
      mbar_init(bars.pv_full(s), 1);
      mbar_init(bars.pv_empty(s), 1);
    }
    mbar_init(bars.q_full(), 1);
    mbar_init(bars.q_empty(), 2);   // the two QK issuers
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars.s_full(i), 1);
      mbar_init(bars.p_full(i), 2 * kSoftmaxWarps);  // softmax warps of both CTAs
      mbar_init(bars.p_empty(i), 1);  // the PV issuer
      mbar_init(bars.s_free(i), 2 * kSoftmaxWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpProducer0 && lane == 0) {
    tma_prefetch(&qmap);
    tma_prefetch(&kv1);
    tma_prefetch(&kv2);
  }
  if (warp == kWarpIssuer0) {
    tmem_alloc_pair(sbase + kOffTmemSlot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmemSlot);

  if (warp < kWarpProducer0) {
    if (lane == 0 && rank == 0)
      mma_issuer(p, cl, warp - kWarpIssuer0, sbase, tmem, bars, abort_flag);
  } else if (warp < kWarpSoftmax0) {
    producer(p, &qmap, &kv1, &kv2, cl, warp - kWarpProducer0, rank, sbase, bars, abort_flag);
  } else {
    softmax_warps(p, cl, rank, sbase, smem, tmem, bars, abort_flag);
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (warp == kWarpIssuer0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ================================================================ shard kernel (G >= 2)
//
// One CTA computes one TPLA shard, as one tensor-parallel rank would: all
// 128 heads of the request in one single-CTA MMA (M = 128), over the shard's
// latent columns and its rope columns.  The CTAs of a token range (one per
// shard) are launched next to each other and run together, so the rope chunk
// they share is read from DRAM once and from L2 by the others.  Unlike the
// pair kernel, every cache byte is staged into shared memory once: the tile's
// latent chunks stay in the ring from QK^T through P.V (the P.V operand is
// MN-major over the same bytes), and P lives in tensor memory over the S it
// came from, so the ring gets the shared memory the pair kernel spends on P
// and on re-reading the peer's tokens.
//  * Tiles of 128 tokens (two pages).  A stage is chunk c of both pages:
//    [64 rows][64 bf16] x 2, 16 KB, in the 128-byte swizzle.  Per tile the
//    rope chunk first (its slot is free again as soon as QK^T has read it),
//    then the shard's d/64 latent chunks.  With 9 slots at G = 2 (5 stages
//    per tile) the loads of tile i then wait only for P.V of tile i - 2 and
//    QK^T of tile i - 1: two tiles in flight.
//  * QK^T: M = 128 heads, N = 128 tokens, K-steps over the stage; S in TMEM
//    (two buffers of 128 columns).  P.V: M = 128, N = 64 latent columns per
//    chunk, K = 128 tokens, A = P read from TMEM; O (d <= 256 columns) in
//    TMEM.  The rope slot is released after QK^T, latent slots after P.V.
//  * Warps: 0 QK^T issuer (and TMEM allocation), 1 P.V issuer, 2-3 TMA
//    producers, 4-7 softmax: one thread per head (its TMEM lane) over all
//    128 tokens of a tile, so the row max needs no exchange between threads
//    and P overwrites only the thread's own lane of S.
namespace shd {

constexpr int kTile = 128;
constexpr int kStage = 16384;
constexpr int kQChunkBytes = 16384;  // [128 heads][64 columns] bf16
constexpr int kMaxRing = 12;
constexpr int kWarpQK = 0, kWarpPV = 1, kWarpProd0 = 2, kWarpSm0 = 4;  // producers: warps 2, 3
constexpr int kSoftmaxWarps = 4;
constexpr int kThreads = 32 * (kWarpSm0 + kSoftmaxWarps);
constexpr uint32_t kColS = 0;    // S / P buffers: 128 columns each, nS of them
constexpr int kMaxS = 3;         // O (d columns) follows them: 128 nS + d <= 512
constexpr int kNumBars = 2 * kMaxRing + 2 + 3 * kMaxS;
constexpr int kMiscBytes = kNumBars * 8 + 16;
constexpr int kSmemBytes = 232448;  // the per-block maximum; the ring takes what Q leaves

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false, false);
__constant__ uint32_t kIdescPVn[2] = {idesc_bf16_f32(128, 64, false, true),
                                      idesc_bf16_f32(128, 128, false, true)};

struct Bars {
  uint32_t base;
  __device__ uint32_t full(int s) const { return base + 8 * s; }
  __device__ uint32_t empty(int s) const { return base + 8 * (kMaxRing + s); }
  __device__ uint32_t q_full() const { return base + 8 * (2 * kMaxRing); }
  __device__ uint32_t q_empty() const { return base + 8 * (2 * kMaxRing + 1); }
  __device__ uint32_t s_full(int i) const { return base + 8 * (2 * kMaxRing + 2 + i); }
  __device__ uint32_t p_full(int i) const { return base + 8 * (2 * kMaxRing + 2 + kMaxS + i); }
  __device__ uint32_t pv_done(int i) const {
    return base + 8 * (2 * kMaxRing + 2 + 2 * kMaxS + i);
  }
};

struct Layout {  // shared-memory offsets (bytes from the 1 KB aligned base)
  uint32_t ring, bars, tmem_slot, abort;
};

// q chunks (rope first, then the shard's latent chunks), ring, barriers
__device__ __forceinline__ Layout layout(const Params& p) {
  Layout L;
  L.ring = (uint32_t)(p.dq + 1) * kQChunkBytes;
  L.bars = L.ring + (uint32_t)p.ring * kStage;
  L.tmem_slot = L.bars + kNumBars * 8;
  L.abort = L.tmem_slot + 4;
  return L;
}

// cache / q chunk of stage `st` of a tile: the rope chunk, then the latent
__device__ __forceinline__ int stage_chunk(const Params& p, int g, int st) {
  return st == 0 ? kRopeChunk : g * p.dq + st - 1;
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];"
      :
      : "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2),
        "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      :
      : "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// D[tmem] (+)= A[smem] B[smem]^T (single CTA), descriptors as 32-bit halves
__device__ __forceinline__ void mma_ss(uint32_t d, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo,
                                       uint32_t b_hi, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "mov.b64 da, {%1, %2};\n\t"
      "mov.b64 db, {%3, %4};\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}"
      :
      : "r"(d), "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(acc)
      : "memory");
}

// D[tmem] (+)= A[tmem] B[smem]^T: A (M x 16) in TMEM, lane = row, 16-bit
// elements packed two per 32-bit column.
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi,
                                       uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}"
      :
      : "r"(d), "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

__device__ __forceinline__ void arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// CTA `cta` of the grid: token range `range`, shard index `i` among the
// range's nsh shards.
__device__ __forceinline__ void cta_role(const Params& p, int cta, int& range, int& i) {
  range = cta / p.nsh;
  i = cta % p.nsh;
}

__device__ void producer(const Params& p, const CUtensorMap* qmap, const CUtensorMap* kvmap,
                         int range, int g, int pid, uint32_t sbase, const Layout& L,
                         const Bars& bars, volatile int* abort_flag) {
  const int lane = threadIdx.x & 31;
  Cursor cur;
  seg_begin(p, range, cur);
  Segment s;
  PageWindow win;
  uint32_t n = 0, qloads = 0;
  const int nq = p.dq + 1;
  while (seg_next(p, range, cur, s)) {
    const int ntiles = s.t_hi - s.t_lo;
    if (ntiles == 0) continue;
    if (pid == 0) {  // the shard's q, once the previous segment's QK^T is done
      if (qloads > 0 && !wait_bar_warp(bars.q_empty(), (qloads - 1) & 1, abort_flag)) return;
      if (lane == 0) mbar_arrive_expect_tx(bars.q_full(), nq * kQChunkBytes);
      __syncwarp();
      if (lane < nq)
        tma_load_3d(sbase + lane * kQChunkBytes, qmap, 64 * stage_chunk(p, g, lane), 0, s.b,
                    bars.q_full());
    }
    ++qloads;
    for (int j = 0; j < ntiles; ++j) {
      const int t = s.t_lo + j;
      int blk0 = 0, blk1 = 0;
      if (p.paged) {
        blk0 = win.get(p, s, 2 * t, lane);
        blk1 = win.get(p, s, 2 * t + 1, lane);
      }
      for (int st = 0; st < nq; ++st) {
        const uint32_t me = n++;
        const uint32_t slot = me % (uint32_t)p.ring;
        if ((slot & 1u) != (uint32_t)pid) continue;
        if (me >= (uint32_t)p.ring &&
            !wait_bar_warp(bars.empty(slot), ((me / p.ring) - 1) & 1, abort_flag))
          return;
        if (lane == 0) mbar_arrive_expect_tx(bars.full(slot), kStage);
        __syncwarp();
        if (lane < 2) {  // one page per lane
          const int c = stage_chunk(p, g, st);
          const uint32_t dst = sbase + L.ring + slot * kStage + lane * (kStage / 2);
          if (p.paged)
            tma_load_4d(dst, kvmap, 0, 0, c, lane == 0 ? blk0 : blk1, bars.full(slot));
          else
            tma_load_4d(dst, kvmap, 0, kTile * t + 64 * lane, c, s.b, bars.full(slot));
        }
      }
    }
  }
}

__device__ void qk_issuer(const Params& p, int range, int g, uint32_t sbase, uint32_t tmem,
                          const Layout& L, const Bars& bars, volatile int* abort_flag) {
  Cursor cur;
  seg_begin(p, range, cur);
  Segment s;
  uint32_t n = 0, qloads = 0, U = 0, parity = 0;
  uint32_t si = 0, sph = 0;  // S buffer of tile U, parity of its use count
  const int nq = p.dq + 1;
  int rk0, rk1;
  rope_steps(p, g, rk0, rk1);
  const uint64_t dQ = sw128_desc(sbase, 16, 1024);
  const uint64_t dR = sw128_desc(sbase + L.ring, 16, 1024);
  const uint32_t q_lo = (uint32_t)dQ, q_hi = (uint32_t)(dQ >> 32);
  const uint32_t r_lo = (uint32_t)dR, r_hi = (uint32_t)(dR >> 32);
  constexpr uint32_t kQDesc = kQChunkBytes >> 4, kStageDesc = kStage >> 4;
  while (seg_next(p, range, cur, s)) {
    const int ntiles = s.t_hi - s.t_lo;
    if (ntiles == 0) continue;
    if (!wait_bar(bars.q_full(), qloads & 1, abort_flag)) return;
    ++qloads;
    tc_fence_after();
    for (int j = 0; j < ntiles; ++j, ++U) {
      // S buffer si (with the P over it) is free once P.V of tile U - nS completed
      if (U >= (uint32_t)p.nS && !wait_bar(bars.pv_done(si), sph ^ 1u, abort_flag)) return;
      tc_fence_after();
      const uint32_t dS = tmem + kColS + 128 * si;
      uint32_t acc = 0;
      for (int st = 0; st < nq; ++st) {
        const uint32_t slot = (n + st) % (uint32_t)p.ring;
        if (!wait_bar(bars.full(slot), (parity >> slot) & 1u, abort_flag)) return;
        parity ^= 1u << slot;
        const uint32_t a = q_lo + (uint32_t)st * kQDesc;
        const uint32_t b = r_lo + slot * kStageDesc;
        if (st > 0) {
          mma_ss(dS, a, q_hi, b, r_hi, kIdescQK, acc);
          mma_ss(dS, a + 2, q_hi, b + 2, r_hi, kIdescQK, 1u);
          mma_ss(dS, a + 4, q_hi, b + 4, r_hi, kIdescQK, 1u);
          mma_ss(dS, a + 6, q_hi, b + 6, r_hi, kIdescQK, 1u);
          acc = 1;
        } else {
          for (int kk = rk0; kk < rk1; ++kk) {
            mma_ss(dS, a + 2 * kk, q_hi, b + 2 * kk, r_hi, kIdescQK, acc);
            acc = 1;
          }
          commit(bars.empty(slot));  // the rope chunk is needed by QK^T only
        }
      }
      commit(bars.s_full(si));
      n += nq;
      if (++si == (uint32_t)p.nS) {
        si = 0;
        sph ^= 1u;
      }
    }
    commit(bars.q_empty());
  }
}

__device__ void pv_issuer(const Params& p, int range, uint32_t sbase, uint32_t tmem,
                          const Layout& L, const Bars& bars, volatile int* abort_flag) {
  Cursor cur;
  seg_begin(p, range, cur);
  Segment s;
  uint32_t n = 0, U = 0;
  uint32_t si = 0, sph = 0;  // S / P buffer of tile U, parity of its use count
  const uint32_t colO = kColS + 128 * (uint32_t)p.nS;
  const int nq = p.dq + 1;
  // MN-major V operand: rows = tokens (K), 64 latent columns per 128-byte
  // row; chunks in consecutive slots form one operand whose 64-column groups
  // lie one stage apart (the leading-byte offset)
  const uint64_t dV = sw128_desc(sbase + L.ring, kStage / 2, 1024);
  const uint64_t dV2 = sw128_desc(sbase + L.ring, kStage, 1024);
  const uint32_t v_lo = (uint32_t)dV, v_hi = (uint32_t)(dV >> 32);
  const uint32_t v2_lo = (uint32_t)dV2, v2_hi = (uint32_t)(dV2 >> 32);
  constexpr uint32_t kStageDesc = kStage >> 4;
  const uint32_t ring = (uint32_t)p.ring;
  while (seg_next(p, range, cur, s)) {
    const int ntiles = s.t_hi - s.t_lo;
    if (ntiles == 0) continue;
    for (int j = 0; j < ntiles; ++j, ++U) {
      if (!wait_bar(bars.p_full(si), sph, abort_flag)) return;
      tc_fence_after();
      const uint32_t pa = tmem + kColS + 128 * si;  // P: 64 columns of bf16 pairs
      for (int c = 0; c < p.dq;) {
        // the tile's next latent chunks, two at a time where their slots are
        // consecutive, are one operand of N = 64 x run.  (Runs of four, N =
        // 256, measured slower at G = 2: the first slot of a run is released
        // only when the whole run is done.)
        const uint32_t slot = (n + 1 + c) % ring;
        const int run = min(min(p.dq - c, (int)(ring - slot)), 2);
        const uint32_t dO = tmem + colO + 64 * c;
        const uint32_t idesc = kIdescPVn[run - 1];
        const uint32_t b = (run > 1 ? v2_lo : v_lo) + slot * kStageDesc;
        const uint32_t bh = run > 1 ? v2_hi : v_hi;
#pragma unroll
        for (int k = 0; k < 8; ++k)  // 16 tokens per step: P +8 columns, V +2 KB
          mma_ts(dO, pa + 8 * k, b + 128 * k, bh, idesc, (j | k) != 0);
        for (int r = 0; r < run; ++r) commit(bars.empty(slot + r));
        c += run;
      }
      commit(bars.pv_done(si));
      n += nq;
      if (++si == (uint32_t)p.nS) {
        si = 0;
        sph ^= 1u;
      }
    }
  }
}

__device__ void softmax(const Params& p, int range, int i_sh, int g, uint32_t tmem,
                        const Bars& bars, volatile int* abort_flag) {
  const int w = (int)(threadIdx.x >> 5);
  const int head = 32 * (w & 3) + (int)(threadIdx.x & 31);  // = this thread's TMEM lane
  const uint32_t lane_base = (uint32_t)(32 * (w & 3)) << 16;
  const int col_base = p.shard < 0 ? g * p.d : 0;
  const uint32_t colO = kColS + 128 * (uint32_t)p.nS;
  Cursor cur;
  seg_begin(p, range, cur);
  Segment s;
  uint32_t U = 0;
  uint32_t si = 0, sph = 0;  // S buffer of tile U, parity of its use count
  // buffer and parity of tile U - 1 (the previous P.V)
  auto prev_buf = [&]() { return si == 0 ? (uint32_t)p.nS - 1 : si - 1; };
  auto prev_ph = [&]() { return si == 0 ? sph ^ 1u : sph; };
  while (seg_next(p, range, cur, s)) {
    const int ntiles = s.t_hi - s.t_lo;
    if (ntiles == 0) {  // empty chunk: out 0, lse -inf
      float z[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) z[j] = 0.f;
      for (int c0 = 0; c0 < p.d; c0 += 32) write_out_row(p, s, head, col_base + c0, z, 0.f);
      write_lse(p, s, head, i_sh, -INFINITY);
      continue;
    }
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < ntiles; ++j, ++U) {
      const int t = s.t_lo + j;
      if (!wait_bar(bars.s_full(si), sph, abort_flag)) return;
      tc_fence_after();
      const uint32_t sb = tmem + lane_base + kColS + 128 * si;
      float x[128];
      {
        uint32_t r[4][32];
        tmem_ld32(sb, r[0]);
        tmem_ld32(sb + 32, r[1]);
        tmem_ld32(sb + 64, r[2]);
        tmem_ld32(sb + 96, r[3]);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 128; ++k) x[k] = __uint_as_float(r[k >> 5][k & 31]);
      }
      if (p.negate) {
#pragma unroll
        for (int k = 0; k < 128; ++k) x[k] = -x[k];
      }
      const int nv = max(0, min(kTile, s.L - kTile * t));
      if (nv < kTile) {  // warp-uniform: the request's last tile
#pragma unroll
        for (int k = 0; k < 128; ++k) x[k] = k < nv ? x[k] : -INFINITY;
      }
      float mx0 = fmaxf(x[0], x[1]), mx1 = fmaxf(x[2], x[3]);
#pragma unroll
      for (int k = 4; k < 128; k += 4) {
        mx0 = fmaxf(mx0, fmaxf(x[k], x[k + 1]));
        mx1 = fmaxf(mx1, fmaxf(x[k + 2], x[k + 3]));
      }
      const float mx = fmaxf(mx0, mx1) * p.scale_log2;
      float factor = 1.f;
      int resc = 0;
      if (m == -INFINITY) {
        m = mx;
      } else if (mx > m + kRescaleThreshold) {
        factor = ex2(m - mx);
        m = mx;
        resc = 1;
      }
      l *= factor;
      if (__any_sync(0xffffffffu, resc)) {
        // O was last written by P.V of tile U - 1 (not the first of the segment)
        if (!wait_bar(bars.pv_done(prev_buf()), prev_ph(), abort_flag)) return;
        tc_fence_after();
        for (int c0 = 0; c0 < p.d; c0 += 32) {
          const uint32_t ta = tmem + lane_base + colO + c0;
          uint32_t o[32];
          tmem_ld32(ta, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * factor);
          tmem_st32(ta, o);
        }
        tmem_wait_st();
      }
      // P = 2^(x - m) in bf16 (masked tokens give 0); l sums the rounded values.
      // P goes over this lane's own S columns [0, 64): the thread has read them.
      const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nm2 = f2_pack(-m, -m);
      uint64_t ls2 = f2_pack(0.f, 0.f);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          float e0, e1;
          f2_unpack(f2_fma(f2_pack(x[64 * h + 2 * k], x[64 * h + 2 * k + 1]), sc2, nm2), e0, e1);
          const uint32_t u = cvt_bf16x2(ex2(e0), ex2(e1));
          ls2 = f2_add(ls2, f2_pack(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u)));
          pk[k] = u;
        }
        tmem_st32(sb + 32 * h, pk);
      }
      float ls0, ls1;
      f2_unpack(ls2, ls0, ls1);
      l += ls0 + ls1;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) arrive(bars.p_full(si));
      if (++si == (uint32_t)p.nS) {
        si = 0;
        sph ^= 1u;
      }
    }
    // epilogue: the segment's last P.V done
    if (!wait_bar(bars.pv_done(prev_buf()), prev_ph(), abort_flag)) return;
    tc_fence_after();
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const float lse = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
    for (int c0 = 0; c0 < p.d; c0 += 32) {
      uint32_t o[32];
      tmem_ld32(tmem + lane_base + colO + c0, o);
      tmem_wait_ld();
      write_out_row(p, s, head, col_base + c0, reinterpret_cast<const float*>(o), inv);
    }
    write_lse(p, s, head, i_sh, lse);
    tc_fence_before();
  }
}

__global__ void __launch_bounds__(kThreads, 1)
tpla_decode_shard_kernel(const __grid_constant__ CUtensorMap qmap,
                         const __grid_constant__ CUtensorMap kvmap, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Layout L = layout(p);
  const Bars bars{sbase + L.bars};
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.abort);
  int range, i_sh;
  cta_role(p, (int)blockIdx.x, range, i_sh);
  const int g = shard_of(p, i_sh);
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.ring; ++s) {
      mbar_init(bars.full(s), 1);
      mbar_init(bars.empty(s), 1);
    }
    mbar_init(bars.q_full(), 1);
    mbar_init(bars.q_empty(), 1);
    for (int i = 0; i < kMaxS; ++i) {
      mbar_init(bars.s_full(i), 1);
      mbar_init(bars.p_full(i), kSoftmaxWarps);
      mbar_init(bars.pv_done(i), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpProd0 && lane == 0) {
    tma_prefetch(&qmap);
    tma_prefetch(&kvmap);
  }
  if (warp == kWarpQK) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     sbase + L.tmem_slot)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L.tmem_slot);

  if (warp == kWarpQK) {
    if (lane == 0) qk_issuer(p, range, g, sbase, tmem, L, bars, abort_flag);
  } else if (warp == kWarpPV) {
    if (lane == 0) pv_issuer(p, range, sbase, tmem, L, bars, abort_flag);
  } else if (warp < kWarpSm0) {
    producer(p, &qmap, &kvmap, range, g, warp - kWarpProd0, sbase, L, bars, abort_flag);
  } else {
    softmax(p, range, i_sh, g, tmem, bars, abort_flag);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpQK) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

}  // namespace shd

// ---------------------------------------------------------------- merge of partial slots
//
// Requests cut by a range boundary (or explicitly split) left normalised
// partial outputs and their lse in workspace slots; the exact log-sum-exp
// rule combines them.  A block covers one request and kMergeHeads heads, one
// warp per head: the lanes hold the slots' lse (32 at a time) and 16-byte
// column groups, so every warp keeps several independent loads in flight.
// Requests that one cluster finished (written final by the decode kernel)
// return after the block's prefix sum.

constexpr int kMergeHeads = 8;
constexpr int kMergeThreads = 32 * kMergeHeads;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kMergeThreads)
sm100_merge_kernel(const Params p) {
  // every block waits for the decode grid (launched as its programmatic
  // dependent), so that this grid cannot finish before the decode has
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * kMergeHeads + warp;
  __shared__ long long red[2][kMergeHeads];
  long long pre = 0, tot = 0;
  if (p.mode == 0 && !p.seq_lens) {  // causal lengths: closed form
    pre = cost_before(p, b);
    tot = cost_before(p, p.B);
  } else if (p.mode == 0) {  // schedule cost before request b and in total
    for (int bb = threadIdx.x; bb < p.B; bb += kMergeThreads) {
      const long long nc = req_cost(p, bb);
      tot += nc;
      if (bb < b) pre += nc;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      pre += __shfl_xor_sync(0xffffffffu, pre, o);
      tot += __shfl_xor_sync(0xffffffffu, tot, o);
    }
    if (lane == 0) {
      red[0][warp] = pre;
      red[1][warp] = tot;
    }
    __syncthreads();
    pre = tot = 0;
    for (int w = 0; w < kMergeHeads; ++w) {
      pre += red[0][w];
      tot += red[1][w];
    }
  }
  const long long T = tot;
  const int nt = req_tiles(p, b);
  int s_lo = 0, s_hi = 0;  // cluster range of request b
  const long long P = min((long long)p.P, T);  // clusters that received work
  if (nt > 0) {
    if (p.mode == 0) {  // the ranges holding the request's first and last tile
      const long long x0 = pre + p.seg_cost;
      s_lo = (int)(((x0 + 1) * P + T - 1) / T - 1);
      s_hi = (int)(((x0 + nt) * P + T - 1) / T - 1);
      if (s_lo == s_hi) return;  // one cluster wrote the final result
    } else {
      if (p.S == 1) return;
      s_lo = b * p.S;
      s_hi = b * p.S + p.S - 1;
    }
  }
  if (h >= p.H) return;
  const int cw = p.W / p.nsh;  // columns per shard (a multiple of 64)
  auto write4 = [&](int col, float4 v) {
    const int64_t off = (int64_t)b * p.o_sb + (int64_t)h * p.o_sh + col;
    if (p.out_bf16) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
      uint2 w;
      w.x = *reinterpret_cast<uint32_t*>(&lo);
      w.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.out) + off) = w;
    } else {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + off) = v;
    }
  };
  auto write_lse = [&](int k, float v) {
    if (p.lse && lane == 0) p.lse[(int64_t)b * p.l_sb + (int64_t)h * p.l_sh + k] = v;
  };
  if (nt == 0) {  // empty request: never reached by the decode kernel
    for (int k = 0; k < p.nsh; ++k) {
      for (int c = 4 * lane; c < cw; c += 128) write4(k * cw + c, make_float4(0.f, 0.f, 0.f, 0.f));
      write_lse(k, -INFINITY);
    }
    return;
  }
  // Slot of range c's partial of this request: 2c, except the first range,
  // which used its second slot when it began before the request (an earlier
  // request's tiles came first; the one 64-bit division is done once here).
  const int first_slot = (p.mode == 0 && (long long)s_lo * T / P < pre) ? 2 * s_lo + 1 : 2 * s_lo;
  auto slot_of = [&](int c) -> int { return c == s_lo ? first_slot : 2 * c; };
  // Column groups of this lane: 16-byte groups 4 * lane + 128 * i of each
  // shard (cw <= 512, so at most four).  Loads of two slots x all groups go
  // out together before the multiply-adds.
  const int ngrp = (cw + 127) / 128;
  if (s_hi == s_lo + 1 && p.nsh * ngrp <= 4) {
    // The usual case, a request cut once: two slots.  Every shard's lse and
    // row groups of both slots are loaded before any is used, so the merge
    // costs one round trip to memory instead of two per shard.
    const int sa = first_slot, sb = 2 * s_hi;
    const int nj = p.nsh * ngrp;
    float4 oa[4], ob[4];
    float la[4], lb[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      oa[j] = ob[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      la[j] = lb[j] = -INFINITY;
      if (j < nj) {
        const int k = j / ngrp, i = j - k * ngrp;
        if (4 * lane + 128 * i < cw) {
          const int64_t col = (int64_t)h * p.W + k * cw + 4 * lane + 128 * i;
          oa[j] = __ldcg(reinterpret_cast<const float4*>(p.part_o + (int64_t)sa * p.H * p.W + col));
          ob[j] = __ldcg(reinterpret_cast<const float4*>(p.part_o + (int64_t)sb * p.H * p.W + col));
        }
      }
      if (j < p.nsh) {
        la[j] = __ldcg(p.part_l + ((int64_t)sa * p.H + h) * p.nsh + j);
        lb[j] = __ldcg(p.part_l + ((int64_t)sb * p.H + h) * p.nsh + j);
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (k >= p.nsh) break;
      const float M = fmaxf(la[k], lb[k]);
      float total = -INFINITY, wa = 0.f, wb = 0.f;
      if (M != -INFINITY) {
        total = M + logf(expf(la[k] - M) + expf(lb[k] - M));
        wa = la[k] == -INFINITY ? 0.f : expf(la[k] - total);
        wb = lb[k] == -INFINITY ? 0.f : expf(lb[k] - total);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (j < nj && j / ngrp == k) {
          const int i = j - k * ngrp;
          if (4 * lane + 128 * i < cw) {
            // a slot of weight 0 contributes nothing, whatever its row holds
            const float4 a = wa != 0.f ? oa[j] : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 c = wb != 0.f ? ob[j] : make_float4(0.f, 0.f, 0.f, 0.f);
            write4(k * cw + 4 * lane + 128 * i,
                   make_float4(fmaf(wb, c.x, wa * a.x), fmaf(wb, c.y, wa * a.y),
                               fmaf(wb, c.z, wa * a.z), fmaf(wb, c.w, wa * a.w)));
          }
        }
      }
      write_lse(k, total);
    }
    return;
  }
  for (int k = 0; k < p.nsh; ++k) {
    auto lse_of = [&](int c) { return __ldcg(p.part_l + ((int64_t)slot_of(c) * p.H + h) * p.nsh + k); };
    auto row_of = [&](int c) {
      return reinterpret_cast<const float4*>(p.part_o + ((int64_t)slot_of(c) * p.H + h) * p.W +
                                             k * cw) + lane;
    };
    // lane i holds the lse of slot s_lo + i (the first 32 slots; the usual
    // case has two)
    const float ls_lane = s_lo + lane <= s_hi ? lse_of(s_lo + lane) : -INFINITY;
    float M = ls_lane;
    for (int c = s_lo + 32 + lane; c <= s_hi; c += 32) M = fmaxf(M, lse_of(c));
    M = warp_max(M);
    float z = 0.f;
    if (M != -INFINITY) {
      z = ls_lane == -INFINITY ? 0.f : expf(ls_lane - M);
      for (int c = s_lo + 32 + lane; c <= s_hi; c += 32) {
        const float ls = lse_of(c);
        z += ls == -INFINITY ? 0.f : expf(ls - M);
      }
    }
    z = warp_sum(z);
    const float total = M == -INFINITY ? -INFINITY : M + logf(z);
    float4 acc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (total != -INFINITY) {
      for (int g0 = s_lo; g0 <= s_hi; g0 += 32) {
        const float lsm = g0 == s_lo ? ls_lane : (g0 + lane <= s_hi ? lse_of(g0 + lane) : -INFINITY);
        const float wmine = lsm == -INFINITY ? 0.f : expf(lsm - total);
        const int n = min(32, s_hi - g0 + 1);
        for (int i0 = 0; i0 < n; i0 += 2) {
          const float w0 = __shfl_sync(0xffffffffu, wmine, i0);
          const float w1 = __shfl_sync(0xffffffffu, wmine, min(i0 + 1, 31));
          const bool has1 = i0 + 1 < n && w1 != 0.f;
          const float4* r0 = row_of(g0 + i0);
          const float4* r1 = has1 ? row_of(g0 + i0 + 1) : r0;
          float4 o0[4], o1[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (i < ngrp && 4 * lane + 128 * i < cw) {
              o0[i] = w0 != 0.f ? __ldcg(r0 + 32 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
              o1[i] = has1 ? __ldcg(r1 + 32 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }
          const float v1 = has1 ? w1 : 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (i < ngrp && 4 * lane + 128 * i < cw) {
              acc[i].x = fmaf(v1, o1[i].x, fmaf(w0, o0[i].x, acc[i].x));
              acc[i].y = fmaf(v1, o1[i].y, fmaf(w0, o0[i].y, acc[i].y));
              acc[i].z = fmaf(v1, o1[i].z, fmaf(w0, o0[i].z, acc[i].z));
              acc[i].w = fmaf(v1, o1[i].w, fmaf(w0, o0[i].w, acc[i].w));
            }
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (i < ngrp && 4 * lane + 128 * i < cw) write4(k * cw + 4 * lane + 128 * i, acc[i]);
    write_lse(k, total);
  }
}

// ---------------------------------------------------------------- timeout self-test

// One thread waits, through the kernels' bounded barrier wait, on a barrier
// that nothing completes: after `limit` cycles the wait records
// TPLA_ERR_DEVICE_TIMEOUT in the status word and returns, and the kernel
// exits.  Lets a test exercise the timeout path without faulting the GPU.
__global__ void wait_timeout_selftest_kernel(long long limit) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_addr(&bar);
  mbar_init(b, 1);
  abort_flag = 0;
  fence_mbar_init();
  wait_bar(b, 0, &abort_flag, limit);
}

// ---------------------------------------------------------------- host side

struct DeviceInfo {
  bool init = false;
  bool sm100 = false;
  int max_clusters = 0;  // pair kernel: co-resident clusters of 2
  int shard_ctas = 0;    // shard kernel: co-resident CTAs (one per SM)
};
std::mutex g_mu;
DeviceInfo g_dev[64];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// cuTensorMapEncodeTiled from the driver (looked up once; g_mu held).
void* encoder_locked() {
  static void* fn = nullptr;
  if (fn) return fn;
  void* f = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !f) {
    cudaGetLastError();
    return nullptr;
  }
  fn = f;
  return fn;
}

cudaError_t launch_config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attr, int clusters,
                          cudaStream_t stream) {
  cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaSuccess;
}

const DeviceInfo& device_info(int dev) {
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev & 63];
  if (d.init) return d;
  d.init = true;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return d;
  }
  if (major != 10 || minor != 0) return d;
  if (!g_encode) {
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(encoder_locked());
    if (!g_encode) return d;
  }
  if (cudaFuncSetAttribute(tpla_decode_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kSmemBytes) != cudaSuccess) {
    cudaGetLastError();
    return d;
  }
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  launch_config(cfg, attr, sms / 2, nullptr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, tpla_decode_sm100_kernel, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return d;
  }
  d.max_clusters = n;
  if (cudaFuncSetAttribute(shd::tpla_decode_shard_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           shd::kSmemBytes) != cudaSuccess) {
    cudaGetLastError();
    return d;
  }
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, shd::tpla_decode_shard_kernel,
                                                    shd::kThreads, shd::kSmemBytes) !=
          cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    return d;
  }
  d.shard_ctas = sms * per_sm;
  d.sm100 = true;
  return d;
}

bool encode_map(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box_rows = 64) {
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Cache as a 4-D tensor (column within chunk, row, 64-column chunk, page or
// request): a box of `k` chunks lands k consecutive [64 rows][64 bf16]
// swizzled tiles.  Rows past `rows` (and pages past `pages`) read as zeros.
bool encode_kv_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t pages,
                   uint64_t row_stride_bytes, uint64_t page_stride_bytes, int k) {
  cuuint64_t dims[4] = {64, rows, (cuuint64_t)kQChunks, pages};
  cuuint64_t strides[3] = {row_stride_bytes, 128, page_stride_bytes};
  cuuint32_t box[4] = {64, 64, (cuuint32_t)k, 1};
  cuuint32_t estride[4] = {1, 1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                        strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_slots(const DecodeProblem& p, int num_splits, int max_clusters) {
  if (num_splits == 0) return 2 * max_clusters;
  if (num_splits == 1) return 0;
  return 2 * p.B * num_splits;
}

// TPLA shards (G >= 2) run on the shard kernel, exact MLA on the pair kernel.
bool use_shard_kernel(const DecodeProblem& p) { return p.G >= 2; }

// Token ranges of the persistent schedule.
int num_ranges(const DecodeProblem& p, const DeviceInfo& d) {
  return use_shard_kernel(p) ? d.shard_ctas / p.n_shards : d.max_clusters;
}

}  // namespace

void* tensor_map_encoder() {
  std::lock_guard<std::mutex> lock(g_mu);
  return encoder_locked();
}

bool sm100_device(int device) {
  if (device < 0 || device >= 64) return false;
  return device_info(device).sm100;
}

bool sm100_supported(const DecodeProblem& p, int device) {
  if (device < 0 || device >= 64) return false;
  if (!(p.G == 1 || p.G == 2 || p.G == 4)) return false;
  if (p.H < 1) return false;  // more than 128 heads: one launch per 128-head group
  if (!isfinite(p.scale)) return false;
  if (p.cache_rows > (1 << 30) || (p.page_table && p.num_blocks >= (1LL << 31) - 1)) return false;
  if (p.page_table && p.max_pages > (1 << 24)) return false;
  // 16-byte vector stores of out rows
  const int vec = p.out_bf16 ? 8 : 4;
  if ((reinterpret_cast<uintptr_t>(p.out) & 15u) || (p.o_sb % vec) || (p.o_sh % vec)) return false;
  const DeviceInfo& d = device_info(device);
  return d.sm100;
}

size_t sm100_workspace_bytes(const DecodeProblem& p, int num_splits, int device) {
  const DeviceInfo& d = device_info(device);
  const int slots = num_slots(p, num_splits, num_ranges(p, d));
  if (slots == 0) return 0;
  const size_t Hg = p.H < 128 ? p.H : 128;  // heads of one launch (128-head groups)
  const size_t o = (size_t)slots * Hg * p.out_width * sizeof(float);
  return ((o + 255) / 256) * 256 + (size_t)slots * Hg * p.n_shards * sizeof(float);
}

cudaError_t launch_decode_sm100_group(const DecodeProblem& dp, int num_splits, void* ws,
                                      size_t ws_bytes, cudaStream_t stream);
cudaError_t launch_decode_shard_group(const DecodeProblem& dp, int num_splits, void* ws,
                                      size_t ws_bytes, cudaStream_t stream);

// More than 128 heads: one launch (plus merge) per group of up to 128 heads,
// in stream order, reusing the same workspace.
cudaError_t launch_decode_sm100(const DecodeProblem& dp, int num_splits, void* ws, size_t ws_bytes,
                                cudaStream_t stream) {
  for (int h0 = 0; h0 < dp.H; h0 += 128) {
    DecodeProblem g = dp;
    g.H = dp.H - h0 < 128 ? dp.H - h0 : 128;
    g.q = reinterpret_cast<const __nv_bfloat16*>(dp.q) + (int64_t)h0 * dp.q_sh;
    g.out = reinterpret_cast<char*>(dp.out) + (int64_t)h0 * dp.o_sh * (dp.out_bf16 ? 2 : 4);
    g.lse = dp.lse ? dp.lse + (int64_t)h0 * dp.l_sh : nullptr;
    cudaError_t e = use_shard_kernel(g) ? launch_decode_shard_group(g, num_splits, ws, ws_bytes, stream)
                                        : launch_decode_sm100_group(g, num_splits, ws, ws_bytes, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Fields both kernels share; the caller sets the schedule and the ring.
void fill_params(const DecodeProblem& dp, Params& p) {
  p = Params{};
  p.seq_lens = dp.seq_lens;
  p.causal_base = dp.causal_base;
  p.page_table = dp.page_table;
  p.pt_sb = dp.pt_sb;
  p.num_blocks = (int)dp.num_blocks;
  p.cap_tokens = (int)dp.cache_rows;
  p.paged = dp.page_table != nullptr;
  p.B = dp.B;
  p.H = dp.H;
  p.G = dp.G;
  p.split_rope = dp.rope_mode == TPLA_ROPE_SPLIT;
  p.shard = dp.shard;
  p.nsh = dp.n_shards;
  p.d = kLatent / dp.G;
  p.dq = p.d / 64;
  p.NB = p.d < 256 ? p.d : 256;
  p.nblk = p.d / p.NB;
  // The kernels take the row max of the sign-corrected raw scores and apply
  // |scale| inside exp2.  A zero scale becomes 1e-30 (log2 units): every
  // finite score then gives exp2(~0) = 1 exactly in f32, as scale 0 does,
  // while masked (-inf) scores still give 0.
  p.scale_log2 = fmaxf((float)(fabs((double)dp.scale) * 1.4426950408889634), 1e-30f);
  p.negate = dp.scale < 0.f;
  p.out = dp.out;
  p.out_bf16 = dp.out_bf16;
  p.o_sb = dp.o_sb;
  p.o_sh = dp.o_sh;
  p.lse = dp.lse;
  p.l_sb = dp.l_sb;
  p.l_sh = dp.l_sh;
  p.W = dp.out_width;
}

// Split slots in the workspace and the schedule (balanced ranges or explicit
// splits); returns false when the workspace is missing or short.
bool set_schedule(const DecodeProblem& dp, int num_splits, int ranges, void* ws, size_t ws_bytes,
                  Params& p) {
  const int slots = num_slots(dp, num_splits, ranges);
  if (slots > 0) {
    const size_t o = (size_t)slots * dp.H * dp.out_width * sizeof(float);
    const size_t need = ((o + 255) / 256) * 256 + (size_t)slots * dp.H * dp.n_shards * sizeof(float);
    if (!ws || ws_bytes < need) return false;
    p.part_o = reinterpret_cast<float*>(ws);
    p.part_l = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + ((o + 255) / 256) * 256);
  }
  if (num_splits == 0) {
    p.mode = 0;
    p.P = ranges;
    p.S = 1;
  } else {
    p.mode = 1;
    p.S = num_splits;
    p.P = dp.B * num_splits;
  }
  return true;
}

// The merge is launched as a programmatic dependent of the decode kernel:
// its blocks are scheduled as the decode's CTAs retire and wait (griddepcontrol)
// for the whole decode grid and its writes before reading anything.
cudaError_t launch_merge(const DecodeProblem& dp, const Params& p, cudaStream_t stream) {
  if (p.mode == 1 && p.S == 1) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(dp.B, (dp.H + kMergeHeads - 1) / kMergeHeads);
  cfg.blockDim = dim3(kMergeThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, sm100_merge_kernel, p);
  count_launch();
  return e;
}

cudaError_t launch_decode_sm100_group(const DecodeProblem& dp, int num_splits, void* ws,
                                      size_t ws_bytes, cudaStream_t stream) {
  int dev = 0;
  cudaGetDevice(&dev);
  const DeviceInfo& d = device_info(dev);
  if (!d.sm100) return cudaErrorNotSupported;
  CUtensorMap qmap, kv[2];
  if (!encode_map(&qmap, dp.q, kWidth, dp.H, dp.B, dp.q_sh * 2, dp.q_sb * 2))
    return cudaErrorInvalidValue;
  for (int k = 1; k <= kSlotChunks; ++k) {
    const bool ok = dp.page_table
                        ? encode_kv_map(&kv[k - 1], dp.cache, kBlock, dp.num_blocks, dp.c_s1 * 2,
                                        dp.c_s0 * 2, k)
                        : encode_kv_map(&kv[k - 1], dp.cache, dp.cache_rows, dp.B, dp.c_s1 * 2,
                                        dp.c_s0 * 2, k);
    if (!ok) return cudaErrorInvalidValue;
  }
  Params p;
  fill_params(dp, p);
  // QK^T stages wait ~2 us to land and then only for the tensor core, so
  // they get most of the ring; PV stages are consumed at the softmax's pace.
  // Measured (slot sweep on the DeepSeek-V3 workload): G=1 (eight PV stages
  // per tile) and G=4 (two) want 3 QK^T slots, G=2 wants 4.
  p.qk_slots = dp.G == 2 ? 4 : 3;
  p.pv_slots = kRingSlots - p.qk_slots;
  p.tile_tok = kTileTok;
  p.seg_cost = 2;  // q load and epilogue (measured best of 1-3 on prompt prefill)
  if (!set_schedule(dp, num_splits, d.max_clusters, ws, ws_bytes, p)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  launch_config(cfg, attr, p.P, stream);
  cudaError_t e = cudaLaunchKernelEx(&cfg, tpla_decode_sm100_kernel, qmap, kv[0], kv[1], p);
  count_launch();
  if (e != cudaSuccess) return e;
  return launch_merge(dp, p, stream);
}

cudaError_t launch_decode_shard_group(const DecodeProblem& dp, int num_splits, void* ws,
                                      size_t ws_bytes, cudaStream_t stream) {
  int dev = 0;
  cudaGetDevice(&dev);
  const DeviceInfo& d = device_info(dev);
  if (!d.sm100 || d.shard_ctas < dp.n_shards) return cudaErrorNotSupported;
  CUtensorMap qmap, kv;
  if (!encode_map(&qmap, dp.q, kWidth, dp.H, dp.B, dp.q_sh * 2, dp.q_sb * 2, 128))
    return cudaErrorInvalidValue;
  const bool ok = dp.page_table ? encode_kv_map(&kv, dp.cache, kBlock, dp.num_blocks, dp.c_s1 * 2,
                                                dp.c_s0 * 2, 1)
                                : encode_kv_map(&kv, dp.cache, dp.cache_rows, dp.B, dp.c_s1 * 2,
                                                dp.c_s0 * 2, 1);
  if (!ok) return cudaErrorInvalidValue;
  Params p;
  fill_params(dp, p);
  p.tile_tok = shd::kTile;
  p.seg_cost = 2;  // q load and epilogue (measured best of 2-6 on mixed lengths)
  // the ring takes the shared memory the shard's q leaves
  const int q_bytes = (p.dq + 1) * shd::kQChunkBytes;
  int ring = (shd::kSmemBytes - 1024 - q_bytes - shd::kMiscBytes) / shd::kStage;
  p.ring = ring > shd::kMaxRing ? shd::kMaxRing : ring;
  if (p.ring < 2) return cudaErrorNotSupported;
  // TMEM holds nS S buffers of 128 columns and O (d columns): a third
  // buffer fits for d <= 128 (G >= 4) and lets a third tile into flight
  p.nS = (512 - p.d) / 128 < shd::kMaxS ? (512 - p.d) / 128 : shd::kMaxS;
  if (!set_schedule(dp, num_splits, num_ranges(dp, d), ws, ws_bytes, p))
    return cudaErrorInvalidValue;
  const int ctas = p.P * p.nsh;
  shd::tpla_decode_shard_kernel<<<ctas, shd::kThreads, shd::kSmemBytes, stream>>>(qmap, kv, p);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_merge(dp, p, stream);
}

cudaError_t launch_wait_timeout_selftest(long long cycles, cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(cycles);
  count_launch();
  return cudaGetLastError();
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
