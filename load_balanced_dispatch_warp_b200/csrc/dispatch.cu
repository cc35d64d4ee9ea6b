// Zero-copy placement and dispatch of token rows: the rank of every assignment within its
// expert, its row in the static per-rank (or per-expert) buffers, and the row copy.
//
// Dispatch is the first all-to-all phase of "DeepEP-on-EFA Guidance, section 1: What is
// MoE" (each token goes to its k chosen experts only); the MoonEP news article
// (paragraph 3) places tokens straight into their final rows of static-shape buffers.  The
// fixed-capacity layout follows "MoE Load Balancing: Find Expert Hotspots", section "Make
// expert capacity, overflow, and padding explicit".
//
// Two launches:
//   rank_kernel     one pass over 256-token tiles.  A tile counts its assignments per
//                   expert (per-warp lane masks keep token order), publishes the counts,
//                   and adds up the counts of all earlier tiles by a decoupled look-back:
//                   one warp reads the status words of 32 predecessors at once and the
//                   block sums their vectors, stopping at the nearest predecessor that has
//                   already published its inclusive prefix.  Tiles are claimed in order
//                   through an atomic counter, so every tile a block waits on belongs to a
//                   block that is already running and waits on nothing later; each wait is
//                   bounded (%globaltimer) and gives up with MOE_DERR_TIMEOUT.  Then each
//                   assignment's rank q in token order gives its row, perm and src.
//   scatter_kernel  the row copy on the Tensor Memory Accelerator: one thread per CTA
//                   drives a ring of shared-memory row buffers, loading token rows with
//                   cp.async.bulk (completion on an mbarrier) and storing each to its k
//                   rows with bulk stores.  In the fixed-capacity layout the other warps
//                   zero the padding rows meanwhile.  Below 32 tokens per SM the ring
//                   does not fill, and scatter_warp_kernel (one warp per token, 16-byte
//                   loads and stores; padding by pad_rows_kernel) runs instead.
// The error word is read once at each kernel's start.  rank_kernel's blocks never write
// it during the launch: their error bits collect in the workspace and the block that
// finishes the last tile publishes them, so every block takes the same entry decision.
#include "rows.cuh"

namespace moe {
namespace {

constexpr int kRankTile = 256;  // tokens per tile: 8 warps x 32 lanes, one token per lane
constexpr int kRankWarps = kRankTile / 32;
constexpr uint64_t kWaitLimitNs = 500000000ull;  // 0.5 s

// workspace words: [0] tile counter, [1] finished tiles, [2] error bits, [3] unused,
// [4, 4 + ntiles) tile status (0 nothing, 1 counts published, 2 inclusive prefix
// published), then counts[ntiles][E] and inclusive[ntiles][E].
__host__ __device__ inline int64_t ws_agg_off(int ntiles) { return ((4 + (int64_t)ntiles) + 3) / 4 * 4; }
__host__ __device__ inline int64_t ws_incl_off(int ntiles, int E) {
  return ws_agg_off(ntiles) + (int64_t)ntiles * E;
}

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ int ld_volatile(const int32_t* p) {
  return *reinterpret_cast<const volatile int32_t*>(p);
}
__device__ __forceinline__ void st_volatile(int32_t* p, int v) {
  *reinterpret_cast<volatile int32_t*>(p) = v;
}

struct RankArgs {
  const int32_t* idx;
  int T, k, E, R, C;
  int cap;               // > 0: fixed-capacity layout, row = e * cap + q (q < cap), else -1
  const int32_t* plan;   // dropless layout (cap == 0): the plan's fields
  moe_plan_layout L;
  const int32_t* q_base; // nullable: [E] assignments of each expert that come before this
                         // launch's tokens in the job's token order (expert parallelism
                         // across processes: the lower ranks' tokens)
  int32_t* ws;
  int ntiles;
  int32_t* perm;
  int32_t* src;
  int32_t* err;
};

// dynamic shared memory: masks [W][E] u32, pre [W][E] int, cnt [E], excl [E], then (plan
// layout) room_prefix [R+1], kept_rows [R], home_off [E], stream_off [E].
__host__ __device__ inline int rank_smem_words(int E, int R) {
  return 2 * kRankWarps * E + 2 * E + 2 * E + 2 * R + 1;
}

__global__ void __launch_bounds__(kRankTile) rank_kernel(RankArgs a) {
  extern __shared__ int smem[];
  const int E = a.E;
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem);  // [W][E]
  int* s_pre = smem + kRankWarps * E;                     // [W][E]
  int* s_cnt = s_pre + kRankWarps * E;                    // [E]
  int* s_excl = s_cnt + E;                                // [E]
  int* s_home = s_excl + E;                               // [E]
  int* s_so = s_home + E;                                 // [E]
  int* s_rp = s_so + E;                                   // [R+1]
  int* s_kr = s_rp + a.R + 1;                             // [R]
  __shared__ int s_tile, s_err, s_lo, s_hi, s_incl, s_stop;
  if (block_should_stop(a.err)) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* status = a.ws + 4;
  int32_t* agg = a.ws + ws_agg_off(a.ntiles);
  int32_t* incl = a.ws + ws_incl_off(a.ntiles, E);
  if (tid == 0) {
    s_tile = atomicAdd(a.ws, 1);
    s_err = 0;
  }
  for (int i = tid; i < kRankWarps * E; i += blockDim.x) s_mask[i] = 0;
  if (a.cap == 0) {
    for (int r = tid; r <= a.R; r += blockDim.x) s_rp[r] = __ldg(a.plan + a.L.room_prefix + r);
    for (int r = tid; r < a.R; r += blockDim.x) s_kr[r] = __ldg(a.plan + a.L.kept_rows + r);
    for (int e = tid; e < E; e += blockDim.x) {
      s_home[e] = __ldg(a.plan + a.L.expert_home_off + e);
      s_so[e] = __ldg(a.plan + a.L.stream_off + e);
    }
  }
  __syncthreads();
  const int tile = s_tile;
  if (tile >= a.ntiles) return;  // never taken: the grid has one block per tile
  const int64_t t = (int64_t)tile * kRankTile + tid;
  const bool tok = t < a.T;
  int my_err = 0;
  // one lane per distinct expert of the warp ORs in the lanes naming it (a token names an
  // expert at most once, so one bit per lane per expert); no shared-memory atomics even
  // when the warp's tokens share hot experts
  for (int j = 0; j < a.k; ++j) {
    int e = tok ? __ldg(a.idx + t * a.k + j) : -1;
    if (tok && (e < 0 || e >= E)) {
      my_err |= MOE_DERR_ID_RANGE;
      e = -1;
    }
    const uint32_t peers = __match_any_sync(MOE_FULL_MASK, e);
    if (e >= 0 && lane == __ffs(peers) - 1) s_mask[warp * E + e] |= peers;
    __syncwarp();
  }
  __syncthreads();
  // counts of this tile; publish them (status 1), or for tile 0 the inclusive prefix
  for (int e = tid; e < E; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kRankWarps; ++w) c += __popc(s_mask[w * E + e]);
    s_cnt[e] = c;
    s_excl[e] = 0;
    __stcg((tile == 0 ? incl : agg) + (int64_t)tile * E + e, c);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) st_volatile(status + tile, tile == 0 ? 2 : 1);
  // decoupled look-back over windows of 32 predecessors
  if (tile > 0) {
    int hi = tile - 1;
    for (;;) {
      if (warp == 0) {
        const int tj = hi - lane;
        int st = 2;
        if (tj >= 0) {
          st = ld_volatile(status + tj);
          if (st == 0) {
            const uint64_t t0 = now_ns();
            while ((st = ld_volatile(status + tj)) == 0) {
              if (now_ns() - t0 > kWaitLimitNs) break;
            }
          }
        }
        const bool lost = tj >= 0 && st == 0;  // the bound ran out
        const uint32_t inclusive = __ballot_sync(MOE_FULL_MASK, tj >= 0 && st == 2);
        const uint32_t timed_out = __ballot_sync(MOE_FULL_MASK, lost);
        if (lane == 0) {
          int stop;
          if (inclusive) {
            stop = __ffs(inclusive) - 1;  // nearest predecessor with an inclusive prefix
          } else {
            stop = min(31, hi);  // all 32 (or down to tile 0, which only ever publishes
                                 // an inclusive prefix) hold counts: sum them, go further
          }
          s_lo = hi - stop;
          s_hi = hi;
          s_incl = inclusive != 0;
          s_stop = inclusive != 0 || timed_out != 0;
          if (timed_out) s_err |= MOE_DERR_TIMEOUT;
        }
        __threadfence();  // order the status reads before the vector reads below
      }
      __syncthreads();
      const int lo = s_lo, hi_w = s_hi, has_incl = s_incl;
      for (int e = tid; e < E; e += blockDim.x) {
        int sum = has_incl ? __ldcg(incl + (int64_t)lo * E + e) : 0;
        for (int p = lo + has_incl; p <= hi_w; ++p) sum += __ldcg(agg + (int64_t)p * E + e);
        s_excl[e] += sum;
      }
      const bool stop = s_stop;
      __syncthreads();
      if (stop) break;
      hi = lo - 1;
    }
    // publish the inclusive prefix
    for (int e = tid; e < E; e += blockDim.x)
      __stcg(incl + (int64_t)tile * E + e, s_excl[e] + s_cnt[e]);
    __threadfence();
    __syncthreads();
    if (tid == 0) st_volatile(status + tile, 2);
  }
  // start of each warp's run of every expert inside the tile
  for (int e = tid; e < E; e += blockDim.x) {
    int run = s_excl[e];
#pragma unroll
    for (int w = 0; w < kRankWarps; ++w) {
      s_pre[w * E + e] = run;
      run += __popc(s_mask[w * E + e]);
    }
  }
  __syncthreads();
  if (tok) {
    const uint32_t lt = lanemask_lt();
    const int64_t rows_total = a.cap > 0 ? (int64_t)E * a.cap : (int64_t)a.R * a.C;
    const int B = E / a.R;
    for (int j = 0; j < a.k; ++j) {
      const int e = __ldg(a.idx + t * a.k + j);
      if (e < 0 || e >= E) continue;
      int q = s_pre[warp * E + e] + __popc(s_mask[warp * E + e] & lt);
      if (a.q_base != nullptr) q += __ldg(a.q_base + e);
      int64_t row;
      if (a.cap > 0) {
        row = q < a.cap ? (int64_t)e * a.cap + q : -1;  // past the capacity: dropped
      } else {
        const int off = s_home[e];
        if (off >= 0) {
          row = (int64_t)(e / B) * a.C + off + q;
        } else {
          const int p = s_so[e] + q;
          int lo = 0, hi = a.R - 1;  // last rank with room_prefix <= p
          while (lo < hi) {
            const int m = (lo + hi + 1) >> 1;
            if (s_rp[m] <= p) lo = m; else hi = m - 1;
          }
          row = (int64_t)lo * a.C + s_kr[lo] + (p - s_rp[lo]);
        }
        if (row < 0 || row >= rows_total) {
          my_err |= MOE_DERR_ID_RANGE;
          row = -1;
        }
      }
      a.perm[t * a.k + j] = (int32_t)row;
      if (row >= 0 && a.src != nullptr) a.src[row] = (int32_t)t;
    }
  }
  if (my_err) atomicOr(&s_err, my_err);
  __syncthreads();
  // the block finishing the last tile publishes the launch's error bits
  if (tid == 0) {
    if (s_err) atomicOr(a.ws + 2, s_err);
    __threadfence();
    if (atomicAdd(a.ws + 1, 1) == a.ntiles - 1) {
      __threadfence();
      const int bits = ld_volatile(a.ws + 2);
      if (bits) atomicOr(a.err, bits);
    }
  }
}

// ----------------------------------------------------------------------------- TMA scatter
constexpr int kScatterThreads = 256;
constexpr int kMaxBuf = 16;
constexpr int kChunkBytes = 16384;   // one bulk copy moves at most this much of a row
constexpr int kMaxTokensPerCta = 256;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  for (;;) {
    if (mbar_try(bar, parity)) return true;
    if (now_ns() - t0 > kWaitLimitNs) return false;
  }
}
// global -> shared bulk copy; completion counted in bytes on `bar`
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
// shared -> global bulk copy, tracked by the thread's bulk groups
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// every committed group but the newest has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all_but_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

struct ScatterArgs {
  const uint8_t* x;        // [T, row_bytes]
  const int32_t* perm;     // [T, k]
  int T, k;
  int row_bytes;
  int chunks;              // copies per row: ceil(row_bytes / kChunkBytes)
  int tokens_per_cta;
  int nbuf;
  int64_t rows_total;
  uint8_t* recv;           // [rows_total, row_bytes]
  // fixed-capacity layout: padding rows e*cap + [min(count_e, cap), cap) are zeroed and
  // their src set to -1 (counts == nullptr: dropless layout, no padding)
  const int32_t* counts;
  int E, cap;
  int32_t* src;
  const int32_t* err;
};

// dynamic shared memory: perm of the CTA's tokens, then nbuf buffers of min(row, chunk)
__global__ void __launch_bounds__(kScatterThreads) scatter_kernel(ScatterArgs a) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ __align__(8) uint64_t s_bar[kMaxBuf];
  if (block_should_stop(a.err)) return;
  const int tid = threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.x * a.tokens_per_cta;
  const int n_tok = (int)max((int64_t)0, min((int64_t)a.T - t0, (int64_t)a.tokens_per_cta));
  int32_t* s_perm = reinterpret_cast<int32_t*>(sm);
  const int perm_bytes = ((a.tokens_per_cta * a.k * 4) + 127) / 128 * 128;
  uint8_t* bufs = sm + perm_bytes;
  const int buf_bytes = min(a.row_bytes, kChunkBytes);
  for (int i = tid; i < n_tok * a.k; i += blockDim.x) s_perm[i] = __ldg(a.perm + t0 * a.k + i);
  if (tid == 0) {
    for (int b = 0; b < a.nbuf; ++b) mbar_init(smem_addr(&s_bar[b]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (tid == 0) {
    // unit u = token i * chunks + chunk c
    const int n_units = n_tok * a.chunks;
    bool ok = true;
    int issued = 0, u = 0;
    auto issue_load = [&](int u) {
      issued = u + 1;
      const int i = u / a.chunks, c = u - i * a.chunks;
      const int off = c * kChunkBytes;
      const int bytes = min(kChunkBytes, a.row_bytes - off);
      const int b = u % a.nbuf;
      bulk_load(smem_addr(bufs + (size_t)b * buf_bytes), a.x + (t0 + i) * a.row_bytes + off,
                (uint32_t)bytes, smem_addr(&s_bar[b]));
    };
    for (int v = 0; v < min(n_units, a.nbuf - 1); ++v) issue_load(v);
    for (; u < n_units; ++u) {
      const int b = u % a.nbuf;
      if (!mbar_wait_bounded(smem_addr(&s_bar[b]), (uint32_t)((u / a.nbuf) & 1))) {
        ok = false;
        break;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      const int i = u / a.chunks, c = u - i * a.chunks;
      const int off = c * kChunkBytes;
      const int bytes = min(kChunkBytes, a.row_bytes - off);
      const uint32_t sbuf = smem_addr(bufs + (size_t)b * buf_bytes);
      for (int j = 0; j < a.k; ++j) {
        const int row = s_perm[i * a.k + j];
        if (row < 0 || row >= a.rows_total) continue;  // dropped assignment
        bulk_store(a.recv + (int64_t)row * a.row_bytes + off, sbuf, (uint32_t)bytes);
      }
      bulk_commit();
      const int next = u + a.nbuf - 1;  // goes into the buffer of unit u - 1
      if (next < n_units) {
        bulk_wait_read_all_but_one();
        issue_load(next);
      }
    }
    bulk_wait_all();
    if (!ok) {
      // a load never completed: report it, and wait (bounded) for the other loads still in
      // flight, units u+1 .. issued-1, before the CTA's shared memory goes away
      atomicOr(const_cast<int32_t*>(a.err), MOE_DERR_TIMEOUT);
      for (int v = u + 1; v < issued; ++v)
        mbar_wait_bounded(smem_addr(&s_bar[v % a.nbuf]), (uint32_t)((v / a.nbuf) & 1));
    }
  } else if (tid >= 32 && a.counts != nullptr) {
    // fixed-capacity padding, by warps 1..7 (wt in [0, blockDim.x - 32)): experts
    // blockIdx.x, blockIdx.x + gridDim.x, ...; rows e*cap + [min(count, cap), cap)
    const int vec_per_row = a.row_bytes / 16;
    const int wt = tid - 32, nwt = blockDim.x - 32;
    for (int e = blockIdx.x; e < a.E; e += gridDim.x) {
      const int c = max(0, min(__ldg(a.counts + e), a.cap));
      const int64_t r0 = (int64_t)e * a.cap + c, r1 = (int64_t)(e + 1) * a.cap;
      for (int64_t r = r0 + wt; r < r1; r += nwt) a.src[r] = -1;
      const int64_t nvec = (r1 - r0) * vec_per_row;
      uint4* dst = reinterpret_cast<uint4*>(a.recv + r0 * a.row_bytes);
      for (int64_t v = wt; v < nvec; v += nwt) dst[v] = make_uint4(0, 0, 0, 0);
    }
  }
}

// The same row copy with generic 16-byte loads and stores: one warp per token reads its
// row once and stores it to each of its k rows (rows outside [0, rows_total), i.e.
// dropped assignments, are not stored).
constexpr int kRowVec = 4;

// Dst (rows.cuh): the receive rows on this GPU (LocalRows) or on every rank (RankRows).
template <class Dst>
__global__ void __launch_bounds__(kScatterThreads) scatter_warp_kernel(
    const uint4* __restrict__ x, const int32_t* __restrict__ perm, int T, int k, int dv,
    int64_t rows_total, const __grid_constant__ Dst recv, const int32_t* __restrict__ err) {
  if (load_err(err)) return;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T;
       t += nwarps) {
    int r = lane < k ? __ldg(perm + t * k + lane) : -1;
    if (r < 0 || r >= rows_total) r = -1;
    const uint4* xs = x + t * dv;
    for (int v0 = 0; v0 < dv; v0 += 32 * kRowVec) {
      uint4 buf[kRowVec];
#pragma unroll
      for (int u = 0; u < kRowVec; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < dv) buf[u] = __ldcs(xs + v);
      }
      for (int j = 0; j < k; ++j) {
        const int row = __shfl_sync(MOE_FULL_MASK, r, j);
        if (row < 0) continue;
        uint4* dst = recv.row(row, dv);
#pragma unroll
        for (int u = 0; u < kRowVec; ++u) {
          const int v = v0 + u * 32 + lane;
          if (v < dv) dst[v] = buf[u];
        }
      }
    }
  }
}

// Fixed-capacity padding rows e*cap + [min(count_e, cap), cap): zero rows, src -1.  One
// block per expert (grid-stride).
__global__ void __launch_bounds__(kScatterThreads) pad_rows_kernel(
    const int32_t* __restrict__ counts, int E, int cap, int row_bytes, uint8_t* __restrict__ recv,
    int32_t* __restrict__ src, const int32_t* __restrict__ err) {
  if (load_err(err)) return;
  const int vec_per_row = row_bytes / 16;
  for (int e = blockIdx.x; e < E; e += gridDim.x) {
    const int c = max(0, min(__ldg(counts + e), cap));
    const int64_t r0 = (int64_t)e * cap + c, r1 = (int64_t)(e + 1) * cap;
    for (int64_t r = r0 + threadIdx.x; r < r1; r += blockDim.x) src[r] = -1;
    const int64_t nvec = (r1 - r0) * vec_per_row;
    uint4* dst = reinterpret_cast<uint4*>(recv + r0 * row_bytes);
    for (int64_t v = threadIdx.x; v < nvec; v += blockDim.x) dst[v] = make_uint4(0, 0, 0, 0);
  }
}

// Which row copy the dispatch runs: the TMA ring from this many tokens per SM up, one warp
// per token below (measured on one B200, same box: near_balanced, ~28 tokens per SM, 44.1
// against 46.2 us with the ring; Qwen shape, ~55 per SM, 82.5 against 78.1 us; DeepSeek,
// ~111 per SM, 414 against 408 us alone and 450 against 441 us in the step).
constexpr int kTmaScatterMinTokensPerSm = 32;

int num_tiles(int T) { return (T + kRankTile - 1) / kRankTile; }

int launch_rank(const int32_t* idx, int T, int k, int E, int R, int C, int cap,
                const int32_t* plan, const moe_plan_layout* L, int32_t* ws, int32_t* perm,
                int32_t* src, int32_t* err, cudaStream_t s, const int32_t* q_base = nullptr) {
  const int ntiles = num_tiles(T);
  if (const int st = launch_zero(ws, ws_agg_off(ntiles), nullptr, 0, s); st != MOE_OK) return st;
  RankArgs a;
  a.idx = idx;
  a.T = T;
  a.k = k;
  a.E = E;
  a.R = R;
  a.C = C;
  a.cap = cap;
  a.plan = plan;
  a.q_base = q_base;
  if (L) a.L = *L;
  else memset(&a.L, 0, sizeof(a.L));
  a.ws = ws;
  a.ntiles = ntiles;
  a.perm = perm;
  a.src = src;
  a.err = err;
  const size_t smem = sizeof(int) * (size_t)rank_smem_words(E, R);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess)
    return MOE_ERR_LAUNCH;
  rank_kernel<<<ntiles, kRankTile, smem, s>>>(a);
  return launch_status();
}

int launch_scatter(const __nv_bfloat16* x, const int32_t* perm, int T, int k, int d,
                   int64_t rows_total, __nv_bfloat16* recv, const int32_t* counts, int E,
                   int cap, int32_t* src, const int32_t* err, cudaStream_t s) {
  if ((int64_t)T < (int64_t)kTmaScatterMinTokensPerSm * num_sms()) {
    if (T > 0) {
      const int64_t want = ((int64_t)T + 7) / 8;
      const int64_t capb = (int64_t)num_sms() * 8;
      scatter_warp_kernel<LocalRows><<<(int)(want < capb ? want : capb), kScatterThreads, 0, s>>>(
          reinterpret_cast<const uint4*>(x), perm, T, k, d / 8, rows_total,
          LocalRows{reinterpret_cast<uint4*>(recv)}, err);
      if (launch_status() != MOE_OK) return MOE_ERR_LAUNCH;
    }
    if (counts != nullptr) {
      pad_rows_kernel<<<num_sms(), kScatterThreads, 0, s>>>(
          counts, E, cap, d * 2, reinterpret_cast<uint8_t*>(recv), src, err);
      return launch_status();
    }
    return MOE_OK;
  }
  ScatterArgs a;
  a.x = reinterpret_cast<const uint8_t*>(x);
  a.perm = perm;
  a.T = T;
  a.k = k;
  a.row_bytes = d * 2;
  a.chunks = (a.row_bytes + kChunkBytes - 1) / kChunkBytes;
  const int sms = num_sms();
  a.tokens_per_cta = (T + sms - 1) / sms;
  if (a.tokens_per_cta > kMaxTokensPerCta) a.tokens_per_cta = kMaxTokensPerCta;
  if (a.tokens_per_cta < 1) a.tokens_per_cta = 1;
  int grid = (T + a.tokens_per_cta - 1) / a.tokens_per_cta;
  if (counts != nullptr && grid < sms) grid = sms;  // padding rows spread over every SM
  const int perm_bytes = ((a.tokens_per_cta * k * 4) + 127) / 128 * 128;
  const int buf_bytes = a.row_bytes < kChunkBytes ? a.row_bytes : kChunkBytes;
  const int budget = 200 * 1024 - perm_bytes;
  int nbuf = budget / buf_bytes;
  if (nbuf > kMaxBuf) nbuf = kMaxBuf;
  if (nbuf < 2) return MOE_ERR_SHAPE;  // cannot happen: buf_bytes <= 16 KiB, perm <= 32 KiB
  a.nbuf = nbuf;
  a.rows_total = rows_total;
  a.recv = reinterpret_cast<uint8_t*>(recv);
  a.counts = counts;
  a.E = E;
  a.cap = cap;
  a.src = src;
  a.err = err;
  const size_t smem = (size_t)perm_bytes + (size_t)nbuf * buf_bytes;
  if (cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_ERR_LAUNCH;
  scatter_kernel<<<grid, kScatterThreads, smem, s>>>(a);
  return launch_status();
}

}  // namespace

int64_t dispatch_workspace_words(int T, int E) {
  const int ntiles = num_tiles(T);
  return ws_incl_off(ntiles, E) + (int64_t)ntiles * E;
}

int launch_dispatch(const __nv_bfloat16* x, const int32_t* idx, const int32_t* plan,
                    const moe_plan_layout& L, int T, int k, int E, int R, int d,
                    int32_t* ws, __nv_bfloat16* recv, int32_t* perm, int32_t* src,
                    int32_t* err, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const int C = (int)(((int64_t)T * k) / R);
  const int st = launch_rank(idx, T, k, E, R, C, 0, plan, &L, ws, perm, src, err, s);
  if (st != MOE_OK || recv == nullptr) return st;  // index-only: the FFN gathers the rows
  return launch_scatter(x, perm, T, k, d, (int64_t)R * C, recv, nullptr, E, 0, nullptr, err, s);
}

int launch_ep_dispatch(const __nv_bfloat16* x, const int32_t* idx, const int32_t* q_base,
                       const int32_t* plan, const moe_plan_layout& L, int T, int k, int E,
                       int W, int d, int32_t* ws, __nv_bfloat16* const* recv_ranks,
                       int32_t* perm, int32_t* err, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const int C = T * k;  // every rank receives (W*T*k)/W rows
  const int st = launch_rank(idx, T, k, E, W, C, 0, plan, &L, ws, perm, nullptr, err, s, q_base);
  if (st != MOE_OK) return st;
  RankRows dst;
  for (int u = 0; u < MOE_EP_MAX_RANKS; ++u)
    dst.base[u] = u < W ? reinterpret_cast<uint4*>(recv_ranks[u]) : nullptr;
  dst.C = C;
  const int64_t want = ((int64_t)T + 7) / 8;
  const int64_t capb = (int64_t)num_sms() * 8;
  scatter_warp_kernel<RankRows><<<(int)(want < capb ? want : capb), kScatterThreads, 0, s>>>(
      reinterpret_cast<const uint4*>(x), perm, T, k, d / 8, (int64_t)W * C, dst, err);
  return launch_status();
}

int launch_dispatch_capacity(const __nv_bfloat16* x, const int32_t* idx, const int32_t* counts,
                             int T, int k, int E, int cap, int d, int32_t* ws,
                             __nv_bfloat16* recv, int32_t* perm, int32_t* src, int32_t* err,
                             cudaStream_t s) {
  if (T > 0) {
    const int st = launch_rank(idx, T, k, E, 1, 0, cap, nullptr, nullptr, ws, perm, src, err, s);
    if (st != MOE_OK) return st;
  }
  return launch_scatter(x, perm, T, k, d, (int64_t)E * cap, recv, counts, E, cap, src, err, s);
}

}  // namespace moe
