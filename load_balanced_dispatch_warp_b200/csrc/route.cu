// Router top-k and the demand histogram / maxvio.
//
// Top-k follows the router phase of "DeepEP-on-EFA Guidance, section 1: What is MoE":
// every expert is scored, the top-k are kept, and the gate weights form the routing
// table.  The histogram follows "MoE Load Balancing: Find Expert Hotspots", section
// "Separate expert demand from rank placement" (count by expert, then sum over an
// expert->rank map; balancedness = mean/max), with maxvio = (max - mean)/mean as named in
// the MoonEP news article.
#include "common.cuh"
#include "plan_body.cuh"

namespace moe {
namespace {

// fp32 -> unsigned key whose unsigned order is the float order (finite values; -0 is
// folded onto +0 first so that equal logits compare equal).
__device__ __forceinline__ uint32_t order_key(float v) {
  v = (v == 0.0f) ? 0.0f : v;
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The routing kernels are launched as programmatic dependents of the small kernel that
// zeroes the error word (and the routing workspace): they start while it finishes, and
// wait for it (griddepcontrol.wait: the reset grid complete, its stores visible) only
// before their first write to a word it zeroes.  Without that launch attribute the wait
// returns at once.
__device__ __forceinline__ void wait_for_reset() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Warp-wide fp32 maximum (one instruction on sm_100a).
__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// Exact top-k of one token over order keys, the general procedure (any ties).  Lane l
// holds experts l, l+32, ... (VPL of them) as raw logits x and, when BIASED, biases b;
// pad entries (expert >= E) get key 0, below every finite float.  Three steps:
//   1. tau = the k-th largest of the 32 lane maxima (k rounds over one key per lane).
//      At least k keys are >= tau, so every key of the top-k -- equal keys at the k-th
//      place included -- is >= tau.
//   2. The keys >= tau are compacted to one per lane through shared memory.
//   3. k rounds over one candidate per lane: warp max key, lowest expert id among its
//      holders, the winner drops out.
// More than 32 candidates (many equal keys) runs the rounds over all of the lane's keys.
// On return lane j < k holds the j-th choice: its expert id and its unbiased logit.  The
// token's logits (row) and the biases are read again here rather than handed over from the
// caller's registers: an array passed by address would live in local memory, and the
// caller would store every token's row there although only a few tokens come here.
template <int VPL, bool BIASED>
__device__ __noinline__ void topk_exact(const float* __restrict__ row,
                                        const float* __restrict__ bias, int E, int k, int lane,
                                        uint32_t* s_key, int* s_id, float* s_raw,
                                        float& my_val, int& my_id) {
  float x[VPL], b[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    x[i] = e < E ? row[e] : 0.f;
    b[i] = (BIASED && e < E) ? __ldg(bias + e) : 0.f;
  }
  uint32_t key[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    key[i] = e < E ? order_key(BIASED ? __fadd_rn(x[i], b[i]) : x[i]) : 0u;
  }
  uint32_t lmax = key[0];
#pragma unroll
  for (int i = 1; i < VPL; ++i) lmax = max(lmax, key[i]);
  uint32_t tau = 0, m = lmax;
  for (int j = 0; j < k; ++j) {
    tau = __reduce_max_sync(MOE_FULL_MASK, m);
    const uint32_t holder = __reduce_min_sync(MOE_FULL_MASK, m == tau ? (uint32_t)lane : 32u);
    if ((uint32_t)lane == holder) m = 0;
  }
  int cnt = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) cnt += key[i] >= tau;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(MOE_FULL_MASK, incl, o);
    if (lane >= o) incl += v;
  }
  const int total = __shfl_sync(MOE_FULL_MASK, incl, 31);
  my_val = 0.f;
  my_id = 0;
  if (total <= 32) {
    int pos = incl - cnt;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if (key[i] >= tau) {
        s_key[pos] = key[i];
        s_id[pos] = lane + 32 * i;
        s_raw[pos] = x[i];
        ++pos;
      }
    }
    __syncwarp();
    uint32_t ck = lane < total ? s_key[lane] : 0u;
    const int cid = lane < total ? s_id[lane] : 0;
    const float craw = lane < total ? s_raw[lane] : 0.f;
    for (int j = 0; j < k; ++j) {
      const uint32_t wmax = __reduce_max_sync(MOE_FULL_MASK, ck);
      const uint32_t wid = __reduce_min_sync(
          MOE_FULL_MASK, (ck == wmax && lane < total) ? (uint32_t)cid : 0xffffffffu);
      const bool mine = lane < total && (uint32_t)cid == wid;
      const uint32_t src = __reduce_min_sync(MOE_FULL_MASK, mine ? (uint32_t)lane : 32u);
      const float sel = __shfl_sync(MOE_FULL_MASK, craw, (int)src);
      if (lane == j) {
        my_val = sel;
        my_id = (int)wid;
      }
      if (mine) ck = 0;
    }
    __syncwarp();  // the candidate buffer is rewritten by the warp's next call
  } else {
    for (int j = 0; j < k; ++j) {
      // lane's best: largest key, equal keys -> lowest expert id (= lowest slot)
      uint32_t best = key[0];
      int best_i = 0;
#pragma unroll
      for (int i = 1; i < VPL; ++i) {
        const bool gt = key[i] > best;
        best = gt ? key[i] : best;
        best_i = gt ? i : best_i;
      }
      const uint32_t wmax = __reduce_max_sync(MOE_FULL_MASK, best);
      const uint32_t cand = best == wmax ? (uint32_t)(lane + 32 * best_i) : 0xffffffffu;
      const uint32_t wid = __reduce_min_sync(MOE_FULL_MASK, cand);
      float sel = 0.f;
      bool mine = false;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const bool hit = lane + 32 * i == (int)wid;
        mine |= hit;
        if (hit) sel = x[i];
        key[i] = hit ? 0u : key[i];
      }
      const uint32_t src = __reduce_min_sync(MOE_FULL_MASK, mine ? (uint32_t)lane : 32u);
      sel = __shfl_sync(MOE_FULL_MASK, sel, (int)src);
      if (lane == j) {
        my_val = sel;
        my_id = (int)wid;
      }
    }
  }
}

// One warp per token; lane l holds experts l, l+32, ... (VPL of them), so neighbouring
// experts sit in different lanes.  Fast path, exact whenever it is taken:
//   - each lane keeps its two largest keys h1 >= h2 (a multiset: equal keys count twice);
//   - k rounds: w = warp max of the lane heads; every lane whose head equals w pops it
//     (head <- h2, then -inf) and notes the round in a bit mask;
//   - the rounds are the top-k, in order, iff exactly k pops happened in total and every
//     lane holds exactly as many keys >= w_last as it popped.  Then the popped keys are
//     precisely the keys >= w_last, k of them; one pop per round means no two lanes ever
//     held equal keys at the top, and two equal keys of one lane pop in consecutive
//     rounds, the lower slot (= lower expert id) first.
// Otherwise (equal keys across lanes, a lane holding three of the top-k, overflow to
// -inf) the warp runs topk_exact on the same registers.  Gates: softmax over the chosen
// experts' unbiased logits in fp32.  K > 0 fixes k at compile time (K == k).
// Token t by the calling warp.  Returns false (err flagged, nothing written) on a
// non-finite logit or bias.  COUNT: each written id is also added to counts[id].
// Lane's share of token t's logits: x[i] = logits[t, lane + 32 i] (0 past E).
template <int VPL, bool FULL>
__device__ __forceinline__ void load_row(const float* __restrict__ logits, int64_t t, int E,
                                         int lane, float (&x)[VPL]) {
  const float* row = logits + t * E;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    x[i] = (FULL || e < E) ? __ldcs(row + e) : 0.f;
  }
}

// The selection for token t from the lane's share x of its logits (load_row).  FULL: E is
// exactly 32 * VPL, so no lane holds a slot past the last expert.
template <int VPL, int K, bool BIASED, bool COUNT, bool FULL = false>
__device__ __forceinline__ bool topk_token_loaded(const float (&x)[VPL],
                                                  const float* __restrict__ row,
                                                  const float* __restrict__ bias, int64_t t,
                                                  int E, int k, int lane, uint32_t* s_key,
                                                  int* s_id, float* s_raw,
                                                  int32_t* __restrict__ idx,
                                                  float* __restrict__ gate,
                                                  int32_t* __restrict__ counts,
                                                  int32_t* __restrict__ err) {
  float b[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) b[i] = 0.f;
  if (BIASED) {
    bool bad = false;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      b[i] = e < E ? __ldg(bias + e) : 0.f;
      bad |= !isfinite(b[i]);
    }
    if (__any_sync(MOE_FULL_MASK, bad)) {
      if (lane == 0) {
        wait_for_reset();
        atomicOr(err, MOE_DERR_NONFINITE);
      }
      return false;
    }
  }
  // non-finite check: x * 0 is +-0 for finite x and NaN otherwise
  float key[VPL];
  float z = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    z = __fmaf_rn(x[i], 0.f, z);
    key[i] = (FULL || lane + 32 * i < E) ? (BIASED ? __fadd_rn(x[i], b[i]) : x[i]) : -INFINITY;
  }
  if (__any_sync(MOE_FULL_MASK, !(z == 0.f))) {
    if (lane == 0) {
      wait_for_reset();
      atomicOr(err, MOE_DERR_NONFINITE);
    }
    return false;
  }
  float h1 = key[0], h2 = -INFINITY;
#pragma unroll
  for (int i = 1; i < VPL; ++i) {
    h2 = fmaxf(h2, fminf(h1, key[i]));
    h1 = fmaxf(h1, key[i]);
  }
  float head = h1, nxt = h2, w0 = -INFINITY, tau = -INFINITY;
  uint32_t won = 0;
#pragma unroll
  for (int j = 0; j < (K > 0 ? K : 32); ++j) {
    if (K == 0 && j >= k) break;
    const float w = warp_max_f32(head);
    if (j == 0) w0 = w;
    const bool eq = head == w;
    won |= eq ? (1u << j) : 0u;
    head = eq ? nxt : head;
    nxt = eq ? -INFINITY : nxt;
    tau = w;
  }
  const int npop = __popc(won);
  uint32_t m_tau = 0, m_h1 = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    m_tau |= key[i] >= tau ? (1u << i) : 0u;
    m_h1 |= key[i] >= h1 ? (1u << i) : 0u;
  }
  const int total = (int)__reduce_add_sync(MOE_FULL_MASK, (unsigned)npop);
  const bool fast = __all_sync(MOE_FULL_MASK, __popc(m_tau) == npop) && total == k &&
                    tau > -INFINITY;
  if (fast) {
    // slots of the popped keys: s1 holds h1 (lowest slot among equal keys), s2 the other
    const int s1 = __ffs(m_h1) - 1;
    const int s2 = __ffs(m_tau & ~(1u << (s1 & 31))) - 1;
    const int r1 = __ffs(won) - 1;
    const int r2 = __ffs(won & (won - 1u)) - 1;
    float v1 = h1, v2 = h2;
    if (BIASED) {
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        v1 = i == s1 ? x[i] : v1;
        v2 = i == s2 ? x[i] : v2;
      }
    }
    const float top =
        BIASED ? warp_max_f32(npop > 0 ? fmaxf(v1, npop > 1 ? v2 : -INFINITY) : -INFINITY) : w0;
    const float e1 = npop > 0 ? expf(v1 - top) : 0.f;
    const float e2 = npop > 1 ? expf(v2 - top) : 0.f;
    const float inv = 1.f / warp_sum(e1 + e2);
    if (npop > 0) {
      idx[t * k + r1] = lane + 32 * s1;
      gate[t * k + r1] = e1 * inv;
      if (COUNT) atomicAdd(counts + lane + 32 * s1, 1);
    }
    if (npop > 1) {
      idx[t * k + r2] = lane + 32 * s2;
      gate[t * k + r2] = e2 * inv;
      if (COUNT) atomicAdd(counts + lane + 32 * s2, 1);
    }
    return true;
  }
  float my_val;
  int my_id;
  topk_exact<VPL, BIASED>(row, bias, E, k, lane, s_key, s_id, s_raw, my_val, my_id);
  float top = lane < k ? my_val : -INFINITY;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) top = fmaxf(top, __shfl_xor_sync(MOE_FULL_MASK, top, o));
  const float ex = lane < k ? expf(my_val - top) : 0.f;
  const float sum = warp_sum(ex);
  if (lane < k) {
    idx[t * k + lane] = my_id;
    gate[t * k + lane] = ex / sum;
    if (COUNT) atomicAdd(counts + my_id, 1);
  }
  return true;
}

template <int VPL, int K, bool BIASED, bool COUNT, bool FULL = false>
__device__ __forceinline__ bool topk_token(const float* __restrict__ logits,
                                           const float* __restrict__ bias, int64_t t, int E,
                                           int k, int lane, uint32_t* s_key, int* s_id,
                                           float* s_raw, int32_t* __restrict__ idx,
                                           float* __restrict__ gate, int32_t* __restrict__ counts,
                                           int32_t* __restrict__ err) {
  float x[VPL];
  load_row<VPL, FULL>(logits, t, E, lane, x);
  return topk_token_loaded<VPL, K, BIASED, COUNT, FULL>(x, logits + t * E, bias, t, E, k, lane,
                                                        s_key, s_id, s_raw, idx, gate, counts,
                                                        err);
}

// Warps (tokens) per block of the stand-alone top-k.
constexpr int kTopkWarps = 8;

template <int VPL, int K, bool BIASED, bool FULL = false>
__global__ void __launch_bounds__(kTopkWarps * 32) topk_kernel(const float* __restrict__ logits,
                                                   const float* __restrict__ bias, int T,
                                                   int E, int k_rt, int32_t* __restrict__ idx,
                                                   float* __restrict__ gate,
                                                   int32_t* __restrict__ err) {
  __shared__ uint32_t s_key[kTopkWarps][32];
  __shared__ int s_id[kTopkWarps][32];
  __shared__ float s_raw[kTopkWarps][32];
  const int k = K > 0 ? K : k_rt;
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t t = (int64_t)blockIdx.x * kTopkWarps + wib;
  if (t >= T) return;
  topk_token<VPL, K, BIASED, false, FULL>(logits, bias, t, E, k, lane, s_key[wib], s_id[wib],
                                          s_raw[wib], idx, gate, nullptr, err);
  // no block ends before the reset grid has (warp 0 of every block has a token), so the
  // work that follows this grid on the stream also follows the reset
  wait_for_reset();
}

// Fixed-capacity ledger of "MoE Load Balancing: Find Expert Hotspots" ("Make expert
// capacity, overflow, and padding explicit"): cap = ceil(A * cf / E) with the capacity
// factor an exact rational cf_num / cf_den; per expert processed = min(count, cap),
// overflow = max(count - cap, 0), padding = max(cap - count, 0); totals =
// {cap, sum processed, sum overflow, sum padding}.  One CTA, integer arithmetic.
__global__ void __launch_bounds__(256) capacity_kernel(const int32_t* __restrict__ counts, int E,
                                                       long long A, int cf_num, int cf_den,
                                                       int32_t* __restrict__ processed,
                                                       int32_t* __restrict__ overflow,
                                                       int32_t* __restrict__ padding,
                                                       int32_t* __restrict__ totals,
                                                       const int32_t* __restrict__ err) {
  __shared__ long long s_sum[3][8];
  if (block_should_stop(err)) return;
  const long long num = A * cf_num, den = (long long)E * cf_den;
  const long long cap = (num + den - 1) / den;
  long long sp = 0, so = 0, sd = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const long long c = counts[e];
    const long long p = c < cap ? c : cap;
    const long long o = c > cap ? c - cap : 0;
    const long long d = cap > c ? cap - c : 0;
    processed[e] = (int32_t)p;
    overflow[e] = (int32_t)o;
    padding[e] = (int32_t)d;
    sp += p;
    so += o;
    sd += d;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sp += __shfl_xor_sync(MOE_FULL_MASK, sp, o);
    so += __shfl_xor_sync(MOE_FULL_MASK, so, o);
    sd += __shfl_xor_sync(MOE_FULL_MASK, sd, o);
  }
  if ((threadIdx.x & 31) == 0) {
    s_sum[0][threadIdx.x >> 5] = sp;
    s_sum[1][threadIdx.x >> 5] = so;
    s_sum[2][threadIdx.x >> 5] = sd;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    long long a = 0, b = 0, c = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
      a += s_sum[0][w];
      b += s_sum[1][w];
      c += s_sum[2][w];
    }
    totals[0] = (int32_t)cap;
    totals[1] = (int32_t)a;
    totals[2] = (int32_t)b;
    totals[3] = (int32_t)c;
  }
}

// Last block of a histogram: the rank loads of `counts` under the expert->rank map
// (nullptr: e / (E/R)), maxvio = (R*max - A)/A and balancedness = A/(R*max) from exact
// integers, one fp64 rounding each.  s_hist: R ints of shared memory; s_max: 32 ints.
__device__ __noinline__ void hist_finish(const int32_t* __restrict__ counts, int T, int k, int E,
                                         int R, const int32_t* __restrict__ map,
                                         int32_t* __restrict__ loads, double* __restrict__ maxvio,
                                         double* __restrict__ bal, int32_t* __restrict__ err,
                                         int* s_hist, int* s_max) {
  const int lane = threadIdx.x & 31;
  const int B = E / R;
  for (int r = threadIdx.x; r < R; r += blockDim.x) s_hist[r] = 0;
  __syncthreads();
  int bad = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int r = map ? __ldg(map + e) : e / B;
    if (r < 0 || r >= R) {
      bad = 1;
    } else {
      const int c = __ldcg(counts + e);
      if (c) atomicAdd(&s_hist[r], c);
    }
  }
  if (bad) atomicOr(err, MOE_DERR_ID_RANGE);
  __syncthreads();
  int mx = 0;
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    loads[r] = s_hist[r];
    mx = max(mx, s_hist[r]);
  }
  mx = __reduce_max_sync(MOE_FULL_MASK, mx);
  if (lane == 0) s_max[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    const int nw = (blockDim.x + 31) >> 5;
    int v = threadIdx.x < nw ? s_max[threadIdx.x] : 0;
    v = __reduce_max_sync(MOE_FULL_MASK, v);
    if (threadIdx.x == 0) {
      const long long A = (long long)T * k;
      const long long top = (long long)R * v;
      if (A == 0 || v == 0) {
        *maxvio = 0.0;
        *bal = 1.0;
      } else {
        *maxvio = (double)(top - A) / (double)A;
        *bal = (double)A / (double)top;
      }
    }
  }
}

// Per-block expert histogram over a contiguous token range, with the trace checks of the
// hotspot fixture (known ids, no expert repeated within a token).  Equal ids in a warp
// are merged with match.any before one shared-memory add; block totals go to global
// memory with integer atomics (order-independent, so deterministic).  The last block to
// finish computes the rank loads under the expert->rank map and maxvio = (R*max - A)/A,
// balancedness = A/(R*max) from exact integers, one fp64 rounding each.
//
// The ticket word is loads[0] (zeroed before the launch, overwritten by the result): its
// low 24 bits count finished blocks (at most 2 per SM) and bits 24.. carry the trace
// errors the blocks found (kErrShift).  No block writes *err before the last one
// publishes those bits, so every block's entry check reads the word as it was before the
// launch and the whole grid takes the same decision; every block counts all of its
// in-range ids whatever the others found, so counts and error bits do not depend on
// block scheduling.
constexpr int kErrShift = 24;
constexpr int kTicketMask = (1 << kErrShift) - 1;

__global__ void __launch_bounds__(512) hist_kernel(const int32_t* __restrict__ idx, int T, int k,
                                                   int E, int R, int tokens_per_block,
                                                   const int32_t* __restrict__ map,
                                                   int32_t* __restrict__ counts,
                                                   int32_t* __restrict__ loads,
                                                   double* __restrict__ maxvio,
                                                   double* __restrict__ bal,
                                                   int32_t* __restrict__ err) {
  extern __shared__ int s_hist[];  // [max(E, R)]
  __shared__ int s_err, s_last, s_max[32];
  if (block_should_stop(err)) return;
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
  if (threadIdx.x == 0) s_err = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t t0 = (int64_t)blockIdx.x * tokens_per_block;
  const int64_t t1 = min((int64_t)T, t0 + tokens_per_block);
  int my_err = 0;
  for (int64_t base = t0; base < t1; base += blockDim.x) {
    const int64_t t = base + threadIdx.x;
    const bool tok = t < t1;
    for (int j = 0; j < k; ++j) {
      int e = tok ? __ldg(idx + t * k + j) : -1;
      if (tok) {
        if (e < 0 || e >= E) {
          my_err |= MOE_DERR_ID_RANGE;
          e = -1;
        } else {
          for (int i = 0; i < j; ++i)
            if (__ldg(idx + t * k + i) == e) my_err |= MOE_DERR_DUPLICATE;
        }
      }
      const uint32_t peers = __match_any_sync(MOE_FULL_MASK, e);
      if (e >= 0 && lane == __ffs(peers) - 1) atomicAdd(&s_hist[e], __popc(peers));
    }
  }
  if (my_err) atomicOr(&s_err, my_err);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (s_hist[e]) atomicAdd(counts + e, s_hist[e]);
  // last block: every other block's counts and error bits are visible once its ticket is
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    if (s_err) atomicOr(loads, s_err << kErrShift);
    const int old = atomicAdd(loads, 1);
    s_last = (old & kTicketMask) == (int)gridDim.x - 1;
    if (s_last) s_err = (old >> kErrShift) | s_err;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (threadIdx.x == 0 && s_err) atomicOr(err, s_err);
  hist_finish(counts, T, k, E, R, map, loads, maxvio, bal, err, s_hist, s_max);
}

// Launch of a routing kernel right after launch_zero on the same stream, as its
// programmatic dependent (see wait_for_reset).
template <typename... Params, typename... Args>
void launch_after_reset(void (*kernel)(Params...), unsigned grid, unsigned block, size_t smem,
                        cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(block, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, static_cast<Params>(args)...);  // status: launch_status()
}

// One warp per token, 8 warps per block.  Unbiased calls with k in {2, 4, 6, 8} and up to
// 256 experts run a kernel with k fixed at compile time (the rounds unroll).
template <int VPL>
void launch_topk_vpl(const float* logits, const float* bias, int T, int E, int k, int32_t* idx,
                     float* gate, int32_t* err, cudaStream_t s) {
  const unsigned grid = (unsigned)(((int64_t)T + kTopkWarps - 1) / kTopkWarps);
#define MOE_TOPK(KK, B) launch_after_reset(topk_kernel<VPL, KK, B>, grid, kTopkWarps * 32, 0, s, logits, bias, T, E, k, idx, gate, err)
  if (bias) {
    MOE_TOPK(0, true);
    return;
  }
  if constexpr (VPL <= 8) {
    if (E == 32 * VPL) {
#define MOE_TOPK_FULL(KK) launch_after_reset(topk_kernel<VPL, KK, false, true>, grid, kTopkWarps * 32, 0, s, logits, bias, T, E, k, idx, gate, err)
      switch (k) {
        case 8: MOE_TOPK_FULL(8); return;
        case 6: MOE_TOPK_FULL(6); return;
        case 4: MOE_TOPK_FULL(4); return;
        case 2: MOE_TOPK_FULL(2); return;
        default: break;
      }
#undef MOE_TOPK_FULL
    }
    switch (k) {
      case 8: MOE_TOPK(8, false); return;
      case 6: MOE_TOPK(6, false); return;
      case 4: MOE_TOPK(4, false); return;
      case 2: MOE_TOPK(2, false); return;
      default: break;
    }
  }
  MOE_TOPK(0, false);
#undef MOE_TOPK
}

int launch_topk_impl(const float* logits, const float* bias, int T, int E, int k,
                     int32_t* idx, float* gate, int32_t* err, cudaStream_t s) {
  if (E <= 32) launch_topk_vpl<1>(logits, bias, T, E, k, idx, gate, err, s);
  else if (E <= 64) launch_topk_vpl<2>(logits, bias, T, E, k, idx, gate, err, s);
  else if (E <= 128) launch_topk_vpl<4>(logits, bias, T, E, k, idx, gate, err, s);
  else if (E <= 256) launch_topk_vpl<8>(logits, bias, T, E, k, idx, gate, err, s);
  else if (E <= 512) launch_topk_vpl<16>(logits, bias, T, E, k, idx, gate, err, s);
  else launch_topk_vpl<32>(logits, bias, T, E, k, idx, gate, err, s);
  return launch_status();
}


// Routing, histogram and plan in one launch (the three calls' outputs, bit for bit).  Every
// block runs top-k for its 8 tokens, counting the chosen ids in shared memory, then adds its
// non-zero counts to one of kCountCopies partial histograms in `ws` (copy = block index
// mod kCountCopies: integer atomics, order-independent, spread over the copies so that no
// counter takes more than a 1/kCountCopies share of the blocks).  The last block to finish
// (ticket in ws[kCountCopies * E]; ws zeroed before the launch) sums the copies into
// counts, computes the home-map rank loads, maxvio and balancedness, then the plan.  After
// a non-finite logit it leaves what the separate calls leave: counts and loads[0] zero, the
// rest untouched.
constexpr int kCountCopies = 16;

template <int VPL, int K, bool BIASED, bool FULL = false>
__global__ void __launch_bounds__(kPlanThreads) route_plan_kernel(
    const float* __restrict__ logits, const float* __restrict__ bias, int T, int E, int k_rt,
    int R, int S, int32_t* __restrict__ idx, float* __restrict__ gate,
    int32_t* __restrict__ counts, int32_t* __restrict__ loads, double* __restrict__ maxvio,
    double* __restrict__ bal, int32_t* __restrict__ plan, const moe_plan_layout L,
    int32_t* __restrict__ ws, int32_t* __restrict__ err) {
  static_assert(kPlanThreads == 256, "8 tokens per block, one warp each");
  __shared__ uint32_t s_key[8][32];
  __shared__ int s_id[8][32];
  __shared__ float s_raw[8][32];
  // [0, E): this block's counts, later the last block's rank loads; then the plan's words
  extern __shared__ int s_dyn[];
  __shared__ int s_max[32];
  __shared__ int s_last;
  const int k = K > 0 ? K : k_rt;
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_dyn[e] = 0;
  __syncthreads();
  const int64_t t = (int64_t)blockIdx.x * 8 + wib;
  if (t < T)
    topk_token<VPL, K, BIASED, true, FULL>(logits, bias, t, E, k, lane, s_key[wib], s_id[wib],
                                           s_raw[wib], idx, gate, s_dyn, err);
  __syncthreads();
  wait_for_reset();  // ws and err zeroed
  int32_t* copy = ws + (int64_t)(blockIdx.x % kCountCopies) * E;
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (s_dyn[e]) atomicAdd(copy + e, s_dyn[e]);
  // last block: every other block's counts are visible once its ticket is
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(ws + kCountCopies * E, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (load_err(err) != 0) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = 0;
    if (threadIdx.x == 0) loads[0] = 0;
    return;
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
#pragma unroll 4
    for (int p = 0; p < kCountCopies; ++p) c += __ldcg(ws + (int64_t)p * E + e);
    counts[e] = c;
  }
  __threadfence_block();
  __syncthreads();
  hist_finish(counts, T, k, E, R, nullptr, loads, maxvio, bal, err, s_dyn, s_max);
  __syncthreads();
  plan_block(counts, T, k, E, R, S, plan, L, err, s_dyn + E);
}

template <int VPL>
void launch_route_plan_vpl(const float* logits, const float* bias, int T, int E, int k, int R,
                           int S, int32_t* idx, float* gate, int32_t* counts, int32_t* loads,
                           double* maxvio, double* bal, int32_t* plan, const moe_plan_layout& L,
                           int32_t* ws, int32_t* err, cudaStream_t s) {
  const unsigned grid = T > 0 ? (unsigned)(((int64_t)T + 7) / 8) : 1u;
  const size_t smem = sizeof(int) * (size_t)(E + plan_smem_words(E, R));
#define MOE_RP(KK, B)                                                                           \
  launch_after_reset(route_plan_kernel<VPL, KK, B>, grid, kPlanThreads, smem, s, logits, bias, T, \
                     E, k, R, S, idx, gate, counts, loads, maxvio, bal, plan, L, ws, err)
  if (bias) {
    MOE_RP(0, true);
    return;
  }
  if constexpr (VPL <= 8) {
    if (E == 32 * VPL) {
#define MOE_RP_FULL(KK)                                                                         \
  launch_after_reset(route_plan_kernel<VPL, KK, false, true>, grid, kPlanThreads, smem, s, logits, \
                     bias, T, E, k, R, S, idx, gate, counts, loads, maxvio, bal, plan, L, ws, err)
      switch (k) {
        case 8: MOE_RP_FULL(8); return;
        case 6: MOE_RP_FULL(6); return;
        case 4: MOE_RP_FULL(4); return;
        case 2: MOE_RP_FULL(2); return;
        default: break;
      }
#undef MOE_RP_FULL
    }
    switch (k) {
      case 8: MOE_RP(8, false); return;
      case 6: MOE_RP(6, false); return;
      case 4: MOE_RP(4, false); return;
      case 2: MOE_RP(2, false); return;
      default: break;
    }
  }
  MOE_RP(0, false);
#undef MOE_RP
}

__global__ void __launch_bounds__(256) zero_kernel(int32_t* __restrict__ a, int64_t na,
                                                   int32_t* __restrict__ b, int64_t nb) {
  // a dependent launched with programmatic serialisation may start now; it waits for this
  // grid's completion (griddepcontrol.wait) before touching a or b
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < na + nb; i += stride) {
    if (i < na) a[i] = 0;
    else b[i - na] = 0;
  }
}

}  // namespace

int launch_zero(int32_t* a, int64_t na, int32_t* b, int64_t nb, cudaStream_t s) {
  const int64_t n = na + nb;
  if (n <= 0) return MOE_OK;
  const int64_t want = (n + 255) / 256;
  const int grid = (int)(want < (int64_t)num_sms() * 4 ? want : (int64_t)num_sms() * 4);
  zero_kernel<<<grid, 256, 0, s>>>(a, na, b, nb);
  return launch_status();
}

int launch_topk(const float* logits, int T, int E, int k, int32_t* idx, float* gate,
                int32_t* err, cudaStream_t s) {
  if (const int st = launch_zero(err, 1, nullptr, 0, s); st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  return launch_topk_impl(logits, nullptr, T, E, k, idx, gate, err, s);
}

int launch_topk_biased(const float* logits, const float* bias, int T, int E, int k,
                       int32_t* idx, float* gate, int32_t* err, cudaStream_t s) {
  if (const int st = launch_zero(err, 1, nullptr, 0, s); st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  return launch_topk_impl(logits, bias, T, E, k, idx, gate, err, s);
}

int launch_capacity(const int32_t* counts, int E, long long A, int cf_num, int cf_den,
                    int32_t* processed, int32_t* overflow, int32_t* padding, int32_t* totals,
                    const int32_t* err, cudaStream_t s) {
  capacity_kernel<<<1, 256, 0, s>>>(counts, E, A, cf_num, cf_den, processed, overflow, padding,
                                    totals, err);
  return launch_status();
}

int launch_histogram(const int32_t* idx, int T, int k, int E, int R, const int32_t* map,
                     int32_t* counts, int32_t* loads, double* maxvio, double* bal,
                     int32_t* err, cudaStream_t s) {
  if (const int st = launch_zero(counts, E, loads, 1, s); st != MOE_OK) return st;
  const int threads = 512;
  // about two blocks per SM, each over a contiguous token range (one block when T == 0)
  int blocks = 2 * num_sms();
  int per = (T + blocks - 1) / blocks;
  per = ((per + 31) / 32) * 32;
  if (per == 0) per = 32;
  blocks = T > 0 ? (T + per - 1) / per : 1;
  const size_t smem = sizeof(int) * (size_t)(E > R ? E : R);
  hist_kernel<<<blocks, threads, smem, s>>>(idx, T, k, E, R, per, map, counts, loads, maxvio, bal, err);
  return launch_status();
}

int64_t route_plan_workspace_words(int E) { return (int64_t)kCountCopies * E + 1; }

int launch_route_plan(const float* logits, const float* bias, int T, int E, int k, int R,
                      int S, int32_t* idx, float* gate, int32_t* counts, int32_t* loads,
                      double* maxvio, double* bal, int32_t* plan, const moe_plan_layout& L,
                      int32_t* ws, int32_t* err, cudaStream_t s) {
  if (const int st = launch_zero(err, 1, ws, route_plan_workspace_words(E), s); st != MOE_OK) return st;
#define MOE_RP_VPL(V) \
  launch_route_plan_vpl<V>(logits, bias, T, E, k, R, S, idx, gate, counts, loads, maxvio, bal, plan, L, ws, err, s)
  if (E <= 32) MOE_RP_VPL(1);
  else if (E <= 64) MOE_RP_VPL(2);
  else if (E <= 128) MOE_RP_VPL(4);
  else if (E <= 256) MOE_RP_VPL(8);
  else if (E <= 512) MOE_RP_VPL(16);
  else MOE_RP_VPL(32);
#undef MOE_RP_VPL
  return launch_status();
}

}  // namespace moe
