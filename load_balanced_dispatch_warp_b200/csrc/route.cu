// Router top-k and the demand histogram / maxvio.
//
// Top-k follows the router phase of "DeepEP-on-EFA Guidance, section 1: What is MoE":
// every expert is scored, the top-k are kept, and the gate weights form the routing
// table.  The histogram follows "MoE Load Balancing: Find Expert Hotspots", section
// "Separate expert demand from rank placement" (count by expert, then sum over an
// expert->rank map; balancedness = mean/max), with maxvio = (max - mean)/mean as named in
// the MoonEP news article.
#include "common.cuh"

namespace moe {
namespace {

// fp32 -> unsigned key whose unsigned order is the float order (finite values; -0 is
// folded onto +0 first so that equal logits compare equal).
__device__ __forceinline__ uint32_t order_key(float v) {
  v = (v == 0.0f) ? 0.0f : v;
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t key) {
  const uint32_t u = (key & 0x80000000u) ? (key & 0x7fffffffu) : ~key;
  return __uint_as_float(u);
}

// One warp per token.  Lane l holds experts l, l+32, ... (VPL of them) as
// order-preserving keys (pad entries e >= E: key 0, below every finite float).  Exact
// top-k in three steps:
//   1. tau = the k-th largest of the 32 lane maxima (k rounds of redux.sync over one
//      value per lane).  At least k keys are >= tau, so every key of the top-k -- equal
//      keys at the k-th place included -- is >= tau.
//   2. The keys >= tau (usually close to k of them) are compacted to one per lane
//      through shared memory.
//   3. k rounds over one candidate per lane: warp max key (redux.sync), lowest expert id
//      among its holders (redux.sync), the winner drops out.
// More than 32 candidates (many equal keys) falls back to the same rounds over all of
// the lane's keys.  BIASED: keys from logit + bias[e] (one fp32 add), gates from the
// chosen experts' unbiased logits (bias-only balancing).
// Expert held in slot i of a lane: lane + 32 i (scalar loads), or, with 16-byte loads
// (VEC), 128 (i / 4) + 4 lane + i % 4.
template <bool VEC>
__device__ __forceinline__ int slot_id(int i, int lane) {
  return VEC ? 128 * (i >> 2) + 4 * lane + (i & 3) : lane + 32 * i;
}

template <int VPL, bool BIASED, bool VEC>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits,
                                                   const float* __restrict__ bias, int T,
                                                   int E, int k, int32_t* __restrict__ idx,
                                                   float* __restrict__ gate,
                                                   int32_t* __restrict__ err) {
  __shared__ uint32_t s_key[8][32];
  __shared__ int s_id[8][32];
  __shared__ float s_raw[8][BIASED ? 32 : 1];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + wib; t < T; t += nwarps) {
  const float* row = logits + t * E;
  uint32_t key[VPL];
  float raw[BIASED ? VPL : 1];
  float val[VPL];
  if (VEC) {
#pragma unroll
    for (int q = 0; q < VPL / 4; ++q) {
      const int e0 = 128 * q + 4 * lane;
      float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e0 < E) v4 = __ldcs(reinterpret_cast<const float4*>(row + e0));
      val[4 * q] = v4.x;
      val[4 * q + 1] = v4.y;
      val[4 * q + 2] = v4.z;
      val[4 * q + 3] = v4.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      val[i] = e < E ? __ldcs(row + e) : 0.f;
    }
  }
  bool bad = false;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = slot_id<VEC>(i, lane);
    uint32_t kv = 0;
    if (e < E) {
      const float v = val[i];
      bad |= !isfinite(v);
      if (BIASED) {
        const float b = __ldg(bias + e);
        bad |= !isfinite(b);
        raw[i] = v;
        kv = order_key(__fadd_rn(v, b));
      } else {
        kv = order_key(v);
      }
    }
    key[i] = kv;
  }
  if (__any_sync(MOE_FULL_MASK, bad)) {
    if (lane == 0) atomicOr(err, MOE_DERR_NONFINITE);
    continue;
  }
  // 1. threshold from the lane maxima
  uint32_t lmax = key[0];
#pragma unroll
  for (int i = 1; i < VPL; ++i) lmax = max(lmax, key[i]);
  uint32_t tau = 0, m = lmax;
  for (int j = 0; j < k; ++j) {
    tau = __reduce_max_sync(MOE_FULL_MASK, m);
    const uint32_t holder = __reduce_min_sync(MOE_FULL_MASK, m == tau ? (uint32_t)lane : 32u);
    if ((uint32_t)lane == holder) m = 0;
  }
  // 2. candidates: keys >= tau (tau > 0: pad keys never qualify)
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
  float my_val = 0.f;
  int my_id = 0;
  if (total <= 32) {
    int pos = incl - cnt;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if (key[i] >= tau) {
        s_key[wib][pos] = key[i];
        s_id[wib][pos] = slot_id<VEC>(i, lane);
        if (BIASED) s_raw[wib][pos] = raw[i];
        ++pos;
      }
    }
    __syncwarp();
    uint32_t ck = lane < total ? s_key[wib][lane] : 0u;
    const int cid = lane < total ? s_id[wib][lane] : 0;
    const float craw = (BIASED && lane < total) ? s_raw[wib][BIASED ? lane : 0] : 0.f;
    // 3. k rounds over one candidate per lane
    for (int j = 0; j < k; ++j) {
      const uint32_t wmax = __reduce_max_sync(MOE_FULL_MASK, ck);
      const uint32_t wid =
          __reduce_min_sync(MOE_FULL_MASK, (ck == wmax && lane < total) ? (uint32_t)cid : 0xffffffffu);
      const bool mine = lane < total && (uint32_t)cid == wid;
      if (BIASED) {
        const uint32_t src = __reduce_min_sync(MOE_FULL_MASK, mine ? (uint32_t)lane : 32u);
        const float sel = __shfl_sync(MOE_FULL_MASK, craw, (int)src);
        if (lane == j) my_val = sel;
      } else if (lane == j) {
        my_val = key_value(wmax);
      }
      if (lane == j) my_id = (int)wid;
      if (mine) ck = 0;
    }
  } else {
    // many equal keys: rounds over all of the lane's keys
    for (int j = 0; j < k; ++j) {
      // lane's best: largest key, equal keys -> lowest expert id
      uint32_t best = key[0];
      int best_e = slot_id<VEC>(0, lane);
#pragma unroll
      for (int i = 1; i < VPL; ++i) {
        const int e = slot_id<VEC>(i, lane);
        const bool gt = key[i] > best || (key[i] == best && e < best_e);
        best = gt ? key[i] : best;
        best_e = gt ? e : best_e;
      }
      const uint32_t wmax = __reduce_max_sync(MOE_FULL_MASK, best);
      const uint32_t cand = best == wmax ? (uint32_t)best_e : 0xffffffffu;
      const uint32_t wid = __reduce_min_sync(MOE_FULL_MASK, cand);
      float sel = 0.f;
      bool mine = false;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const bool hit = slot_id<VEC>(i, lane) == (int)wid;
        mine |= hit;
        if (BIASED && hit) sel = raw[i];
        key[i] = hit ? 0u : key[i];
      }
      if (BIASED) {
        const uint32_t src = __reduce_min_sync(MOE_FULL_MASK, mine ? (uint32_t)lane : 32u);
        sel = __shfl_sync(MOE_FULL_MASK, sel, (int)src);
      }
      if (lane == j) {
        my_val = BIASED ? sel : key_value(wmax);
        my_id = (int)wid;
      }
    }
  }
  // softmax over the chosen (unbiased) logits
  float top = lane < k ? my_val : -INFINITY;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) top = fmaxf(top, __shfl_xor_sync(MOE_FULL_MASK, top, o));
  const float ex = lane < k ? expf(my_val - top) : 0.f;
  const float sum = warp_sum(ex);
  if (lane < k) {
    idx[t * k + lane] = my_id;
    gate[t * k + lane] = ex / sum;
  }
  __syncwarp();  // the warp's candidate buffer is rewritten by its next token
  }
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

// Per-block expert histogram over a contiguous token range, with the trace checks of the
// hotspot fixture (known ids, no expert repeated within a token).  Equal ids in a warp
// are merged with match.any before one shared-memory add; block totals go to global
// memory with integer atomics (order-independent, so deterministic).  The last block to
// finish (a ticket counter kept in loads[0], zeroed with counts before the launch and
// overwritten by the result) computes the rank loads under the expert->rank map and
// maxvio = (R*max - A)/A, balancedness = A/(R*max) from exact integers, one fp64 rounding
// each.
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
  if (threadIdx.x == 0 && s_err) atomicOr(err, s_err);
  // last block: every other block's counts are visible once its ticket is
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(loads, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
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

// One warp per token over a persistent grid (8 warps per block, up to 8 blocks per SM);
// 16-byte loads when every lane's slots come in aligned groups of four.
int launch_topk_impl(const float* logits, const float* bias, int T, int E, int k,
                     int32_t* idx, float* gate, int32_t* err, cudaStream_t s) {
  const int threads = 256, per_block = threads / 32;
  const int64_t want = ((int64_t)T + per_block - 1) / per_block;
  const int64_t cap = (int64_t)num_sms() * 8;
  const unsigned grid = (unsigned)(want < cap ? want : cap);
  const bool vec = E % 4 == 0 && (reinterpret_cast<uintptr_t>(logits) & 15u) == 0;
#define MOE_TOPK_CASE(V, VEC)                                                                  \
  (bias ? topk_kernel<V, true, VEC><<<grid, threads, 0, s>>>(logits, bias, T, E, k, idx, gate, err) \
        : topk_kernel<V, false, VEC><<<grid, threads, 0, s>>>(logits, bias, T, E, k, idx, gate, err))
  if (E <= 32) MOE_TOPK_CASE(1, false);
  else if (E <= 64) MOE_TOPK_CASE(2, false);
  else if (E <= 128) { if (vec) MOE_TOPK_CASE(4, true); else MOE_TOPK_CASE(4, false); }
  else if (E <= 256) { if (vec) MOE_TOPK_CASE(8, true); else MOE_TOPK_CASE(8, false); }
  else if (E <= 512) { if (vec) MOE_TOPK_CASE(16, true); else MOE_TOPK_CASE(16, false); }
  else { if (vec) MOE_TOPK_CASE(32, true); else MOE_TOPK_CASE(32, false); }
#undef MOE_TOPK_CASE
  return launch_status();
}

}  // namespace

int launch_topk(const float* logits, int T, int E, int k, int32_t* idx, float* gate,
                int32_t* err, cudaStream_t s) {
  if (cudaMemsetAsync(err, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_LAUNCH;
  if (T == 0) return MOE_OK;
  return launch_topk_impl(logits, nullptr, T, E, k, idx, gate, err, s);
}

int launch_topk_biased(const float* logits, const float* bias, int T, int E, int k,
                       int32_t* idx, float* gate, int32_t* err, cudaStream_t s) {
  if (cudaMemsetAsync(err, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_LAUNCH;
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
  if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s) != cudaSuccess ||
      cudaMemsetAsync(loads, 0, sizeof(int32_t), s) != cudaSuccess)
    return MOE_ERR_LAUNCH;
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

}  // namespace moe
