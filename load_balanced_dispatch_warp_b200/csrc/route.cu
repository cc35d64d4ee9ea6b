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
// order-preserving keys; pad entries (e >= E) and taken entries have key 0, below every
// finite float, so each of the k rounds is a plain max over the lane's keys, a warp-wide
// max key (redux.sync), the lowest expert id among the lanes holding it (redux.sync), and
// the winner zeroes that key.  Instruction count, not memory, bounds this kernel.
// BIASED: keys are built from logit + bias[e] (one fp32 add), the gates from the chosen
// experts' unbiased logits (bias-only balancing).
template <int VPL, bool BIASED>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits,
                                                   const float* __restrict__ bias, int T,
                                                   int E, int k, int32_t* __restrict__ idx,
                                                   float* __restrict__ gate,
                                                   int32_t* __restrict__ err) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* row = logits + t * E;
  uint32_t key[VPL];
  float raw[BIASED ? VPL : 1];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    uint32_t kv = 0;
    if (e < E) {
      const float v = __ldcs(row + e);
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
    return;
  }
  float my_val = 0.f;
  int my_id = 0;
  for (int j = 0; j < k; ++j) {
    // lane maximum; equal keys keep the lower slot (= lower expert id)
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
    const bool mine = (int)(wid & 31u) == lane;
    const int wi = (int)(wid >> 5);
    float sel = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if (BIASED && i == wi) sel = raw[i];
      key[i] = (mine && i == wi) ? 0u : key[i];
    }
    if (BIASED) sel = __shfl_sync(MOE_FULL_MASK, sel, (int)(wid & 31u));
    if (lane == j) {
      my_val = BIASED ? sel : key_value(wmax);
      my_id = (int)wid;
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

}  // namespace

int launch_topk(const float* logits, int T, int E, int k, int32_t* idx, float* gate,
                int32_t* err, cudaStream_t s) {
  if (cudaMemsetAsync(err, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_LAUNCH;
  if (T == 0) return MOE_OK;
  const int threads = 256, per_block = threads / 32;
  const unsigned grid = (unsigned)((T + per_block - 1) / per_block);
#define MOE_TOPK_CASE(V) topk_kernel<V, false><<<grid, threads, 0, s>>>(logits, nullptr, T, E, k, idx, gate, err)
  if (E <= 32) MOE_TOPK_CASE(1);
  else if (E <= 64) MOE_TOPK_CASE(2);
  else if (E <= 128) MOE_TOPK_CASE(4);
  else if (E <= 256) MOE_TOPK_CASE(8);
  else if (E <= 512) MOE_TOPK_CASE(16);
  else MOE_TOPK_CASE(32);
#undef MOE_TOPK_CASE
  return launch_status();
}

int launch_topk_biased(const float* logits, const float* bias, int T, int E, int k,
                       int32_t* idx, float* gate, int32_t* err, cudaStream_t s) {
  if (cudaMemsetAsync(err, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_LAUNCH;
  if (T == 0) return MOE_OK;
  const int threads = 256, per_block = threads / 32;
  const unsigned grid = (unsigned)((T + per_block - 1) / per_block);
#define MOE_TOPKB_CASE(V) topk_kernel<V, true><<<grid, threads, 0, s>>>(logits, bias, T, E, k, idx, gate, err)
  if (E <= 32) MOE_TOPKB_CASE(1);
  else if (E <= 64) MOE_TOPKB_CASE(2);
  else if (E <= 128) MOE_TOPKB_CASE(4);
  else if (E <= 256) MOE_TOPKB_CASE(8);
  else if (E <= 512) MOE_TOPKB_CASE(16);
  else MOE_TOPKB_CASE(32);
#undef MOE_TOPKB_CASE
  return launch_status();
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
