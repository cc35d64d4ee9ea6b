// Expert parallelism across GPUs, one process per GPU: the steps that are specific to it.
//
// With one rank per GPU every rank routes only its own tokens, yet all ranks must place
// rows by the same equal-load plan (the MoonEP news article, paragraphs 2-3: the plan is
// computed from the router output, every rank receives exactly T*k/R rows).  So each
// rank packs its local demand and error word (ep_count_kernel), the caller exchanges those
// vectors between the ranks (an all-gather), and every rank then computes the job's
// demand, the same plan, and its own base offsets inside every expert's token order
// (ep_plan_kernel).  Token order of the job is rank-major: rank u's token t comes after
// every token of the ranks below u.  ep_groups_kernel re-bases the rank's own groups to
// its local receive buffer and its local weight tensors, so that the grouped FFN runs on
// one rank exactly as on the single-GPU layout.  Dispatch and combine across the ranks
// (peer stores and peer loads) live with their single-GPU versions in dispatch.cu and
// move.cu; the phases are those of "DeepEP-on-EFA Guidance, section 1: What is MoE",
// (b) dispatch and (d) combine.
#include "plan_body.cuh"

namespace moe {
namespace {

constexpr int kCountThreads = 256;

// send[e] += assignments of expert e among this rank's T tokens; send[E] |= the rank's
// error word and the validation bits (an id outside [0, E), a repeated id within a token).
// send is zeroed before the launch.  The launch never writes *err: the bits travel in
// send[E] and come back through the exchanged vectors, so every block takes the same
// entry decision and the recorded bits do not depend on block scheduling.
__global__ void __launch_bounds__(kCountThreads) ep_count_kernel(
    const int32_t* __restrict__ idx, int T, int k, int E, const int32_t* __restrict__ err,
    int32_t* __restrict__ send) {
  extern __shared__ int s_cnt[];  // [E]
  __shared__ int s_bits;
  if (threadIdx.x == 0) s_bits = load_err(err);
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_cnt[e] = 0;
  __syncthreads();
  const int e0 = s_bits;
  if (e0 != 0) {  // an earlier step failed: report it, count nothing
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(send + E, e0);
    return;
  }
  int bits = 0;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < T;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int32_t* row = idx + t * k;
    for (int j = 0; j < k; ++j) {
      const int e = __ldg(row + j);
      if (e < 0 || e >= E) {
        bits |= MOE_DERR_ID_RANGE;
        continue;
      }
      for (int i = 0; i < j; ++i)
        if (__ldg(row + i) == e) bits |= MOE_DERR_DUPLICATE;
      atomicAdd(&s_cnt[e], 1);
    }
  }
  if (bits) atomicOr(&s_bits, bits);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (s_cnt[e]) atomicAdd(send + e, s_cnt[e]);
  if (threadIdx.x == 0 && s_bits) atomicOr(send + E, s_bits);
}

// One CTA.  gathered [W][E+1]: every rank's send vector, in rank order.
//   err     |= the OR of every rank's error word; when non-zero nothing else is written,
//              on every rank alike (they all see the same vectors);
//   counts  [E]  demand of the job, sum over the ranks;
//   q_base  [E]  assignments of expert e made by the ranks below `me`;
//   loads [W], maxvio, bal: under the home map e -> e / (E/W), maxvio = (W*max - A)/A and
//              balancedness = A/(W*max), A = W*T*k, one fp64 rounding each;
//   plan         plan_block on the job's demand (T_job = W*T, R = W).
__global__ void __launch_bounds__(kPlanThreads) ep_plan_kernel(
    const int32_t* __restrict__ gathered, int W, int me, int T, int k, int E, int S,
    int32_t* __restrict__ counts, int32_t* __restrict__ q_base, int32_t* __restrict__ loads,
    double* __restrict__ maxvio, double* __restrict__ bal, int32_t* __restrict__ plan,
    moe_plan_layout L, int32_t* __restrict__ err) {
  extern __shared__ int s_plan[];  // plan_smem_words(E, W) >= 32 ints
  __shared__ int s_bits;
  const int tid = threadIdx.x, lane = tid & 31;
  const int64_t ld = E + 1;
  if (tid == 0) s_bits = load_err(err);
  __syncthreads();
  int bits = 0;
  for (int r = tid; r < W; r += blockDim.x) bits |= __ldg(gathered + r * ld + E);
  if (bits) atomicOr(&s_bits, bits);
  __syncthreads();
  if (s_bits != 0) {
    if (tid == 0) atomicOr(err, s_bits);
    return;
  }
  for (int e = tid; e < E; e += blockDim.x) {
    int c = 0, b = 0;
    for (int r = 0; r < W; ++r) {
      const int v = __ldg(gathered + r * ld + e);
      if (r < me) b += v;
      c += v;
    }
    counts[e] = c;
    q_base[e] = b;
  }
  __syncthreads();
  // rank loads under the home map and the imbalance scalars
  const int B = E / W;
  int* s_max = s_plan;  // [32], free until plan_block
  int mx = 0;
  for (int r = tid; r < W; r += blockDim.x) {
    int v = 0;
    for (int e = r * B; e < (r + 1) * B; ++e) v += counts[e];
    loads[r] = v;
    mx = max(mx, v);
  }
  mx = __reduce_max_sync(MOE_FULL_MASK, mx);
  if (lane == 0) s_max[tid >> 5] = mx;
  __syncthreads();
  if (tid < 32) {
    const int nw = (blockDim.x + 31) >> 5;
    int v = tid < nw ? s_max[tid] : 0;
    v = __reduce_max_sync(MOE_FULL_MASK, v);
    if (tid == 0) {
      const long long A = (long long)W * T * k;
      const long long top = (long long)W * v;
      if (A == 0 || v == 0) {
        *maxvio = 0.0;
        *bal = 1.0;
      } else {
        *maxvio = (double)(top - A) / (double)A;
        *bal = (double)A / (double)top;
      }
    }
  }
  __syncthreads();
  plan_block(counts, W * T, k, E, W, S, plan, L, err, s_plan);
}

// The group table of rank `me`, re-based for its own buffers: row_start - me*C (local
// receive rows), weight_ref e -> e - me*B (its home tensors hold experts [me*B, me*B+B)),
// E + me*S + s -> B + s (its own pool slot s); the expert field gets the same local index
// (the backward keys its weight gradients on it: home experts, then slots).  Unused
// entries stay all -1.  A group whose weights are not on this rank (never produced by the
// plan) raises MOE_DERR_ID_RANGE and is dropped.
__global__ void __launch_bounds__(128) ep_groups_kernel(const int32_t* __restrict__ plan,
                                                        moe_plan_layout L, int me, int E,
                                                        int W, int S, int C,
                                                        int4* __restrict__ out,
                                                        int32_t* __restrict__ err) {
  if (load_err(err)) return;
  const int B = E / W, G = B + S;
  const int4* g = reinterpret_cast<const int4*>(plan + L.groups) + (int64_t)me * G;
  for (int i = threadIdx.x; i < G; i += blockDim.x) {
    int4 v = g[i];
    if (v.y >= 0) {
      const int ref = v.w;
      int local;
      if (ref < E) local = ref - me * B;
      else local = B + (ref - E - me * S);
      const bool ok = (ref < E) ? (local >= 0 && local < B) : (local >= B && local < B + S);
      if (ok) {
        v.x -= me * C;
        v.z = local;
        v.w = local;
      } else {
        atomicOr(err, MOE_DERR_ID_RANGE);
        v = make_int4(-1, -1, -1, -1);
      }
    }
    out[i] = v;
  }
}

}  // namespace

int launch_ep_counts(const int32_t* idx, int T, int k, int E, const int32_t* err,
                     int32_t* send, cudaStream_t s) {
  if (const int st = launch_zero(send, E + 1, nullptr, 0, s); st != MOE_OK) return st;
  const int64_t want = ((int64_t)T + kCountThreads - 1) / kCountThreads;
  const int64_t capb = (int64_t)num_sms() * 2;
  const int blocks = (int)(want < 1 ? 1 : (want < capb ? want : capb));
  ep_count_kernel<<<blocks, kCountThreads, sizeof(int) * (size_t)E, s>>>(idx, T, k, E, err, send);
  return launch_status();
}

int launch_ep_plan(const int32_t* gathered, int W, int me, int T, int k, int E, int S,
                   int32_t* counts, int32_t* q_base, int32_t* loads, double* maxvio, double* bal,
                   int32_t* plan, const moe_plan_layout& L, int32_t* err, cudaStream_t s) {
  ep_plan_kernel<<<1, kPlanThreads, sizeof(int) * (size_t)plan_smem_words(E, W), s>>>(
      gathered, W, me, T, k, E, S, counts, q_base, loads, maxvio, bal, plan, L, err);
  return launch_status();
}

int launch_ep_groups(const int32_t* plan, const moe_plan_layout& L, int me, int E, int W, int S,
                     int C, int32_t* groups, int32_t* err, cudaStream_t s) {
  ep_groups_kernel<<<1, 128, 0, s>>>(plan, L, me, E, W, S, C, reinterpret_cast<int4*>(groups),
                                     err);
  return launch_status();
}

}  // namespace moe
