// Equal-load plan with redundant expert copies, in one CTA.
//
// The MoonEP news article (paragraphs 3-4) fixes the contract -- every rank receives
// exactly T*k/R rows, a few redundant expert copies are planned on the fly from the router
// output, and each copy takes one of S prefetch slots per rank from one global pool -- but
// gives no algorithm.  This kernel computes the "keep small, stream the rest" plan:
//   - rank r owns experts [rB, (r+1)B); ordered by (count, id) ascending, its experts
//     are kept whole while their running sum fits in C = T*k/R; the rest are streamed;
//   - the streamed experts in id order form one stream, cut by the ranks' leftover rooms
//     in rank order; each foreign run in a rank's piece is a replica taking the next slot.
// Everything is integer arithmetic, block scans and per-thread walks: deterministic.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t* __restrict__ counts,
                                                            int T, int k, int E, int R, int S,
                                                            int32_t* __restrict__ plan,
                                                            moe_plan_layout L,
                                                            int32_t* __restrict__ err) {
  __shared__ int s_c[1024];       // counts
  __shared__ int s_kept[1024];    // 1 if kept whole at home
  __shared__ int s_so[1025];      // stream offsets (exclusive scan of streamed counts)
  __shared__ int s_room[1025];    // rooms, then their exclusive prefix
  __shared__ int s_kr[1024];      // kept rows per rank
  __shared__ int s_off[1024];     // local row offset of a kept expert, -1 otherwise
  __shared__ int s_nrep[1025];    // replicas per rank, then their exclusive prefix
  __shared__ int s_scan[33];
  if (block_should_stop(err)) return;
  const int tid = threadIdx.x;
  const int B = E / R;
  const int C = (int)(((long long)T * k) / R);

  for (int e = tid; e < E; e += blockDim.x) s_c[e] = counts[e];
  __syncthreads();

  // keep test: inclusive running sum of the rank's experts in (count, id) order <= C
  for (int e = tid; e < E; e += blockDim.x) {
    const int r0 = (e / B) * B, c = s_c[e];
    long long cum = c;
    for (int f = r0; f < r0 + B; ++f) {
      const int cf = s_c[f];
      if (cf < c || (cf == c && f < e)) cum += cf;
    }
    s_kept[e] = cum <= C;
  }
  __syncthreads();

  // local offsets of kept experts (id order) and kept rows per rank
  for (int e = tid; e < E; e += blockDim.x) {
    int off = -1;
    if (s_kept[e]) {
      off = 0;
      for (int f = (e / B) * B; f < e; ++f)
        if (s_kept[f]) off += s_c[f];
    }
    s_off[e] = off;
    s_so[e] = s_kept[e] ? 0 : s_c[e];
  }
  for (int r = tid; r < R; r += blockDim.x) {
    int kr = 0;
    for (int f = r * B; f < (r + 1) * B; ++f)
      if (s_kept[f]) kr += s_c[f];
    s_kr[r] = kr;
    s_room[r] = C - kr;
  }
  __syncthreads();
  const int stream_len = block_exclusive_scan(s_so, E, s_scan);
  const int room_total = block_exclusive_scan(s_room, R, s_scan);
  if (tid == 0) {
    s_so[E] = stream_len;
    s_room[R] = room_total;
  }
  __syncthreads();

  int32_t* kept_rows = plan + L.kept_rows;
  int32_t* room_prefix = plan + L.room_prefix;
  int32_t* home_off = plan + L.expert_home_off;
  int32_t* stream_off = plan + L.stream_off;
  int32_t* rep = plan + L.replica_expert;
  int32_t* rep_list = plan + L.replica_list;
  int32_t* n_groups = plan + L.n_groups;
  int32_t* groups = plan + L.groups;
  for (int r = tid; r < R; r += blockDim.x) kept_rows[r] = s_kr[r];
  for (int r = tid; r <= R; r += blockDim.x) room_prefix[r] = s_room[r];
  for (int e = tid; e < E; e += blockDim.x) home_off[e] = s_off[e];
  for (int e = tid; e <= E; e += blockDim.x) stream_off[e] = s_so[e];

  // one thread per rank: its kept experts, then the runs of its stream piece
  const int G = B + S;
  int overflow = 0;
  for (int u = tid; u < R; u += blockDim.x) {
    int32_t* gu = groups + (int64_t)u * G * 4;
    int g = 0;
    for (int e = u * B; e < (u + 1) * B; ++e) {
      if (s_kept[e] && s_c[e] > 0) {
        gu[4 * g + 0] = u * C + s_off[e];
        gu[4 * g + 1] = s_c[e];
        gu[4 * g + 2] = e;
        gu[4 * g + 3] = e;
        ++g;
      }
    }
    const int lo = s_room[u], hi = s_room[u + 1];
    int nrep = 0;
    if (lo < hi) {
      // first expert whose stream range ends after lo
      int a = 0, b = E - 1;
      while (a < b) {
        const int m = (a + b) >> 1;
        if (s_so[m + 1] > lo) b = m; else a = m + 1;
      }
      for (int e = a; e < E && s_so[e] < hi; ++e) {
        const int s0 = max(lo, s_so[e]), s1 = min(hi, s_so[e + 1]);
        if (s0 >= s1) continue;  // kept or empty experts have zero stream length
        const int row = u * C + s_kr[u] + (s0 - lo);
        int ref;
        if (e / B == u) {
          ref = e;
        } else {
          if (nrep >= S) { ++nrep; continue; }
          rep[u * S + nrep] = e;
          ref = E + u * S + nrep;
          ++nrep;
        }
        gu[4 * g + 0] = row;
        gu[4 * g + 1] = s1 - s0;
        gu[4 * g + 2] = e;
        gu[4 * g + 3] = ref;
        ++g;
      }
    }
    for (int i = 4 * g; i < 4 * G; ++i) gu[i] = -1;
    for (int s = min(nrep, S); s < S; ++s) rep[u * S + s] = -1;
    n_groups[u] = g;
    s_nrep[u] = min(nrep, S);
    if (nrep > S) overflow = 1;
  }
  if (overflow) atomicOr(err, MOE_DERR_SLOTS);
  __syncthreads();
  // compact list of filled slots in ascending slot order (for the prefetch copy)
  const int n_filled = block_exclusive_scan(s_nrep, R, s_scan);
  for (int u = tid; u < R; u += blockDim.x) {
    const int base = s_nrep[u];
    const int n = (u + 1 < R ? s_nrep[u + 1] : n_filled) - base;
    for (int s = 0; s < n; ++s) rep_list[1 + base + s] = u * S + s;
  }
  for (int i = n_filled + tid; i < R * S; i += blockDim.x) rep_list[1 + i] = -1;
  if (tid == 0) rep_list[0] = n_filled;
}

}  // namespace

int launch_plan(const int32_t* counts, int T, int k, int E, int R, int S, int32_t* plan,
                const moe_plan_layout& L, int32_t* err, cudaStream_t s) {
  plan_kernel<<<1, kPlanThreads, 0, s>>>(counts, T, k, E, R, S, plan, L, err);
  return launch_status();
}

}  // namespace moe
