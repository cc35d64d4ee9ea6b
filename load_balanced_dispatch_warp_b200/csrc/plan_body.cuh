// Equal-load plan with redundant expert copies, computed by one CTA (plan_block).
//
// The MoonEP news article (paragraphs 3-4) fixes the contract -- every rank receives
// exactly T*k/R rows, a few redundant expert copies are planned on the fly from the router
// output, and each copy takes one of S prefetch slots per rank from one global pool -- but
// gives no algorithm.  plan_block computes the "keep small, stream the rest" plan:
//   - rank r owns experts [rB, (r+1)B); ordered by (count, id) ascending, its experts
//     are kept whole while their running sum fits in C = T*k/R; the rest are streamed;
//   - the streamed experts in id order form one stream, cut by the ranks' leftover rooms
//     in rank order; each foreign run in a rank's piece is a replica taking the next slot.
// Everything is integer arithmetic, block scans and ballots (one warp per rank):
// deterministic.  Shared by the stand-alone plan kernel and the fused routing kernel.
#pragma once
#include "common.cuh"

namespace moe {
namespace {

constexpr int kPlanThreads = 256;
constexpr int kPlanWarps = kPlanThreads / 32;

// Shared-memory words plan_block needs for E experts and R <= E ranks.
__host__ __device__ constexpr int plan_smem_words(int E, int R) { return 6 * E + 2 * R + 38; }

// The plan of `counts` computed by the calling block (kPlanThreads threads): writes every
// field of `plan`, ORs MOE_DERR_SLOTS into *err when a rank needs more than S replicas.
// counts are read through L2 (they may have been summed by other blocks' atomics).
// smem: plan_smem_words(E, R) ints of shared memory.
__device__ __noinline__ void plan_block(const int32_t* __restrict__ counts, int T, int k, int E,
                                        int R, int S, int32_t* __restrict__ plan,
                                        const moe_plan_layout L, int32_t* __restrict__ err,
                                        int* smem) {
  int* s_c = smem;              // [E] counts
  int* s_kept = s_c + E;        // [E] 1 if kept whole at home
  int* s_so = s_kept + E;       // [E+1] stream offsets (exclusive scan of streamed counts)
  int* s_room = s_so + E + 1;   // [R+1] rooms, then their exclusive prefix
  int* s_kr = s_room + R + 1;   // [R] kept rows per rank
  int* s_off = s_kr + R;        // [E] local row offset of a kept expert, -1 otherwise
  int* s_sidx = s_off + E;      // [E+1] streamed experts (non-zero stream length), id order
  int* s_nrep = s_sidx + E + 1;  // [E+1] streamed flags, then replicas per rank and prefix
  int* s_scan = s_nrep + E + 1;  // [33]
  int& s_ns = s_scan[33];        // one more word: 6E + 2R + 38 in all
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int B = E / R;
  const int C = (int)(((long long)T * k) / R);

  for (int e = tid; e < E; e += blockDim.x) s_c[e] = __ldcg(counts + e);
  for (int r = tid; r < R; r += blockDim.x) s_kr[r] = 0;
  __syncthreads();

  // keep test: inclusive running sum of the rank's experts in (count, id) order <= C
  for (int e = tid; e < E; e += blockDim.x) {
    const int r0 = (e / B) * B, c = s_c[e];
    long long cum = c;
    for (int f = r0; f < r0 + B; ++f) {
      const int cf = s_c[f];
      if (cf < c || (cf == c && f < e)) cum += cf;
    }
    const int kept = cum <= C;
    s_kept[e] = kept;
    if (kept && c) atomicAdd(&s_kr[e / B], c);
  }
  __syncthreads();

  // local offsets of kept experts (id order); stream lengths; rooms
  for (int e = tid; e < E; e += blockDim.x) {
    int off = -1;
    if (s_kept[e]) {
      off = 0;
      for (int f = (e / B) * B; f < e; ++f)
        if (s_kept[f]) off += s_c[f];
    }
    s_off[e] = off;
    s_so[e] = s_kept[e] ? 0 : s_c[e];
    s_nrep[e] = (!s_kept[e] && s_c[e] > 0) ? 1 : 0;  // streamed flag (s_nrep as temp)
  }
  for (int r = tid; r < R; r += blockDim.x) s_room[r] = C - s_kr[r];
  __syncthreads();
  const int stream_len = block_exclusive_scan(s_so, E, s_scan);
  const int room_total = block_exclusive_scan(s_room, R, s_scan);
  // compact list of streamed experts in id order (= stream order)
  const int n_streamed = block_exclusive_scan(s_nrep, E, s_scan);
  for (int e = tid; e < E; e += blockDim.x)
    if (!s_kept[e] && s_c[e] > 0) s_sidx[s_nrep[e]] = e;
  if (tid == 0) {
    s_so[E] = stream_len;
    s_room[R] = room_total;
    s_ns = n_streamed;
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

  // one warp per rank: its kept experts (id order), then the runs of its stream piece
  const int G = B + S;
  for (int u = warp; u < R; u += kPlanWarps) {
    int32_t* gu = groups + (int64_t)u * G * 4;
    int g = 0;
    for (int c0 = 0; c0 < B; c0 += 32) {
      const int e = u * B + c0 + lane;
      const bool on = c0 + lane < B && s_kept[e] && s_c[e] > 0;
      const uint32_t m = __ballot_sync(MOE_FULL_MASK, on);
      if (on) {
        int4* rec = reinterpret_cast<int4*>(gu) + g + __popc(m & lanemask_lt());
        *rec = make_int4(u * C + s_off[e], s_c[e], e, e);
      }
      g += __popc(m);
    }
    const int lo = s_room[u], hi = s_room[u + 1];
    int nrep = 0;
    if (lo < hi) {
      // first streamed expert whose stream range ends after lo
      int a = 0, b = s_ns - 1;
      while (a < b) {
        const int mid = (a + b) >> 1;
        const int em = s_sidx[mid];
        if (s_so[em] + s_c[em] > lo) b = mid; else a = mid + 1;
      }
      for (int i0 = a; i0 < s_ns; i0 += 32) {
        const int i = i0 + lane;
        int e = -1, s0 = 0, s1 = 0;
        if (i < s_ns) {
          e = s_sidx[i];
          s0 = max(lo, s_so[e]);
          s1 = min(hi, s_so[e] + s_c[e]);
        }
        const bool on = e >= 0 && s0 < s1;
        const bool foreign = on && e / B != u;
        const uint32_t mfor = __ballot_sync(MOE_FULL_MASK, foreign);
        const int slot = nrep + __popc(mfor & lanemask_lt());
        // a run at its home rank is always recorded; a replica only while slots remain
        // (more than S replicas leaves the plan invalid: MOE_DERR_SLOTS below)
        const bool write = on && (!foreign || slot < S);
        const uint32_t mw = __ballot_sync(MOE_FULL_MASK, write);
        if (write) {
          int ref = e;
          if (foreign) {
            rep[u * S + slot] = e;
            ref = E + u * S + slot;
          }
          int4* rec = reinterpret_cast<int4*>(gu) + g + __popc(mw & lanemask_lt());
          *rec = make_int4(u * C + s_kr[u] + (s0 - lo), s1 - s0, e, ref);
        }
        g += __popc(mw);
        nrep += __popc(mfor);
        // stop once this chunk reached past the piece
        const bool past = e < 0 || s_so[e] >= hi;
        if (__any_sync(MOE_FULL_MASK, past)) break;
      }
    }
    for (int i = g * 4 + lane; i < 4 * G; i += 32) gu[i] = -1;
    for (int s = min(nrep, S) + lane; s < S; s += 32) rep[u * S + s] = -1;
    if (lane == 0) {
      n_groups[u] = g;
      s_nrep[u] = min(nrep, S);
      if (nrep > S) atomicOr(err, MOE_DERR_SLOTS);
    }
  }
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
}  // namespace moe
