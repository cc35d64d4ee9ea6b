// Row movement of the layer: replica prefetch, zero-copy placement + dispatch, combine.
//
// Dispatch and combine are the two all-to-all phases of "DeepEP-on-EFA Guidance, section
// 1: What is MoE" (dispatch sends each token to its k experts only; combine is its
// transpose with the gate-weighted sum); with ranks simulated as partitions of one GPU's
// HBM they are gathers/scatters of whole rows.  Prefetch and zero-copy placement follow
// the MoonEP news article, paragraph 3.  All of it is HBM-bound: 16-byte vector loads and
// stores, each token row read once.
#include "rows.cuh"

namespace moe {
namespace {

// ----------------------------------------------------------------------------- prefetch

// Replica prefetch through the bulk-copy engine: one thread per CTA (one CTA per SM)
// streams 32 KiB chunks global -> shared (completion on the buffer's mbarrier) -> global
// (bulk group), kBulkBufs buffers in flight, so the copy rate does not depend on how many
// instructions the SM issues (a 16-byte-vector copy with 1024 threads per SM reached 0.92
// of the copy peak alone and 0.86 in the power-capped step; this one 0.97 and 0.94).
// Units are (filled slot, projection, chunk); d*F*2 is a multiple of 32 KiB (d and F are
// multiples of 128).  Every wait is bounded; a wait that runs out ORs MOE_DERR_TIMEOUT into
// *err and the thread drains its copies before the CTA leaves.
//
// Where a slot's expert lives: w[p][u] is rank u's home tensor of projection p (W1, W3,
// W2) and holds experts [u*B, (u+1)*B).  One GPU: one "rank" with B = E, the slots to fill
// from the plan's compact list.  Expert parallelism: this process's pointers to every
// rank's home tensors (a peer GPU's memory mapped here, read over NVLink; bulk loads, no
// multicast) and rank `me`'s own S slots, the filled ones gathered by the copying thread.
struct PrefetchSrc {
  const uint8_t* w[3][MOE_EP_MAX_RANKS];
  int B;
};
constexpr int kBulkChunk = 32768;
constexpr int kBulkBufs = 6;
constexpr int kBulkMaxSlots = 4096;  // slots of one rank: the argument rules keep R*(B+S) <= 4096
constexpr uint64_t kBulkWaitNs = 500000000ull;

__device__ __forceinline__ uint32_t bulk_smem(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ bool bulk_try(uint32_t bar, uint32_t parity) {
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
__device__ __forceinline__ bool bulk_wait(uint32_t bar, uint32_t parity) {
  if (bulk_try(bar, parity)) return true;
  uint64_t t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (;;) {
    if (bulk_try(bar, parity)) return true;
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 > kBulkWaitNs) return false;
  }
}

// rep[0, nslots): the experts of the slots (-1 empty); list: the plan's compact list of
// filled slots ({count, slots...}), or null to take the filled ones of rep in slot order.
// A listed slot outside [0, nslots), or an expert whose home tensor is not in the table,
// sets MOE_DERR_ID_RANGE and is skipped (never read from or written to).
__global__ void __launch_bounds__(32) prefetch_bulk_kernel(
    const int32_t* __restrict__ rep, const int32_t* __restrict__ list, int nslots,
    const __grid_constant__ PrefetchSrc src, uint8_t* __restrict__ P1, uint8_t* __restrict__ P3,
    uint8_t* __restrict__ P2, int64_t proj_bytes, int32_t* __restrict__ err) {
  extern __shared__ __align__(128) uint8_t buf[];  // kBulkBufs * kBulkChunk
  __shared__ __align__(8) uint64_t bar[kBulkBufs];
  __shared__ int s_slots[kBulkMaxSlots];
  const int lane = threadIdx.x;
  if (load_err(err)) return;
  // the slots to fill, in order, gathered by the whole warp (32 candidates per step)
  const int listed = list != nullptr ? __ldg(list) : nslots;
  const int cand = min(listed, kBulkMaxSlots);
  int n = 0;
  bool bad = listed > kBulkMaxSlots;
  for (int base = 0; base < cand; base += 32) {
    const int c = base + lane;
    bool keep = false;
    int q = -1;
    if (c < cand) {
      q = list != nullptr ? __ldg(list + 1 + c) : c;
      if (q < 0 || q >= nslots) {
        bad = true;
      } else {
        const int e = __ldg(rep + q);
        if (e < 0) {
          bad |= list != nullptr;  // the plan lists filled slots only
        } else {
          const int home = e / src.B;
          if (home >= MOE_EP_MAX_RANKS || src.w[0][home] == nullptr) bad = true;
          else keep = true;
        }
      }
    }
    const uint32_t kept = __ballot_sync(MOE_FULL_MASK, keep);
    if (keep) s_slots[n + __popc(kept & ((1u << lane) - 1u))] = q;
    n += __popc(kept);
  }
  if (__any_sync(MOE_FULL_MASK, bad) && lane == 0) atomicOr(err, MOE_DERR_ID_RANGE);
  __syncwarp();
  if (lane != 0) return;
  for (int b = 0; b < kBulkBufs; ++b)
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bulk_smem(&bar[b])) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  const int64_t chunks = proj_bytes / kBulkChunk;
  const int64_t total = (int64_t)n * 3 * chunks;
  // this CTA's units: blockIdx.x + i * gridDim.x, i = 0, 1, ...
  const int64_t mine = total > blockIdx.x ? (total - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  auto unit_ptrs = [&](int64_t i, const uint8_t*& from, uint8_t*& to) {
    const int64_t w = blockIdx.x + i * gridDim.x;
    const int64_t si = w / (3 * chunks);
    const int64_t rem = w - si * 3 * chunks;
    const int proj = (int)(rem / chunks);
    const int64_t off = (rem - (int64_t)proj * chunks) * kBulkChunk;
    const int slot = s_slots[si];
    const int e = __ldg(rep + slot);
    const int home = e / src.B;
    from = src.w[proj][home] + (int64_t)(e - home * src.B) * proj_bytes + off;
    to = (proj == 0 ? P1 : proj == 1 ? P3 : P2) + (int64_t)slot * proj_bytes + off;
  };
  auto issue_load = [&](int64_t i) {
    const uint8_t* from;
    uint8_t* to;
    unit_ptrs(i, from, to);
    const int b = (int)(i % kBulkBufs);
    const uint32_t bb = bulk_smem(&bar[b]);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bb),
                 "r"(kBulkChunk)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            bulk_smem(buf + (size_t)b * kBulkChunk)),
        "l"(from), "r"(kBulkChunk), "r"(bb)
        : "memory");
  };
  int64_t issued = 0, i = 0;
  for (; issued < min(mine, (int64_t)kBulkBufs - 1); ++issued) issue_load(issued);
  bool ok = true;
  for (; i < mine; ++i) {
    const int b = (int)(i % kBulkBufs);
    if (!bulk_wait(bulk_smem(&bar[b]), (uint32_t)((i / kBulkBufs) & 1))) {
      ok = false;
      break;
    }
    const uint8_t* from;
    uint8_t* to;
    unit_ptrs(i, from, to);
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(to),
                 "r"(bulk_smem(buf + (size_t)b * kBulkChunk)), "r"(kBulkChunk)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    if (issued < mine) {
      // the buffer of unit i - 1, which the next load reuses, has been read by its store
      asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
      issue_load(issued++);
    }
  }
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  if (!ok) {
    atomicOr(err, MOE_DERR_TIMEOUT);
    for (int64_t v = i + 1; v < issued; ++v)
      bulk_wait(bulk_smem(&bar[v % kBulkBufs]), (uint32_t)((v / kBulkBufs) & 1));
  }
}

int launch_prefetch_bulk(const int32_t* rep, const int32_t* list, int nslots,
                         const PrefetchSrc& src, uint8_t* P1, uint8_t* P3, uint8_t* P2,
                         int64_t proj_bytes, int32_t* err, cudaStream_t s) {
  const size_t smem = (size_t)kBulkBufs * kBulkChunk;
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaFuncSetAttribute(prefetch_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    configured[dev] = true;
  }
  prefetch_bulk_kernel<<<num_sms(), 32, smem, s>>>(rep, list, nslots, src, P1, P3, P2,
                                                   proj_bytes, err);
  return launch_status();
}

constexpr int kRowThreads = 256;

// ----------------------------------------------------------------------------- combine

__device__ __forceinline__ void acc_bf16x8(float* acc, const uint4& v, float g) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(p[i]);
    acc[2 * i] = fmaf(g, f.x, acc[2 * i]);
    acc[2 * i + 1] = fmaf(g, f.y, acc[2 * i + 1]);
  }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float* a) {
  uint4 o;
  __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = __floats2bfloat162_rn(a[2 * i], a[2 * i + 1]);
  return o;
}

// out[t] = sum_j gate[t,j] * y[perm[t,j]], fp32 in j order, one warp per token.  With the
// top-k known at compile time (K > 0) all K x V gathers of a lane are issued before the
// first FMA; K == 0 is the generic loop.  V (16-byte vectors per lane and gather) is 1
// for K > 4 so that the kernel stays near 40 registers and enough warps are resident
// to keep the gathers in flight.
// DROP: an assignment with perm < 0 (dropped by the fixed-capacity dispatch) is left out
// of the sum.
// Src (rows.cuh) says where row r of y lives: LocalY or RankY; both sum the same values in
// the same order.
template <int K, bool DROP = false, int kCombVec = (K > 4 || K == 0) ? 1 : 2, class Src = LocalY>
__global__ void __launch_bounds__(kRowThreads) combine_kernel(
    const __grid_constant__ Src y, const int32_t* __restrict__ perm,
    const float* __restrict__ gate, int T, int k, int dv, uint4* __restrict__ out,
    const int32_t* __restrict__ err) {
  if (load_err(err)) return;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += nwarps) {
    const int r = lane < k ? __ldg(perm + t * k + lane) : 0;
    // gate == nullptr: unit weights (the backward of dispatch sums the k rows)
    const float gl = lane < k ? (gate ? __ldg(gate + t * k + lane) : 1.f) : 0.f;
    if (K > 0) {
      // rows and gates of the token broadcast once; the vector loop has no warp collective
      int rows[K > 0 ? K : 1];
      float g[K > 0 ? K : 1];
#pragma unroll
      for (int j = 0; j < K; ++j) {
        rows[j] = __shfl_sync(MOE_FULL_MASK, r, j);
        g[j] = __shfl_sync(MOE_FULL_MASK, gl, j);
      }
      for (int v0 = lane; v0 < dv; v0 += 32 * kCombVec) {
        float acc[kCombVec][8];
#pragma unroll
        for (int u = 0; u < kCombVec; ++u)
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
        uint4 buf[K > 0 ? K : 1][kCombVec];
#pragma unroll
        for (int j = 0; j < K; ++j)
#pragma unroll
          for (int u = 0; u < kCombVec; ++u)
            if (v0 + u * 32 < dv && (!DROP || rows[j] >= 0))
              buf[j][u] = __ldcs(y.row(rows[j], dv) + v0 + u * 32);
#pragma unroll
        for (int j = 0; j < K; ++j)
#pragma unroll
          for (int u = 0; u < kCombVec; ++u)
            if (v0 + u * 32 < dv && (!DROP || rows[j] >= 0)) acc_bf16x8(acc[u], buf[j][u], g[j]);
#pragma unroll
        for (int u = 0; u < kCombVec; ++u)
          if (v0 + u * 32 < dv) out[t * dv + v0 + u * 32] = pack_bf16x8(acc[u]);
      }
    } else {
      // generic k: warp-uniform trip count (the shuffles need every lane), lane predicate
      for (int base = 0; base < dv; base += 32) {
        const int v = base + lane;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        for (int j = 0; j < k; ++j) {
          const int row = __shfl_sync(MOE_FULL_MASK, r, j);
          const float gj = __shfl_sync(MOE_FULL_MASK, gl, j);
          if (v < dv && (!DROP || row >= 0)) acc_bf16x8(acc, __ldcs(y.row(row, dv) + v), gj);
        }
        if (v < dv) out[t * dv + v] = pack_bf16x8(acc);
      }
    }
  }
}

int row_grid(int T) {
  const int per_block = kRowThreads / 32;
  const int64_t want = ((int64_t)T + per_block - 1) / per_block;
  const int64_t cap = (int64_t)num_sms() * 8;
  return (int)(want < cap ? want : cap);
}

// bf16 -> fp16, element by element, round to nearest even (exact for 0 and every bf16 value
// with 2^-17 <= |w| <= 65504; smaller ones round to the fp16 subnormal grid), 8 values per
// thread and step.
__global__ void __launch_bounds__(256) bf16_to_f16_kernel(const uint4* __restrict__ in,
                                                          uint4* __restrict__ out, int64_t n8) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = __ldcs(in + i);
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
    uint4 o;
    __half2* h = reinterpret_cast<__half2*>(&o);
#pragma unroll
    for (int j = 0; j < 4; ++j) h[j] = __float22half2_rn(__bfloat1622float2(b[j]));
    out[i] = o;
  }
}

}  // namespace

int launch_bf16_to_f16(const __nv_bfloat16* in, int64_t n, __half* out, cudaStream_t s) {
  if (n == 0) return MOE_OK;
  const int64_t n8 = n / 8;
  const int64_t want = (n8 + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 8;
  bf16_to_f16_kernel<<<(unsigned)(want < cap ? want : cap), 256, 0, s>>>(
      reinterpret_cast<const uint4*>(in), reinterpret_cast<uint4*>(out), n8);
  return launch_status();
}


int launch_prefetch(const int32_t* plan, const moe_plan_layout& L, const __nv_bfloat16* W1,
                    const __nv_bfloat16* W3, const __half* W2, int E, int R, int S, int d,
                    int F, __nv_bfloat16* P1, __nv_bfloat16* P3, __half* P2, int32_t* err,
                    cudaStream_t s) {
  if (S == 0) return MOE_OK;
  PrefetchSrc src = {};
  src.w[0][0] = reinterpret_cast<const uint8_t*>(W1);
  src.w[1][0] = reinterpret_cast<const uint8_t*>(W3);
  src.w[2][0] = reinterpret_cast<const uint8_t*>(W2);
  src.B = E;
  return launch_prefetch_bulk(plan + L.replica_expert, plan + L.replica_list, R * S, src,
                              reinterpret_cast<uint8_t*>(P1), reinterpret_cast<uint8_t*>(P3),
                              reinterpret_cast<uint8_t*>(P2), (int64_t)d * F * 2, err, s);
}

int launch_combine(const __nv_bfloat16* y, const int32_t* perm, const float* gate, int T,
                   int k, int d, __nv_bfloat16* out, const int32_t* err, cudaStream_t s,
                   bool drop) {
  if (T == 0) return MOE_OK;
  const LocalY yv{reinterpret_cast<const uint4*>(y)};
  uint4* ov = reinterpret_cast<uint4*>(out);
  const int g = row_grid(T), dv = d / 8;
  if (drop) {
#define MOE_COMBINE_DROP(KK) combine_kernel<KK, true><<<g, kRowThreads, 0, s>>>(yv, perm, gate, T, k, dv, ov, err)
    switch (k) {
      case 1: MOE_COMBINE_DROP(1); break;
      case 2: MOE_COMBINE_DROP(2); break;
      case 4: MOE_COMBINE_DROP(4); break;
      case 6: MOE_COMBINE_DROP(6); break;
      case 8: MOE_COMBINE_DROP(8); break;
      default: MOE_COMBINE_DROP(0); break;
    }
#undef MOE_COMBINE_DROP
    return launch_status();
  }
  // long rows (d >= 4096): two vectors per gather in flight also for k > 4 (at d = 7168,
  // k = 8: 358 -> 322 us alone; at d = 2048 one vector stays ~1% faster)
  const bool wide = dv >= 512;
#define MOE_COMBINE_CASE(KK)                                                                    \
  do {                                                                                          \
    if (wide && KK > 4)                                                                         \
      combine_kernel<KK, false, 2><<<g, kRowThreads, 0, s>>>(yv, perm, gate, T, k, dv, ov, err); \
    else                                                                                        \
      combine_kernel<KK><<<g, kRowThreads, 0, s>>>(yv, perm, gate, T, k, dv, ov, err);          \
  } while (0)
  switch (k) {
    case 1: MOE_COMBINE_CASE(1); break;
    case 2: MOE_COMBINE_CASE(2); break;
    case 3: MOE_COMBINE_CASE(3); break;
    case 4: MOE_COMBINE_CASE(4); break;
    case 5: MOE_COMBINE_CASE(5); break;
    case 6: MOE_COMBINE_CASE(6); break;
    case 7: MOE_COMBINE_CASE(7); break;
    case 8: MOE_COMBINE_CASE(8); break;
    default: MOE_COMBINE_CASE(0); break;
  }
#undef MOE_COMBINE_CASE
  return launch_status();
}

int launch_ep_prefetch(const int32_t* plan, const moe_plan_layout& L,
                       const __nv_bfloat16* const* W1_ranks, const __nv_bfloat16* const* W3_ranks,
                       const __half* const* W2_ranks, int W, int me, int E, int S, int d, int F,
                       __nv_bfloat16* P1, __nv_bfloat16* P3, __half* P2, int32_t* err,
                       cudaStream_t s) {
  if (S == 0) return MOE_OK;
  if (S > kBulkMaxSlots) return MOE_ERR_SHAPE;
  PrefetchSrc src = {};
  for (int u = 0; u < W && u < MOE_EP_MAX_RANKS; ++u) {
    src.w[0][u] = reinterpret_cast<const uint8_t*>(W1_ranks[u]);
    src.w[1][u] = reinterpret_cast<const uint8_t*>(W3_ranks[u]);
    src.w[2][u] = reinterpret_cast<const uint8_t*>(W2_ranks[u]);
  }
  src.B = E / W;
  return launch_prefetch_bulk(plan + L.replica_expert + (int64_t)me * S, nullptr, S, src,
                              reinterpret_cast<uint8_t*>(P1), reinterpret_cast<uint8_t*>(P3),
                              reinterpret_cast<uint8_t*>(P2), (int64_t)d * F * 2, err, s);
}

int launch_ep_combine(const __nv_bfloat16* const* y_ranks, int W, const int32_t* perm,
                      const float* gate, int T, int k, int d, __nv_bfloat16* out,
                      const int32_t* err, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  RankY yv;
  for (int u = 0; u < MOE_EP_MAX_RANKS; ++u)
    yv.base[u] = u < W ? reinterpret_cast<const uint4*>(y_ranks[u]) : nullptr;
  yv.C = T * k;
  uint4* ov = reinterpret_cast<uint4*>(out);
  const int g = row_grid(T), dv = d / 8;
  const bool wide = dv >= 512;  // as launch_combine
#define MOE_EP_COMBINE(KK)                                                                      \
  do {                                                                                          \
    if (wide && KK > 4)                                                                         \
      combine_kernel<KK, false, 2, RankY><<<g, kRowThreads, 0, s>>>(yv, perm, gate, T, k, dv,   \
                                                                   ov, err);                    \
    else                                                                                        \
      combine_kernel<KK, false, (KK > 4 || KK == 0) ? 1 : 2, RankY><<<g, kRowThreads, 0, s>>>(  \
          yv, perm, gate, T, k, dv, ov, err);                                                   \
  } while (0)
  switch (k) {
    case 1: MOE_EP_COMBINE(1); break;
    case 2: MOE_EP_COMBINE(2); break;
    case 4: MOE_EP_COMBINE(4); break;
    case 6: MOE_EP_COMBINE(6); break;
    case 8: MOE_EP_COMBINE(8); break;
    default: MOE_EP_COMBINE(0); break;
  }
#undef MOE_EP_COMBINE
  return launch_status();
}

}  // namespace moe
