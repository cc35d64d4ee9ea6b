// Shared device/host helpers of the MoE-layer library (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "moe.h"

#define MOE_FULL_MASK 0xffffffffu

namespace moe {

// ----------------------------------------------------------------------------- host side
// Launch helpers return a host status; every launcher below is called from abi.cu after
// the argument checks, so it only enqueues.
inline int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_LAUNCH;
}

int num_sms();  // SM count of the current device (cached per device)

// --------------------------------------------------------------- launchers (one per step)
// a[0, na) = 0 and b[0, nb) = 0 in one kernel launch (b may be null when nb == 0): the
// small resets of the path (error word, workspaces), cheaper as a kernel node of a CUDA
// graph than a memset node.
int launch_zero(int32_t* a, int64_t na, int32_t* b, int64_t nb, cudaStream_t s);
int launch_topk(const float* logits, int T, int E, int k, int32_t* idx, float* gate,
                int32_t* err, cudaStream_t s);
int launch_topk_biased(const float* logits, const float* bias, int T, int E, int k,
                       int32_t* idx, float* gate, int32_t* err, cudaStream_t s);
int launch_capacity(const int32_t* counts, int E, long long A, int cf_num, int cf_den,
                    int32_t* processed, int32_t* overflow, int32_t* padding, int32_t* totals,
                    const int32_t* err, cudaStream_t s);
int launch_histogram(const int32_t* idx, int T, int k, int E, int R, const int32_t* map,
                     int32_t* counts, int32_t* loads, double* maxvio, double* bal,
                     int32_t* err, cudaStream_t s);
int launch_plan(const int32_t* counts, int T, int k, int E, int R, int S, int32_t* plan,
                const moe_plan_layout& L, int32_t* err, cudaStream_t s);
int64_t route_plan_workspace_words(int E);
int launch_route_plan(const float* logits, const float* bias, int T, int E, int k, int R,
                      int S, int32_t* idx, float* gate, int32_t* counts, int32_t* loads,
                      double* maxvio, double* bal, int32_t* plan, const moe_plan_layout& L,
                      int32_t* ws, int32_t* err, cudaStream_t s);
int launch_prefetch(const int32_t* plan, const moe_plan_layout& L, const __nv_bfloat16* W1,
                    const __nv_bfloat16* W3, const __half* W2, int E, int R, int S, int d,
                    int F, __nv_bfloat16* P1, __nv_bfloat16* P3, __half* P2, int32_t* err,
                    cudaStream_t s);
int launch_dispatch(const __nv_bfloat16* x, const int32_t* idx, const int32_t* plan,
                    const moe_plan_layout& L, int T, int k, int E, int R, int d,
                    int32_t* ws, __nv_bfloat16* recv, int32_t* perm, int32_t* src,
                    int32_t* err, cudaStream_t s);
int launch_grouped_ffn(const __nv_bfloat16* recv, const int32_t* plan,
                       const moe_plan_layout& L, const __nv_bfloat16* W1,
                       const __nv_bfloat16* W3, const __half* W2, const __nv_bfloat16* P1,
                       const __nv_bfloat16* P3, const __half* P2, int T, int k, int E, int R,
                       int S, int d, int F, __half* h, __nv_bfloat16* y, int32_t* err,
                       cudaStream_t s);
int launch_grouped_ffn_gather(const __nv_bfloat16* x, const int32_t* src, const int32_t* plan,
                              const moe_plan_layout& L, const __nv_bfloat16* W1,
                              const __nv_bfloat16* W3, const __half* W2,
                              const __nv_bfloat16* P1, const __nv_bfloat16* P3,
                              const __half* P2, int T, int k, int E, int R, int S, int d, int F,
                              __half* h, __nv_bfloat16* y, int32_t* err, cudaStream_t s);
int launch_bounded_wait_selftest(int32_t* err, int limit_us, cudaStream_t s);
// grouped FFN tile mode (0: one CTA per 128-row tile, 1: 2-CTA clusters on 256-row tiles)
int set_ffn_tile_mode(int mode);  // MOE_OK or MOE_ERR_ARG
int ffn_tile_mode();
int ffn_pair_clusters();  // clusters the pair mode launches on the current device (0: none yet)
// backward pass (grouped_ffn_bwd.cu; the dispatch backward is launch_combine with
// gate == nullptr)
int64_t ffn_backward_workspace_bytes(int T, int k, int E, int R, int S, int d, int F, int G);
int launch_combine_backward(const __nv_bfloat16* dout, const __nv_bfloat16* y,
                            const int32_t* perm, const float* gate, int T, int k, int d,
                            __nv_bfloat16* dy, float* dgate, const int32_t* err,
                            cudaStream_t s);
int launch_topk_backward(const float* gate, const float* dgate, const int32_t* idx, int T, int E,
                         int k, float* dlogits, const int32_t* err, cudaStream_t s);
int launch_grouped_ffn_backward(const __nv_bfloat16* recv, const __nv_bfloat16* dy,
                                const __half* h,
                                const int32_t* plan, const moe_plan_layout& L,
                                const __nv_bfloat16* W1, const __nv_bfloat16* W3,
                                const __half* W2, int T, int k, int E, int R, int S, int d,
                                int F, __nv_bfloat16* dx_rows, float* dW1, float* dW3,
                                float* dW2, void* workspace, int64_t workspace_bytes,
                                int32_t* err, cudaStream_t s);
// drop: assignments with perm < 0 (fixed-capacity overflow) are left out of the sum
int launch_combine(const __nv_bfloat16* y, const int32_t* perm, const float* gate, int T,
                   int k, int d, __nv_bfloat16* out, const int32_t* err, cudaStream_t s,
                   bool drop = false);

// launch_dispatch with recv == nullptr computes perm and src only (no row copy).
// Workspace words of the dispatch's rank pass (tile statuses and per-tile expert counts).
int64_t dispatch_workspace_words(int T, int E);
// Fixed-capacity placement: expert e's q-th assignment (token order) at row e*cap + q when
// q < cap, else dropped (perm -1); padding rows of each expert zeroed in recv, src -1.
int launch_dispatch_capacity(const __nv_bfloat16* x, const int32_t* idx, const int32_t* counts,
                             int T, int k, int E, int cap, int d, int32_t* ws,
                             __nv_bfloat16* recv, int32_t* perm, int32_t* src, int32_t* err,
                             cudaStream_t s);
// moe_grouped_ffn with the combine folded into GEMM 2's epilogue: out32 [T,d] fp32
// (zeroed here) accumulates gate * y of every row; out = bf16(out32).  No y is written.
int launch_grouped_ffn_combine(const __nv_bfloat16* recv, const int32_t* plan,
                               const moe_plan_layout& L, const __nv_bfloat16* W1,
                               const __nv_bfloat16* W3, const __half* W2,
                               const __nv_bfloat16* P1, const __nv_bfloat16* P3,
                               const __half* P2, const int32_t* src, const int32_t* perm,
                               const float* gate, int T, int k, int E, int R, int S, int d,
                               int F, __half* h, float* out32, __nv_bfloat16* out, int32_t* err,
                               cudaStream_t s);
// The grouped FFN over E uniform groups of cap rows (group e = rows [e*cap, (e+1)*cap),
// expert e, home weights): the fixed-capacity layout.
int launch_grouped_ffn_capacity(const __nv_bfloat16* recv, const __nv_bfloat16* W1,
                                const __nv_bfloat16* W3, const __half* W2, int E, int cap,
                                int d, int F, __half* h, __nv_bfloat16* y, int32_t* err,
                                cudaStream_t s);

// The grouped FFN over an explicit group table [G][4] {row_start, rows, expert,
// weight_ref} (rows == -1: unused) on `rows` receive rows, one rank's worth: weight_ref
// < E reads the home tensors (E experts), E + s reads pool slot s (S slots).
int launch_grouped_ffn_groups(const __nv_bfloat16* recv, const int32_t* groups, int G,
                              int64_t rows, const __nv_bfloat16* W1, const __nv_bfloat16* W3,
                              const __half* W2, const __nv_bfloat16* P1, const __nv_bfloat16* P3,
                              const __half* P2, int E, int S, int d, int F, __half* h,
                              __nv_bfloat16* y, int32_t* err, cudaStream_t s);

// Expert parallelism across GPUs (ep.cu, and the peer forms of dispatch, prefetch and
// combine).  The *_ranks arrays are HOST arrays of W device pointers, one per rank, as
// mapped in this process.
int launch_ep_counts(const int32_t* idx, int T, int k, int E, const int32_t* err,
                     int32_t* send, cudaStream_t s);
int launch_ep_plan(const int32_t* gathered, int W, int me, int T, int k, int E, int S,
                   int32_t* counts, int32_t* q_base, int32_t* loads, double* maxvio, double* bal,
                   int32_t* plan, const moe_plan_layout& L, int32_t* err, cudaStream_t s);
int launch_ep_groups(const int32_t* plan, const moe_plan_layout& L, int me, int E, int W, int S,
                     int C, int32_t* groups, int32_t* err, cudaStream_t s);
int launch_ep_prefetch(const int32_t* plan, const moe_plan_layout& L,
                       const __nv_bfloat16* const* W1_ranks, const __nv_bfloat16* const* W3_ranks,
                       const __half* const* W2_ranks, int W, int me, int E, int S, int d, int F,
                       __nv_bfloat16* P1, __nv_bfloat16* P3, __half* P2, int32_t* err,
                       cudaStream_t s);
int launch_ep_dispatch(const __nv_bfloat16* x, const int32_t* idx, const int32_t* q_base,
                       const int32_t* plan, const moe_plan_layout& L, int T, int k, int E,
                       int W, int d, int32_t* ws, __nv_bfloat16* const* recv_ranks,
                       int32_t* perm, int32_t* err, cudaStream_t s);
int launch_ep_combine(const __nv_bfloat16* const* y_ranks, int W, const int32_t* perm,
                      const float* gate, int T, int k, int d, __nv_bfloat16* out,
                      const int32_t* err, cudaStream_t s);
// Backward of the expert-parallel layer (grouped_ffn_bwd.cu): dy rows written and y rows
// read on every rank; one rank's grouped-FFN backward over its re-based group table, the
// weight gradients of its home experts and of its pool slots ([B+S] entries); the slots'
// gradients added, in place, to their home experts' entries across ranks.  (The dispatch backward is
// launch_ep_combine with gate == nullptr.)
int64_t ep_ffn_backward_workspace_bytes(int T, int k, int E, int W, int S, int d, int F);
int launch_ep_combine_backward(const __nv_bfloat16* dout, const __nv_bfloat16* const* y_ranks,
                               const int32_t* perm, const float* gate, int W, int T, int k, int d,
                               __nv_bfloat16* const* dy_ranks, float* dgate, const int32_t* err,
                               cudaStream_t s);
int launch_ep_grouped_ffn_backward(const __nv_bfloat16* recv, const __nv_bfloat16* dy,
                                   const int32_t* groups, int B, int S, int C,
                                   const __nv_bfloat16* W1, const __nv_bfloat16* W3,
                                   const __half* W2, const __nv_bfloat16* P1,
                                   const __nv_bfloat16* P3, const __half* P2, int d, int F,
                                   __nv_bfloat16* dx_rows, float* dP1, float* dP3, float* dP2,
                                   void* workspace, int64_t workspace_bytes, int32_t* err,
                                   cudaStream_t s);
int launch_ep_reduce_home(const int32_t* plan, const moe_plan_layout& L,
                          float* const* part1_ranks, float* const* part3_ranks,
                          float* const* part2_ranks, int W, int me, int E, int S, int d, int F,
                          const int32_t* err, cudaStream_t s);

// bf16 -> fp16 copy of n (multiple of 8) values: the down projection's operand type.
int launch_bf16_to_f16(const __nv_bfloat16* in, int64_t n, __half* out, cudaStream_t s);

// ----------------------------------------------------------------------------- device side
// Reads the layer's error word once per thread; every kernel after moe_topk returns
// early when it is non-zero.
__device__ __forceinline__ int load_err(const int32_t* err) {
  return *reinterpret_cast<const volatile int32_t*>(err);
}

// Block-uniform version for kernels with barriers: thread 0 reads the word and the whole
// block takes the same decision.  Call at most once per kernel, before any other barrier.
__device__ __forceinline__ bool block_should_stop(const int32_t* err) {
  __shared__ int s_stop;
  if (threadIdx.x == 0) s_stop = load_err(err);
  __syncthreads();
  return s_stop != 0;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Warp-wide sum of a float (butterfly).
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(MOE_FULL_MASK, v, o);
  return v;
}

// Exclusive prefix sum of n <= 32*blockDim.x ints held in shared memory, in place, by
// the whole block; returns the total.  Chunked over blockDim.x with a running carry.
// `scratch` needs 33 ints of shared memory.  Every thread of the block must call it.
__device__ __forceinline__ int block_exclusive_scan(int* data, int n, int* scratch) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  int carry = 0;
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + tid;
    const int v = i < n ? data[i] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int t = __shfl_up_sync(MOE_FULL_MASK, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = lane < nwarps ? scratch[lane] : 0;
      int wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(MOE_FULL_MASK, wi, o);
        if (lane >= o) wi += t;
      }
      if (lane < nwarps) scratch[lane] = wi - w;  // exclusive warp offsets
      if (lane == 31) scratch[32] = wi;           // chunk total
    }
    __syncthreads();
    if (i < n) data[i] = carry + scratch[warp] + incl - v;
    carry += scratch[32];
    __syncthreads();
  }
  return carry;
}

}  // namespace moe
