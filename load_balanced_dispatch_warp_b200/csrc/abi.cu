// The C ABI (include/moe.h): argument checks, then one launcher per step.
// Every check runs on the host before anything is enqueued.
#include "checks.cuh"
#include "common.cuh"

namespace moe {

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64) {
    if (!cached[dev]) {
      int n = 0;
      if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
      cached[dev] = n;
    }
    return cached[dev];
  }
  return 148;
}

}  // namespace moe

namespace {

using moe::checks::aligned16;
using moe::checks::kMaxElems;
constexpr auto check_route = moe::checks::route;
constexpr auto check_ranks = moe::checks::ranks;
constexpr auto check_dims = moe::checks::dims;
constexpr auto check_groups = moe::checks::groups;

cudaStream_t as_stream(moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

#define MOE_TRY(expr)          \
  do {                         \
    const int st_ = (expr);    \
    if (st_ != MOE_OK) return st_; \
  } while (0)

// W ranks, rank me, T tokens per rank: the single-GPU rules on the job (W*T tokens,
// R = W) and on this rank's T*k receive rows.
int check_ep(int W, int me, int T, int k, int E, int S) {
  if (W < 1 || me < 0 || me >= W || T < 0) return MOE_ERR_ARG;
  if (W > MOE_EP_MAX_RANKS) return MOE_ERR_SHAPE;
  MOE_TRY(check_route(T, E, k));
  if ((int64_t)W * T * k >= kMaxElems || (int64_t)W * T * E >= kMaxElems) return MOE_ERR_SHAPE;
  MOE_TRY(check_ranks(W * T, k, E, W, true));
  return check_groups(E, W, S);
}

// every entry of a host table of W device pointers non-null and 16-byte aligned
template <typename P>
int check_table(P const* table, int W) {
  if (!table) return MOE_ERR_ARG;
  for (int u = 0; u < W; ++u)
    if (!table[u] || !aligned16(table[u])) return MOE_ERR_ARG;
  return MOE_OK;
}


}  // namespace

extern "C" {

int moe_plan_get_layout(int E, int R, int S, moe_plan_layout* out) {
  if (!out || E < 1 || R < 1 || S < 0) return MOE_ERR_ARG;
  if (E % R != 0) return MOE_ERR_SHAPE;
  const int64_t B = E / R;
  moe_plan_layout L;
  L.kept_rows = 0;
  L.room_prefix = L.kept_rows + R;
  L.expert_home_off = L.room_prefix + R + 1;
  L.stream_off = L.expert_home_off + E;
  L.replica_expert = L.stream_off + E + 1;
  L.replica_list = L.replica_expert + (int64_t)R * S;
  L.n_groups = L.replica_list + 1 + (int64_t)R * S;
  L.groups = ((L.n_groups + R) + 3) / 4 * 4;  // 16-byte aligned group records
  L.words = L.groups + (int64_t)R * (B + S) * 4;
  L.max_groups_per_rank = (int32_t)(B + S);
  *out = L;
  return MOE_OK;
}

int64_t moe_dispatch_workspace_words(int T, int E) {
  if (T < 0 || E < 1) return 0;
  return moe::dispatch_workspace_words(T, E);
}

int64_t moe_capacity_rows(int T, int k, int E, int cf_num, int cf_den) {
  if (T < 0 || k < 1 || E < 1 || cf_num < 1 || cf_den < 1) return -1;
  const long long num = (long long)T * k * cf_num, den = (long long)E * cf_den;
  return (num + den - 1) / den;
}

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_ARG: return "null pointer, misaligned pointer or negative size";
    case MOE_ERR_SHAPE: return "size limit violated";
    case MOE_ERR_LAUNCH: return "CUDA launch failed";
    case MOE_ERR_DEVICE: return "no usable sm_100 device or driver entry point";
    default: return "unknown status";
  }
}

int moe_topk(const float* logits, int T, int E, int k, int32_t* idx, float* gate,
             int32_t* err, moe_stream_t stream) {
  if (!err || (T > 0 && (!logits || !idx || !gate))) return MOE_ERR_ARG;
  MOE_TRY(check_route(T, E, k));
  return moe::launch_topk(logits, T, E, k, idx, gate, err, as_stream(stream));
}

int moe_topk_biased(const float* logits, const float* bias, int T, int E, int k, int32_t* idx,
                    float* gate, int32_t* err, moe_stream_t stream) {
  if (!err || !bias || (T > 0 && (!logits || !idx || !gate))) return MOE_ERR_ARG;
  MOE_TRY(check_route(T, E, k));
  return moe::launch_topk_biased(logits, bias, T, E, k, idx, gate, err, as_stream(stream));
}

int moe_capacity_ledger(const int32_t* counts, int T, int k, int E, int cf_num, int cf_den,
                        int32_t* processed, int32_t* overflow, int32_t* padding,
                        int32_t* totals, const int32_t* err, moe_stream_t stream) {
  if (!counts || !processed || !overflow || !padding || !totals || !err) return MOE_ERR_ARG;
  if (cf_num < 1 || cf_den < 1) return MOE_ERR_ARG;
  MOE_TRY(check_route(T, E, 1));
  if (k < 1 || k > E) return MOE_ERR_SHAPE;
  const long long A = (long long)T * k;
  if ((A * cf_num + (long long)E * cf_den) / ((long long)E * cf_den) >= ((long long)1 << 31))
    return MOE_ERR_SHAPE;
  return moe::launch_capacity(counts, E, A, cf_num, cf_den, processed, overflow, padding, totals,
                              err, as_stream(stream));
}

int moe_histogram_maxvio(const int32_t* idx, int T, int k, int E, int R,
                         const int32_t* expert_to_rank, int32_t* counts, int32_t* loads,
                         double* maxvio, double* balancedness, int32_t* err,
                         moe_stream_t stream) {
  if (!counts || !loads || !maxvio || !balancedness || !err || (T > 0 && !idx)) return MOE_ERR_ARG;
  MOE_TRY(check_route(T, E, k));
  MOE_TRY(check_ranks(T, k, E, R, false));
  return moe::launch_histogram(idx, T, k, E, R, expert_to_rank, counts, loads, maxvio,
                               balancedness, err, as_stream(stream));
}

int moe_plan_balanced(const int32_t* counts, int T, int k, int E, int R, int S, int32_t* plan,
                      int32_t* err, moe_stream_t stream) {
  if (!counts || !plan || !err) return MOE_ERR_ARG;
  MOE_TRY(check_route(T, E, k));
  MOE_TRY(check_ranks(T, k, E, R, true));
  MOE_TRY(check_groups(E, R, S));
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, R, S, &L));
  return moe::launch_plan(counts, T, k, E, R, S, plan, L, err, as_stream(stream));
}

int64_t moe_route_plan_workspace_words(int E) {
  if (E < 1 || E > 1024) return -1;
  return moe::route_plan_workspace_words(E);
}

int moe_route_plan(const float* logits, const float* bias, int T, int E, int k, int R, int S,
                   int32_t* idx, float* gate, int32_t* counts, int32_t* loads, double* maxvio,
                   double* balancedness, int32_t* plan, int32_t* workspace, int32_t* err,
                   moe_stream_t stream) {
  if (!err || !counts || !loads || !maxvio || !balancedness || !plan || !workspace)
    return MOE_ERR_ARG;
  if (T > 0 && (!logits || !idx || !gate)) return MOE_ERR_ARG;
  MOE_TRY(check_route(T, E, k));
  MOE_TRY(check_ranks(T, k, E, R, true));
  MOE_TRY(check_groups(E, R, S));
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, R, S, &L));
  return moe::launch_route_plan(logits, bias, T, E, k, R, S, idx, gate, counts, loads, maxvio,
                                balancedness, plan, L, workspace, err, as_stream(stream));
}

int moe_prefetch_replicas(const int32_t* plan, const moe_bf16* W1, const moe_bf16* W3,
                          const moe_f16* W2, int E, int R, int S, int d, int F,
                          moe_bf16* P1, moe_bf16* P3, moe_f16* P2, int32_t* err,
                          moe_stream_t stream) {
  if (!plan || !W1 || !W3 || !W2 || !err) return MOE_ERR_ARG;
  if (S > 0 && (!P1 || !P3 || !P2)) return MOE_ERR_ARG;
  if (E < 1 || R < 1) return MOE_ERR_ARG;
  MOE_TRY(check_ranks(0, 1, E, R, false));
  MOE_TRY(check_groups(E, R, S));
  MOE_TRY(check_dims(0, 1, d, F));
  if ((int64_t)E * d * F >= ((int64_t)1 << 40)) return MOE_ERR_SHAPE;
  if (!aligned16(W1) || !aligned16(W3) || !aligned16(W2) ||
      (S > 0 && (!aligned16(P1) || !aligned16(P3) || !aligned16(P2))))
    return MOE_ERR_ARG;
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, R, S, &L));
  return moe::launch_prefetch(plan, L, reinterpret_cast<const __nv_bfloat16*>(W1),
                              reinterpret_cast<const __nv_bfloat16*>(W3),
                              reinterpret_cast<const __half*>(W2), E, R, S, d, F,
                              reinterpret_cast<__nv_bfloat16*>(P1),
                              reinterpret_cast<__nv_bfloat16*>(P3),
                              reinterpret_cast<__half*>(P2), err, as_stream(stream));
}

int moe_dispatch(const moe_bf16* x, const int32_t* idx, const int32_t* plan, int T, int k,
                 int E, int R, int S, int d, int32_t* workspace, moe_bf16* recv,
                 int32_t* perm, int32_t* src, int32_t* err, moe_stream_t stream) {
  MOE_TRY(moe::checks::dispatch(x, idx, plan, T, k, E, R, S, d, recv, perm, src, err));
  if (T > 0 && !workspace) return MOE_ERR_ARG;
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, R, S, &L));
  return moe::launch_dispatch(reinterpret_cast<const __nv_bfloat16*>(x), idx, plan, L, T, k, E,
                              R, d, workspace, reinterpret_cast<__nv_bfloat16*>(recv), perm,
                              src, err, as_stream(stream));
}

int moe_dispatch_index(const int32_t* idx, const int32_t* plan, int T, int k, int E, int R,
                       int S, int32_t* workspace, int32_t* perm, int32_t* src, int32_t* err,
                       moe_stream_t stream) {
  if (!plan || !err) return MOE_ERR_ARG;
  if (T > 0 && (!idx || !workspace || !perm || !src)) return MOE_ERR_ARG;
  MOE_TRY(check_route(T, E, k));
  MOE_TRY(check_ranks(T, k, E, R, true));
  MOE_TRY(check_groups(E, R, S));
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, R, S, &L));
  return moe::launch_dispatch(nullptr, idx, plan, L, T, k, E, R, 0, workspace, nullptr, perm,
                              src, err, as_stream(stream));
}

int moe_grouped_ffn_gather(const moe_bf16* x, const int32_t* src, const int32_t* plan,
                           const moe_bf16* W1, const moe_bf16* W3, const moe_f16* W2,
                           const moe_bf16* P1, const moe_bf16* P3, const moe_f16* P2, int T,
                           int k, int E, int R, int S, int d, int F, moe_f16* h, moe_bf16* y,
                           int32_t* err, moe_stream_t stream) {
  if (!plan || !W1 || !W3 || !W2 || !err) return MOE_ERR_ARG;
  if (T > 0 && (!x || !src || !h || !y)) return MOE_ERR_ARG;
  if (S > 0 && (!P1 || !P3 || !P2)) return MOE_ERR_ARG;
  MOE_TRY(check_route(T, E, k));
  MOE_TRY(check_ranks(T, k, E, R, true));
  MOE_TRY(check_groups(E, R, S));
  MOE_TRY(check_dims(T, k, d, F));
  if ((int64_t)E * F >= kMaxElems || (int64_t)E * d >= kMaxElems ||
      (int64_t)R * S * F >= kMaxElems || (int64_t)R * S * d >= kMaxElems)
    return MOE_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(h) || !aligned16(y) || !aligned16(W1) || !aligned16(W3) ||
      !aligned16(W2) || (S > 0 && (!aligned16(P1) || !aligned16(P3) || !aligned16(P2))))
    return MOE_ERR_ARG;
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, R, S, &L));
  return moe::launch_grouped_ffn_gather(
      reinterpret_cast<const __nv_bfloat16*>(x), src, plan, L,
      reinterpret_cast<const __nv_bfloat16*>(W1), reinterpret_cast<const __nv_bfloat16*>(W3),
      reinterpret_cast<const __half*>(W2), reinterpret_cast<const __nv_bfloat16*>(P1),
      reinterpret_cast<const __nv_bfloat16*>(P3), reinterpret_cast<const __half*>(P2), T, k, E,
      R, S, d, F, reinterpret_cast<__half*>(h), reinterpret_cast<__nv_bfloat16*>(y), err,
      as_stream(stream));
}

int moe_grouped_ffn(const moe_bf16* recv, const int32_t* plan, const moe_bf16* W1,
                    const moe_bf16* W3, const moe_f16* W2, const moe_bf16* P1,
                    const moe_bf16* P3, const moe_f16* P2, int T, int k, int E, int R,
                    int S, int d, int F, moe_f16* h, moe_bf16* y, int32_t* err,
                    moe_stream_t stream) {
  if (!plan || !W1 || !W3 || !W2 || !err) return MOE_ERR_ARG;
  if (T > 0 && (!recv || !h || !y)) return MOE_ERR_ARG;
  if (S > 0 && (!P1 || !P3 || !P2)) return MOE_ERR_ARG;
  MOE_TRY(check_route(T, E, k));
  MOE_TRY(check_ranks(T, k, E, R, true));
  MOE_TRY(check_groups(E, R, S));
  MOE_TRY(check_dims(T, k, d, F));
  if ((int64_t)E * F >= kMaxElems || (int64_t)E * d >= kMaxElems ||
      (int64_t)R * S * F >= kMaxElems || (int64_t)R * S * d >= kMaxElems)
    return MOE_ERR_SHAPE;
  if (!aligned16(recv) || !aligned16(h) || !aligned16(y) || !aligned16(W1) || !aligned16(W3) ||
      !aligned16(W2) || (S > 0 && (!aligned16(P1) || !aligned16(P3) || !aligned16(P2))))
    return MOE_ERR_ARG;
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, R, S, &L));
  return moe::launch_grouped_ffn(
      reinterpret_cast<const __nv_bfloat16*>(recv), plan, L,
      reinterpret_cast<const __nv_bfloat16*>(W1), reinterpret_cast<const __nv_bfloat16*>(W3),
      reinterpret_cast<const __half*>(W2), reinterpret_cast<const __nv_bfloat16*>(P1),
      reinterpret_cast<const __nv_bfloat16*>(P3), reinterpret_cast<const __half*>(P2), T, k, E,
      R, S, d, F, reinterpret_cast<__half*>(h), reinterpret_cast<__nv_bfloat16*>(y), err,
      as_stream(stream));
}

int moe_grouped_ffn_combine(const moe_bf16* recv, const int32_t* plan, const moe_bf16* W1,
                            const moe_bf16* W3, const moe_f16* W2, const moe_bf16* P1,
                            const moe_bf16* P3, const moe_f16* P2, const int32_t* src,
                            const int32_t* perm, const float* gate, int T, int k, int E, int R,
                            int S, int d, int F, moe_f16* h, float* out32, moe_bf16* out,
                            int32_t* err, moe_stream_t stream) {
  if (!plan || !W1 || !W3 || !W2 || !err) return MOE_ERR_ARG;
  if (T > 0 && (!recv || !src || !perm || !gate || !h || !out32 || !out)) return MOE_ERR_ARG;
  if (S > 0 && (!P1 || !P3 || !P2)) return MOE_ERR_ARG;
  MOE_TRY(check_route(T, E, k));
  MOE_TRY(check_ranks(T, k, E, R, true));
  MOE_TRY(check_groups(E, R, S));
  MOE_TRY(check_dims(T, k, d, F));
  if ((int64_t)E * F >= kMaxElems || (int64_t)E * d >= kMaxElems ||
      (int64_t)R * S * F >= kMaxElems || (int64_t)R * S * d >= kMaxElems)
    return MOE_ERR_SHAPE;
  if (!aligned16(recv) || !aligned16(h) || !aligned16(out32) || !aligned16(out) ||
      !aligned16(W1) || !aligned16(W3) || !aligned16(W2) ||
      (S > 0 && (!aligned16(P1) || !aligned16(P3) || !aligned16(P2))))
    return MOE_ERR_ARG;
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, R, S, &L));
  return moe::launch_grouped_ffn_combine(
      reinterpret_cast<const __nv_bfloat16*>(recv), plan, L,
      reinterpret_cast<const __nv_bfloat16*>(W1), reinterpret_cast<const __nv_bfloat16*>(W3),
      reinterpret_cast<const __half*>(W2), reinterpret_cast<const __nv_bfloat16*>(P1),
      reinterpret_cast<const __nv_bfloat16*>(P3), reinterpret_cast<const __half*>(P2), src, perm,
      gate, T, k, E, R, S, d, F, reinterpret_cast<__half*>(h), out32,
      reinterpret_cast<__nv_bfloat16*>(out), err, as_stream(stream));
}

int moe_dispatch_capacity(const moe_bf16* x, const int32_t* idx, const int32_t* counts, int T,
                          int k, int E, int cap, int d, int32_t* workspace, moe_bf16* recv,
                          int32_t* perm, int32_t* src, int32_t* err, moe_stream_t stream) {
  if (!err || !counts || !recv || !src) return MOE_ERR_ARG;
  if (T > 0 && (!x || !idx || !perm || !workspace)) return MOE_ERR_ARG;
  if (cap < 0) return MOE_ERR_ARG;
  MOE_TRY(check_route(T, E, k));
  MOE_TRY(check_dims(T, k, d, 128));
  const int64_t rows = (int64_t)E * cap;
  if (rows * d >= kMaxElems) return MOE_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(recv)) return MOE_ERR_ARG;
  return moe::launch_dispatch_capacity(reinterpret_cast<const __nv_bfloat16*>(x), idx, counts, T,
                                       k, E, cap, d, workspace,
                                       reinterpret_cast<__nv_bfloat16*>(recv), perm, src, err,
                                       as_stream(stream));
}

int moe_grouped_ffn_capacity(const moe_bf16* recv, const moe_bf16* W1, const moe_bf16* W3,
                             const moe_f16* W2, int E, int cap, int d, int F, moe_f16* h,
                             moe_bf16* y, int32_t* err, moe_stream_t stream) {
  if (!W1 || !W3 || !W2 || !err) return MOE_ERR_ARG;
  if (cap > 0 && (!recv || !h || !y)) return MOE_ERR_ARG;
  if (E < 1 || cap < 0) return MOE_ERR_ARG;
  if (E > 1024) return MOE_ERR_SHAPE;
  if (d < 1 || F < 1) return MOE_ERR_ARG;
  if (d % 128 != 0 || F % 128 != 0) return MOE_ERR_SHAPE;
  const int64_t rows = (int64_t)E * cap;
  if (rows * d >= kMaxElems || rows * F >= kMaxElems) return MOE_ERR_SHAPE;
  if ((int64_t)E * F >= kMaxElems || (int64_t)E * d >= kMaxElems) return MOE_ERR_SHAPE;
  if (!aligned16(recv) || !aligned16(h) || !aligned16(y) || !aligned16(W1) || !aligned16(W3) ||
      !aligned16(W2))
    return MOE_ERR_ARG;
  return moe::launch_grouped_ffn_capacity(
      reinterpret_cast<const __nv_bfloat16*>(recv), reinterpret_cast<const __nv_bfloat16*>(W1),
      reinterpret_cast<const __nv_bfloat16*>(W3), reinterpret_cast<const __half*>(W2), E, cap, d,
      F, reinterpret_cast<__half*>(h), reinterpret_cast<__nv_bfloat16*>(y), err,
      as_stream(stream));
}

int moe_combine_capacity(const moe_bf16* y, const int32_t* perm, const float* gate, int T, int k,
                         int d, moe_bf16* out, const int32_t* err, moe_stream_t stream) {
  if (!err) return MOE_ERR_ARG;
  if (T > 0 && (!y || !perm || !gate || !out)) return MOE_ERR_ARG;
  if (T < 0 || k < 1) return MOE_ERR_ARG;
  if (k > 32) return MOE_ERR_SHAPE;
  MOE_TRY(check_dims(T, k, d, 128));
  if (!aligned16(y) || !aligned16(out)) return MOE_ERR_ARG;
  return moe::launch_combine(reinterpret_cast<const __nv_bfloat16*>(y), perm, gate, T, k, d,
                             reinterpret_cast<__nv_bfloat16*>(out), err, as_stream(stream),
                             true);
}

int moe_combine(const moe_bf16* y, const int32_t* perm, const float* gate, int T, int k, int d,
                moe_bf16* out, const int32_t* err, moe_stream_t stream) {
  if (!err) return MOE_ERR_ARG;
  if (T > 0 && (!y || !perm || !gate || !out)) return MOE_ERR_ARG;
  if (T < 0 || k < 1) return MOE_ERR_ARG;
  if (k > 32) return MOE_ERR_SHAPE;
  MOE_TRY(check_dims(T, k, d, 128));
  if (!aligned16(y) || !aligned16(out)) return MOE_ERR_ARG;
  return moe::launch_combine(reinterpret_cast<const __nv_bfloat16*>(y), perm, gate, T, k, d,
                             reinterpret_cast<__nv_bfloat16*>(out), err, as_stream(stream));
}

int moe_combine_backward(const moe_bf16* dout, const moe_bf16* y, const int32_t* perm,
                         const float* gate, int T, int k, int d, moe_bf16* dy, float* dgate,
                         const int32_t* err, moe_stream_t stream) {
  if (!err) return MOE_ERR_ARG;
  if (T > 0 && (!dout || !y || !perm || !gate || !dy || !dgate)) return MOE_ERR_ARG;
  if (T < 0 || k < 1) return MOE_ERR_ARG;
  if (k > 32) return MOE_ERR_SHAPE;
  MOE_TRY(check_dims(T, k, d, 128));
  if (!aligned16(dout) || !aligned16(y) || !aligned16(dy)) return MOE_ERR_ARG;
  return moe::launch_combine_backward(reinterpret_cast<const __nv_bfloat16*>(dout),
                                      reinterpret_cast<const __nv_bfloat16*>(y), perm, gate, T,
                                      k, d, reinterpret_cast<__nv_bfloat16*>(dy), dgate, err,
                                      as_stream(stream));
}

int moe_dispatch_backward(const moe_bf16* dx_rows, const int32_t* perm, int T, int k, int d,
                          moe_bf16* dx, const int32_t* err, moe_stream_t stream) {
  if (!err) return MOE_ERR_ARG;
  if (T > 0 && (!dx_rows || !perm || !dx)) return MOE_ERR_ARG;
  if (T < 0 || k < 1) return MOE_ERR_ARG;
  if (k > 32) return MOE_ERR_SHAPE;
  MOE_TRY(check_dims(T, k, d, 128));
  if (!aligned16(dx_rows) || !aligned16(dx)) return MOE_ERR_ARG;
  return moe::launch_combine(reinterpret_cast<const __nv_bfloat16*>(dx_rows), perm, nullptr, T,
                             k, d, reinterpret_cast<__nv_bfloat16*>(dx), err, as_stream(stream));
}

int moe_topk_backward(const float* gate, const float* dgate, const int32_t* idx, int T, int E,
                      int k, float* dlogits, const int32_t* err, moe_stream_t stream) {
  if (!err) return MOE_ERR_ARG;
  if (T > 0 && (!gate || !dgate || !idx || !dlogits)) return MOE_ERR_ARG;
  MOE_TRY(check_route(T, E, k));
  return moe::launch_topk_backward(gate, dgate, idx, T, E, k, dlogits, err, as_stream(stream));
}

int64_t moe_ffn_backward_workspace_bytes(int T, int k, int E, int R, int S, int d, int F) {
  if (T < 0 || k < 1 || E < 1 || R < 1 || S < 0 || d < 1 || F < 1 || E % R != 0) return -1;
  moe_plan_layout L;
  if (moe_plan_get_layout(E, R, S, &L) != MOE_OK) return -1;
  return moe::ffn_backward_workspace_bytes(T, k, E, R, S, d, F, R * L.max_groups_per_rank);
}

int moe_grouped_ffn_backward(const moe_bf16* recv, const moe_bf16* dy, const moe_f16* h,
                             const int32_t* plan, const moe_bf16* W1, const moe_bf16* W3,
                             const moe_f16* W2, int T, int k, int E, int R, int S, int d, int F,
                             moe_bf16* dx_rows, float* dW1, float* dW3, float* dW2,
                             void* workspace, int64_t workspace_bytes, int32_t* err,
                             moe_stream_t stream) {
  if (!plan || !W1 || !W3 || !W2 || !err || !dW1 || !dW3 || !dW2) return MOE_ERR_ARG;
  if (T > 0 && (!recv || !dy || !dx_rows || !workspace)) return MOE_ERR_ARG;  // h may be NULL
  MOE_TRY(check_route(T, E, k));
  MOE_TRY(check_ranks(T, k, E, R, true));
  MOE_TRY(check_groups(E, R, S));
  MOE_TRY(check_dims(T, k, d, F));
  if ((int64_t)E * F >= kMaxElems || (int64_t)E * d >= kMaxElems) return MOE_ERR_SHAPE;
  if ((int64_t)T * k * 2 * F >= kMaxElems) return MOE_ERR_SHAPE;
  if (!aligned16(recv) || !aligned16(dy) || !aligned16(h) || !aligned16(dx_rows) ||
      !aligned16(W1) || !aligned16(W3) || !aligned16(W2) || !aligned16(dW1) || !aligned16(dW3) ||
      !aligned16(dW2) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return MOE_ERR_ARG;
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, R, S, &L));
  if (moe::ffn_backward_workspace_bytes(T, k, E, R, S, d, F, R * L.max_groups_per_rank) >
      workspace_bytes)
    return MOE_ERR_ARG;
  return moe::launch_grouped_ffn_backward(
      reinterpret_cast<const __nv_bfloat16*>(recv), reinterpret_cast<const __nv_bfloat16*>(dy),
      reinterpret_cast<const __half*>(h), plan, L, reinterpret_cast<const __nv_bfloat16*>(W1),
      reinterpret_cast<const __nv_bfloat16*>(W3), reinterpret_cast<const __half*>(W2), T, k, E,
      R, S, d, F, reinterpret_cast<__nv_bfloat16*>(dx_rows), dW1, dW3, dW2, workspace,
      workspace_bytes, err, as_stream(stream));
}

// ------------------------------------------------------- expert parallelism across GPUs

int moe_ep_counts(const int32_t* idx, int T, int k, int E, const int32_t* err, int32_t* send,
                  moe_stream_t stream) {
  if (!err || !send) return MOE_ERR_ARG;
  if (T > 0 && !idx) return MOE_ERR_ARG;
  MOE_TRY(check_route(T, E, k));
  return moe::launch_ep_counts(idx, T, k, E, err, send, as_stream(stream));
}

int moe_ep_plan(const int32_t* gathered, int W, int me, int T, int k, int E, int S,
                int32_t* counts, int32_t* q_base, int32_t* loads, double* maxvio,
                double* balancedness, int32_t* plan, int32_t* err, moe_stream_t stream) {
  if (!gathered || !counts || !q_base || !loads || !maxvio || !balancedness || !plan || !err)
    return MOE_ERR_ARG;
  MOE_TRY(check_ep(W, me, T, k, E, S));
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, W, S, &L));
  return moe::launch_ep_plan(gathered, W, me, T, k, E, S, counts, q_base, loads, maxvio,
                             balancedness, plan, L, err, as_stream(stream));
}

int moe_ep_prefetch(const int32_t* plan, const moe_bf16* const* W1_ranks,
                    const moe_bf16* const* W3_ranks, const moe_f16* const* W2_ranks, int W,
                    int me, int E, int S, int d, int F, moe_bf16* P1, moe_bf16* P3, moe_f16* P2,
                    int32_t* err, moe_stream_t stream) {
  if (!plan || !err) return MOE_ERR_ARG;
  MOE_TRY(check_ep(W, me, 0, 1, E, S));
  MOE_TRY(check_dims(0, 1, d, F));
  if ((int64_t)(E / W) * d * F >= kMaxElems || (int64_t)S * d * F >= kMaxElems)
    return MOE_ERR_SHAPE;
  if (S == 0) return MOE_OK;
  MOE_TRY(check_table(W1_ranks, W));
  MOE_TRY(check_table(W3_ranks, W));
  MOE_TRY(check_table(W2_ranks, W));
  if (!P1 || !P3 || !P2 || !aligned16(P1) || !aligned16(P3) || !aligned16(P2)) return MOE_ERR_ARG;
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, W, S, &L));
  return moe::launch_ep_prefetch(
      plan, L, reinterpret_cast<const __nv_bfloat16* const*>(W1_ranks),
      reinterpret_cast<const __nv_bfloat16* const*>(W3_ranks),
      reinterpret_cast<const __half* const*>(W2_ranks), W, me, E, S, d, F,
      reinterpret_cast<__nv_bfloat16*>(P1), reinterpret_cast<__nv_bfloat16*>(P3),
      reinterpret_cast<__half*>(P2), err, as_stream(stream));
}

int moe_ep_dispatch(const moe_bf16* x, const int32_t* idx, const int32_t* q_base,
                    const int32_t* plan, int W, int T, int k, int E, int S, int d,
                    int32_t* workspace, moe_bf16* const* recv_ranks, int32_t* perm,
                    int32_t* err, moe_stream_t stream) {
  if (!plan || !q_base || !err) return MOE_ERR_ARG;
  if (T > 0 && (!x || !idx || !workspace || !perm)) return MOE_ERR_ARG;
  MOE_TRY(check_ep(W, 0, T, k, E, S));
  MOE_TRY(check_dims(T, k, d, 128));
  if (T > 0) {
    MOE_TRY(check_table(recv_ranks, W));
    if (!aligned16(x)) return MOE_ERR_ARG;
  }
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, W, S, &L));
  return moe::launch_ep_dispatch(reinterpret_cast<const __nv_bfloat16*>(x), idx, q_base, plan, L,
                                 T, k, E, W, d, workspace,
                                 reinterpret_cast<__nv_bfloat16* const*>(recv_ranks), perm, err,
                                 as_stream(stream));
}

int moe_ep_grouped_ffn(const moe_bf16* recv, const int32_t* plan, int W, int me,
                       const moe_bf16* W1, const moe_bf16* W3, const moe_f16* W2,
                       const moe_bf16* P1, const moe_bf16* P3, const moe_f16* P2, int T, int k,
                       int E, int S, int d, int F, int32_t* groups_ws, moe_f16* h, moe_bf16* y,
                       int32_t* err, moe_stream_t stream) {
  if (!plan || !W1 || !W3 || !W2 || !groups_ws || !err) return MOE_ERR_ARG;
  if (T > 0 && (!recv || !h || !y)) return MOE_ERR_ARG;
  if (S > 0 && (!P1 || !P3 || !P2)) return MOE_ERR_ARG;
  MOE_TRY(check_ep(W, me, T, k, E, S));
  MOE_TRY(check_dims(T, k, d, F));
  const int B = E / W;
  if ((int64_t)B * F >= kMaxElems || (int64_t)B * d >= kMaxElems ||
      (int64_t)S * F >= kMaxElems || (int64_t)S * d >= kMaxElems)
    return MOE_ERR_SHAPE;
  if (!aligned16(recv) || !aligned16(h) || !aligned16(y) || !aligned16(W1) || !aligned16(W3) ||
      !aligned16(W2) || !aligned16(groups_ws) ||
      (S > 0 && (!aligned16(P1) || !aligned16(P3) || !aligned16(P2))))
    return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, W, S, &L));
  const int C = T * k;
  cudaStream_t s = as_stream(stream);
  MOE_TRY(moe::launch_ep_groups(plan, L, me, E, W, S, C, groups_ws, err, s));
  return moe::launch_grouped_ffn_groups(
      reinterpret_cast<const __nv_bfloat16*>(recv), groups_ws, B + S, C,
      reinterpret_cast<const __nv_bfloat16*>(W1), reinterpret_cast<const __nv_bfloat16*>(W3),
      reinterpret_cast<const __half*>(W2), reinterpret_cast<const __nv_bfloat16*>(P1),
      reinterpret_cast<const __nv_bfloat16*>(P3), reinterpret_cast<const __half*>(P2), B, S, d,
      F, reinterpret_cast<__half*>(h), reinterpret_cast<__nv_bfloat16*>(y), err, s);
}

int moe_ep_combine(const moe_bf16* const* y_ranks, const int32_t* perm, const float* gate,
                   int W, int T, int k, int d, moe_bf16* out, const int32_t* err,
                   moe_stream_t stream) {
  if (!err) return MOE_ERR_ARG;
  if (T > 0 && (!perm || !gate || !out)) return MOE_ERR_ARG;
  if (W < 1 || T < 0 || k < 1) return MOE_ERR_ARG;
  if (W > MOE_EP_MAX_RANKS || k > 32) return MOE_ERR_SHAPE;
  if ((int64_t)W * T * k >= kMaxElems) return MOE_ERR_SHAPE;
  MOE_TRY(check_dims(T, k, d, 128));
  if (T == 0) return MOE_OK;
  MOE_TRY(check_table(y_ranks, W));
  if (!aligned16(out)) return MOE_ERR_ARG;
  return moe::launch_ep_combine(reinterpret_cast<const __nv_bfloat16* const*>(y_ranks), W, perm,
                                gate, T, k, d, reinterpret_cast<__nv_bfloat16*>(out), err,
                                as_stream(stream));
}

int moe_ep_combine_backward(const moe_bf16* dout, const moe_bf16* const* y_ranks,
                            const int32_t* perm, const float* gate, int W, int T, int k, int d,
                            moe_bf16* const* dy_ranks, float* dgate, const int32_t* err,
                            moe_stream_t stream) {
  if (!err) return MOE_ERR_ARG;
  if (T > 0 && (!dout || !perm || !gate || !dgate)) return MOE_ERR_ARG;
  if (W < 1 || T < 0 || k < 1) return MOE_ERR_ARG;
  if (W > MOE_EP_MAX_RANKS || k > 32) return MOE_ERR_SHAPE;
  if ((int64_t)W * T * k >= kMaxElems) return MOE_ERR_SHAPE;
  MOE_TRY(check_dims(T, k, d, 128));
  if (T == 0) return MOE_OK;
  MOE_TRY(check_table(y_ranks, W));
  MOE_TRY(check_table(dy_ranks, W));
  if (!aligned16(dout)) return MOE_ERR_ARG;
  return moe::launch_ep_combine_backward(
      reinterpret_cast<const __nv_bfloat16*>(dout),
      reinterpret_cast<const __nv_bfloat16* const*>(y_ranks), perm, gate, W, T, k, d,
      reinterpret_cast<__nv_bfloat16* const*>(dy_ranks), dgate, err, as_stream(stream));
}

int64_t moe_ep_ffn_backward_workspace_bytes(int T, int k, int E, int W, int S, int d, int F) {
  if (check_ep(W, 0, T, k, E, S) != MOE_OK || check_dims(T, k, d, F) != MOE_OK) return -1;
  if (E / W + S > 1024) return -1;
  return moe::ep_ffn_backward_workspace_bytes(T, k, E, W, S, d, F);
}

int moe_ep_grouped_ffn_backward(const moe_bf16* recv, const moe_bf16* dy, const int32_t* plan,
                                int W, int me, const moe_bf16* W1, const moe_bf16* W3,
                                const moe_f16* W2, const moe_bf16* P1, const moe_bf16* P3,
                                const moe_f16* P2, int T, int k, int E, int S, int d, int F,
                                int32_t* groups_ws, moe_bf16* dx_rows, float* dP1, float* dP3,
                                float* dP2, void* workspace, int64_t workspace_bytes,
                                int32_t* err, moe_stream_t stream) {
  if (!plan || !W1 || !W3 || !W2 || !groups_ws || !err || !dP1 || !dP3 || !dP2)
    return MOE_ERR_ARG;
  if (T > 0 && (!recv || !dy || !dx_rows || !workspace)) return MOE_ERR_ARG;
  if (S > 0 && (!P1 || !P3 || !P2)) return MOE_ERR_ARG;
  MOE_TRY(check_ep(W, me, T, k, E, S));
  MOE_TRY(check_dims(T, k, d, F));
  const int B = E / W;
  if (B + S > 1024) return MOE_ERR_SHAPE;
  if ((int64_t)(B + S) * F * d >= kMaxElems || (int64_t)T * k * 2 * F >= kMaxElems)
    return MOE_ERR_SHAPE;
  if (!aligned16(recv) || !aligned16(dy) || !aligned16(dx_rows) || !aligned16(W1) ||
      !aligned16(W3) || !aligned16(W2) || !aligned16(groups_ws) || !aligned16(dP1) ||
      !aligned16(dP3) || !aligned16(dP2) ||
      (S > 0 && (!aligned16(P1) || !aligned16(P3) || !aligned16(P2))) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return MOE_ERR_ARG;
  if (moe::ep_ffn_backward_workspace_bytes(T, k, E, W, S, d, F) > workspace_bytes)
    return MOE_ERR_ARG;
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, W, S, &L));
  cudaStream_t s = as_stream(stream);
  const int C = T * k;
  if (T > 0) MOE_TRY(moe::launch_ep_groups(plan, L, me, E, W, S, C, groups_ws, err, s));
  return moe::launch_ep_grouped_ffn_backward(
      reinterpret_cast<const __nv_bfloat16*>(recv), reinterpret_cast<const __nv_bfloat16*>(dy),
      groups_ws, B, S, C, reinterpret_cast<const __nv_bfloat16*>(W1),
      reinterpret_cast<const __nv_bfloat16*>(W3), reinterpret_cast<const __half*>(W2),
      reinterpret_cast<const __nv_bfloat16*>(P1), reinterpret_cast<const __nv_bfloat16*>(P3),
      reinterpret_cast<const __half*>(P2), d, F, reinterpret_cast<__nv_bfloat16*>(dx_rows), dP1,
      dP3, dP2, workspace, workspace_bytes, err, s);
}

int moe_ep_reduce_home(const int32_t* plan, float* const* dP1_ranks, float* const* dP3_ranks,
                       float* const* dP2_ranks, int W, int me, int E, int S, int d, int F,
                       const int32_t* err, moe_stream_t stream) {
  if (!plan || !err) return MOE_ERR_ARG;
  MOE_TRY(check_ep(W, me, 0, 1, E, S));
  MOE_TRY(check_dims(0, 1, d, F));
  if ((int64_t)(E / W + S) * F * d >= kMaxElems) return MOE_ERR_SHAPE;
  MOE_TRY(check_table(dP1_ranks, W));
  MOE_TRY(check_table(dP3_ranks, W));
  MOE_TRY(check_table(dP2_ranks, W));
  moe_plan_layout L;
  MOE_TRY(moe_plan_get_layout(E, W, S, &L));
  return moe::launch_ep_reduce_home(plan, L, dP1_ranks, dP3_ranks, dP2_ranks, W, me, E, S, d, F,
                                    err, as_stream(stream));
}

int moe_ep_dispatch_backward(const moe_bf16* const* dx_rows_ranks, const int32_t* perm, int W,
                             int T, int k, int d, moe_bf16* dx, const int32_t* err,
                             moe_stream_t stream) {
  if (!err) return MOE_ERR_ARG;
  if (T > 0 && (!perm || !dx)) return MOE_ERR_ARG;
  if (W < 1 || T < 0 || k < 1) return MOE_ERR_ARG;
  if (W > MOE_EP_MAX_RANKS || k > 32) return MOE_ERR_SHAPE;
  if ((int64_t)W * T * k >= kMaxElems) return MOE_ERR_SHAPE;
  MOE_TRY(check_dims(T, k, d, 128));
  if (T == 0) return MOE_OK;
  MOE_TRY(check_table(dx_rows_ranks, W));
  if (!aligned16(dx)) return MOE_ERR_ARG;
  return moe::launch_ep_combine(reinterpret_cast<const __nv_bfloat16* const*>(dx_rows_ranks), W,
                                perm, nullptr, T, k, d, reinterpret_cast<__nv_bfloat16*>(dx), err,
                                as_stream(stream));
}

int moe_w2_to_f16(const moe_bf16* w2_bf16, int64_t n, moe_f16* w2_f16, moe_stream_t stream) {
  if (n < 0 || (n > 0 && (!w2_bf16 || !w2_f16))) return MOE_ERR_ARG;
  if (n % 8 != 0) return MOE_ERR_SHAPE;
  if (!aligned16(w2_bf16) || !aligned16(w2_f16)) return MOE_ERR_ARG;
  return moe::launch_bf16_to_f16(reinterpret_cast<const __nv_bfloat16*>(w2_bf16), n,
                                 reinterpret_cast<__half*>(w2_f16), as_stream(stream));
}

int moe_set_ffn_tile_mode(int mode) { return moe::set_ffn_tile_mode(mode); }

int moe_ffn_tile_mode(void) { return moe::ffn_tile_mode(); }

int moe_ffn_pair_clusters(void) { return moe::ffn_pair_clusters(); }

int moe_selftest_bounded_wait(int32_t* err, int limit_us, moe_stream_t stream) {
  if (!err || limit_us < 1 || limit_us > 10000000) return MOE_ERR_ARG;
  return moe::launch_bounded_wait_selftest(err, limit_us, as_stream(stream));
}

}  // extern "C"
