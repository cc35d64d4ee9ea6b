// moe_dispatch_noalloc: moe_dispatch with the library's own static scratch instead of a
// caller workspace.
//
// Some callers cannot allocate device memory when they dispatch: an operator or plugin
// interface of another runtime that hands the library only its input and output buffers,
// or a host program whose hot path must not call cudaMalloc (cudaMalloc may synchronise
// the device and stalls every stream).  This entry point needs nothing beyond the buffers
// moe_dispatch already takes as inputs and outputs: the per-tile expert counts of the
// placement pass live in a file-scope device array of MOE_NOALLOC_SCRATCH_WORDS int32
// words (1 MiB), which every GPU that loads the library holds until the process exits.
//
// The array's name is only a host-side stand-in in host code, so the first call on each
// device looks up its device address with cudaGetSymbolAddress (with that device
// current) and keeps it; that first call should be made before any stream capture.
// Every call shares the one array and leaves its contents behind; nothing in it has to
// start at zero, because the count pass writes every word the rank pass reads within the
// same call.  Calls that overlap on the GPU (two streams, or two host threads on one
// device) race on the array.
#include <mutex>

#include "common.cuh"

namespace {

__device__ __align__(256) int32_t g_dispatch_scratch[MOE_NOALLOC_SCRATCH_WORDS];

constexpr int kMaxDevices = 64;
int32_t* g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (looked up once per device).
int scratch_for_current_device(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return MOE_ERR_DEVICE;
    }
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" int moe_dispatch_noalloc(const moe_bf16* x, const int32_t* idx, const int32_t* plan,
                                    int T, int k, int E, int R, int S, int d, moe_bf16* recv,
                                    int32_t* perm, int32_t* src, int32_t* err,
                                    moe_stream_t stream) {
  // same argument rules as moe_dispatch, plus the scratch limit
  if (!plan || !err) return MOE_ERR_ARG;
  if (T > 0 && (!x || !idx || !recv || !perm || !src)) return MOE_ERR_ARG;
  if (T < 0 || E < 1 || k < 1 || R < 1 || S < 0 || d < 1) return MOE_ERR_ARG;
  if (E > 1024 || k > E || k > 32 || R > E || E % R != 0 || ((int64_t)T * k) % R != 0)
    return MOE_ERR_SHAPE;
  if ((int64_t)R * (E / R + S) > 4096 || d % 128 != 0) return MOE_ERR_SHAPE;
  const int64_t rows = (int64_t)T * k;
  if ((int64_t)T * E >= ((int64_t)1 << 31) || rows * d >= ((int64_t)1 << 31) ||
      (int64_t)T * d >= ((int64_t)1 << 31))
    return MOE_ERR_SHAPE;
  if (moe_dispatch_workspace_words(T, E) > MOE_NOALLOC_SCRATCH_WORDS) return MOE_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(recv) & 15u))
    return MOE_ERR_ARG;
  moe_plan_layout L;
  const int st = moe_plan_get_layout(E, R, S, &L);
  if (st != MOE_OK) return st;
  int32_t* scratch = nullptr;
  const int sst = scratch_for_current_device(&scratch);
  if (sst != MOE_OK) return sst;
  return moe::launch_dispatch(reinterpret_cast<const __nv_bfloat16*>(x), idx, plan, L, T, k, E,
                              R, d, scratch, reinterpret_cast<__nv_bfloat16*>(recv), perm, src,
                              err, reinterpret_cast<cudaStream_t>(stream));
}
