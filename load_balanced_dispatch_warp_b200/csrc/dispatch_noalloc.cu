// moe_dispatch_noalloc: moe_dispatch with the library's own static scratch instead of a
// caller workspace.
//
// Some callers cannot allocate device memory when they dispatch: an operator or plugin
// interface of another runtime that hands the library only its input and output buffers,
// or a host program whose hot path must not call cudaMalloc (cudaMalloc may synchronise
// the device and stalls every stream).  This entry point needs nothing beyond the buffers
// moe_dispatch already takes as inputs and outputs: the dispatch workspace lives in a
// file-scope device array of MOE_NOALLOC_SCRATCH_WORDS int32 words, which every GPU that
// loads the library holds until the process exits.
//
// In host code the array's name is only a host-side stand-in, so its device address is
// looked up with cudaGetSymbolAddress, with the device current, on the first call in each
// CUDA context (per device, keyed by the driver's context id, so a cudaDeviceReset --
// which ends the context and may move the array -- makes the next call look it up again);
// that first call should be made before any stream capture.  Every call shares the one
// array and leaves its contents behind; the dispatch clears what it needs cleared itself.
// Calls that overlap on the GPU (two streams, or two host threads on one device) race on
// the array.
#include <cuda.h>

#include <mutex>

#include "checks.cuh"
#include "common.cuh"

namespace {

__device__ __align__(256) int32_t g_dispatch_scratch[MOE_NOALLOC_SCRATCH_WORDS];

constexpr int kMaxDevices = 64;
struct ScratchEntry {
  unsigned long long ctx_id;
  int32_t* ptr;
};
ScratchEntry g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Driver id of the current context (unique within the process, never reused), 0 if none.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array in the current context of the current device.
int scratch_for_current_device(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  unsigned long long id = current_context_id();
  ScratchEntry& ent = g_scratch[dev];
  if (id == 0 || ent.ptr == nullptr || ent.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return MOE_ERR_DEVICE;
    }
    if (id == 0) id = current_context_id();  // the lookup made the context current
    ent.ptr = static_cast<int32_t*>(p);
    ent.ctx_id = id;
  }
  *out = ent.ptr;
  return MOE_OK;
}

}  // namespace

extern "C" int moe_dispatch_noalloc(const moe_bf16* x, const int32_t* idx, const int32_t* plan,
                                    int T, int k, int E, int R, int S, int d, moe_bf16* recv,
                                    int32_t* perm, int32_t* src, int32_t* err,
                                    moe_stream_t stream) {
  // moe_dispatch's argument rules (the same function), then the scratch limit
  const int st = moe::checks::dispatch(x, idx, plan, T, k, E, R, S, d, recv, perm, src, err);
  if (st != MOE_OK) return st;
  if (moe_dispatch_workspace_words(T, E) > MOE_NOALLOC_SCRATCH_WORDS) return MOE_ERR_SHAPE;
  moe_plan_layout L;
  const int lst = moe_plan_get_layout(E, R, S, &L);
  if (lst != MOE_OK) return lst;
  int32_t* scratch = nullptr;
  const int sst = scratch_for_current_device(&scratch);
  if (sst != MOE_OK) return sst;
  return moe::launch_dispatch(reinterpret_cast<const __nv_bfloat16*>(x), idx, plan, L, T, k, E,
                              R, d, scratch, reinterpret_cast<__nv_bfloat16*>(recv), perm, src,
                              err, reinterpret_cast<cudaStream_t>(stream));
}
