// Stand-alone plan call: one CTA runs plan_block (plan_body.cuh) on the histogram's counts.
#include "plan_body.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t* __restrict__ counts,
                                                            int T, int k, int E, int R, int S,
                                                            int32_t* __restrict__ plan,
                                                            moe_plan_layout L,
                                                            int32_t* __restrict__ err) {
  extern __shared__ int s_plan[];  // plan_smem_words(E, R)
  if (block_should_stop(err)) return;
  plan_block(counts, T, k, E, R, S, plan, L, err, s_plan);
}

}  // namespace

int launch_plan(const int32_t* counts, int T, int k, int E, int R, int S, int32_t* plan,
                const moe_plan_layout& L, int32_t* err, cudaStream_t s) {
  plan_kernel<<<1, kPlanThreads, sizeof(int) * plan_smem_words(E, R), s>>>(counts, T, k, E, R,
                                                                         S, plan, L, err);
  return launch_status();
}

}  // namespace moe
