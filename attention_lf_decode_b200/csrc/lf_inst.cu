// One variant of the fused decode kernel, compiled once per (KV storage,
// kernel mode) pair with -DLF_KVB=<2|1> -DLF_MODE=<0|1|2>: its launch
// planning and launching for every head dim and group size.
#include "lf_kernel.cuh"

#if !defined(LF_KVB) || !defined(LF_MODE)
#error "compile with -DLF_KVB=<bytes per element> -DLF_MODE=<kernel mode>"
#endif

#define LF_NAME3(a, k, m) a##_kv##k##_m##m
#define LF_NAME2(a, k, m) LF_NAME3(a, k, m)
#define LF_NAME(a) LF_NAME2(a, LF_KVB, LF_MODE)

namespace lf {

cudaError_t LF_NAME(plan)(int D, int G, const PlanIn& in, int budget, Plan* out) {
  cudaError_t e = cudaErrorInvalidValue;
  LF_DISPATCH(D, G, (e = plan_t<DD, GG, LF_MODE, LF_KVB>(in, budget, out)));
  return e;
}

cudaError_t LF_NAME(launch)(int D, int G, const Params& p, const Plan& pl, cudaStream_t st) {
  cudaError_t e = cudaErrorInvalidValue;
  LF_DISPATCH(D, G, (e = launch_t<DD, GG, LF_MODE, LF_KVB>(p, pl, st)));
  return e;
}

}  // namespace lf
