// The FP8 (E4M3) instances of the fused gating kernels and their launches.
#include "gating_launch_impl.cuh"

namespace tkg {

template bool set_up_gating_kernels<true>();
template tk_status launch_planned<true>(const tk_gating_plan&, const LaunchEnv&, const CUtensorMap&,
                                        const CUtensorMap&, const CUtensorMap&, int64_t, int64_t, int64_t, int32_t,
                                        float*, int32_t*, const float*, const float*, float*, cudaStream_t);

}  // namespace tkg
