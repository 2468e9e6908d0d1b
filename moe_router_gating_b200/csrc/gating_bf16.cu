// The bf16 instances of the fused gating kernels and their launches, and the
// split-H cluster capacity query.
#include "gating_launch_impl.cuh"

namespace tkg {

template bool set_up_gating_kernels<false>();
template tk_status launch_planned<false>(const tk_gating_plan&, const LaunchEnv&, const CUtensorMap&,
                                         const CUtensorMap&, const CUtensorMap&, int64_t, int64_t, int64_t, int32_t,
                                         float*, int32_t*, const float*, const float*, float*, cudaStream_t);

void measure_split_cluster_capacity(int counts[4]) {
  for (int i = 1; i <= 4; ++i) {
    const int C = 1 << i;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C);
    cfg.blockDim = dim3(SPLIT_THREADS);
    cfg.dynamicSmemBytes = kMaxDynamicSmem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    const cudaError_t e = C == 16 ? cudaOccupancyMaxActiveClusters(&n, gating_split_h_kernel<8, 16, false>, &cfg)
                                  : cudaOccupancyMaxActiveClusters(&n, gating_split_h_kernel<8, 8, false>, &cfg);
    if (e != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    counts[i - 1] = n;
  }
}

}  // namespace tkg
