// gemm_tc.cu -- bf16 grouped GEMMs (placeholder delegating to the CUDA-core kernels
// until the tcgen05 kernels are in).
#include "common.cuh"

namespace smoe {
int simt_tile_cols();

bool tc_supported() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10;
}
int tc_tile_cols() { return simt_tile_cols(); }
cudaError_t launch_grouped_gemm_tc(const GroupedGemm& g, cudaStream_t s) {
  return launch_grouped_gemm_simt(g, SMOE_BF16, s);
}
cudaError_t launch_dw_gemm_tc(const DwGemm& g, cudaStream_t s) { return launch_dw_gemm_simt(g, SMOE_BF16, s); }
}  // namespace smoe
