// pre_cluster_tc.cu -- thread-block-cluster tensor-core kernel for the mHC pre stage.
// (Not yet enabled: the shape test rejects every problem, so MHC_PRE_AUTO takes the
// generic kernel.)
#include "launch.cuh"

namespace mhc {

bool pre_cluster_tc_shape_ok(int64_t, int, int, DType) { return false; }
bool pre_cluster_tc_device_ok() { return false; }
cudaError_t launch_pre_cluster_tc(const PreArgs&) { return cudaErrorNotSupported; }

}  // namespace mhc
