// dense.cu -- placeholder entry points for the tanh RNN (dense DEER / quasi-DEER) and
// the dense standalone scan; replaced by the real kernels.
#include "internal.h"
namespace prn {
int newton_tanh_plan(const NewtonTanhReq &, int, Plan *) { return 1; }
cudaError_t newton_tanh_launch(const NewtonTanhReq &, const Plan &, const Work &, const DbgHost &, cudaStream_t) {
    return cudaErrorNotSupported;
}
int scan_dense_plan(const ScanReq &, int, Plan *) { return 1; }
cudaError_t scan_dense_launch(const ScanReq &, const Plan &, const Work &, const DbgHost &, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace prn
