// Empty kernel chained like the library's kernels (programmatic dependent launch), for
// measuring the launch floor of a CUDA graph: the cost of a step whose kernels do nothing.
#include "pbd_common.cuh"
#include "pbd_kernels.h"

namespace la {
namespace {

__global__ void noop_kernel() {
  pdl_trigger();
  pdl_wait();
}

}  // namespace

cudaError_t launch_noop(int ctas, int threads, cudaStream_t stream) {
  return launch_pdl(noop_kernel, dim3(ctas), dim3(threads), 0, stream);
}

}  // namespace la
