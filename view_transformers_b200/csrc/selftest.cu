// Self-check of the bounded waits used by the tensor-core kernels: one thread waits on an
// mbarrier that nothing arrives on. The wait gives up after its limit, records
// BSA_ERR_TIMEOUT in the status word and the kernel returns normally, which is the same
// exit every producer / MMA / softmax wait of the attention kernel takes on a timeout.
#include "common.cuh"
#include "sm100.cuh"

namespace bsa {
namespace {

__global__ void wait_timeout_kernel(int32_t* status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::fence_mbar_init();
        abort_flag = 0;
        // phase 0 of a fresh barrier with one expected arrival: it never completes
        sm100::mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
    }
}

}  // namespace

cudaError_t launch_wait_timeout(int32_t* status, uint64_t limit_ns, cudaStream_t st) {
    wait_timeout_kernel<<<1, 32, 0, st>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace bsa
