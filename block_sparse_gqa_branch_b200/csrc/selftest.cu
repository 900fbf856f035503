// selftest.cu -- a kernel whose only wait can never complete, to exercise the bounded-wait
// failure path that every kernel of the library shares: the wait gives up after its limit,
// records MSA_ERR_TIMEOUT in the workspace's error word, and the kernel returns.
#include "msa_common.cuh"

namespace msa {

__global__ void __launch_bounds__(32) selftest_timeout_kernel(WsHeader* hdr) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, hdr, KID_SELFTEST);   // nothing arrives on `bar`
}

}  // namespace msa

extern "C" msa_status_t msa_selftest_wait_timeout(void* workspace, size_t workspace_bytes, msa_stream_t stream) {
    MSA_CALL_RANGE();
    using namespace msa;
    if (workspace == nullptr || workspace_bytes < sizeof(WsHeader) || !aligned16(workspace)) return MSA_ERR_WORKSPACE;
    const KernelTimer kt(KID_SELFTEST, reinterpret_cast<cudaStream_t>(stream));
    selftest_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<WsHeader*>(workspace));
    return cuda_status();
}
