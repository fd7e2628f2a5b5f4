// selftest.cu -- kda_selftest_bounded_wait: runs the failure path of the
// library's bounded mbarrier waits on purpose, without any GPU fault.
//
// Every kernel of the library that waits on an mbarrier (the bf16 prefill's
// prep and chain, the backward chains, the serving decode) polls it a bounded
// number of times; when the bound runs out it sets the device error word to
// kErrWaitTimeout and leaves, instead of spinning forever or trapping.  This
// entry point launches one CTA whose thread 0 waits, with the caller's bound,
// on an mbarrier that nothing ever arrives on -- no copy or MMA is in flight
// -- so the host can check that such a timeout reaches kda_get_device_error()
// and that the context stays usable afterwards.
#include "../../include/kda.h"
#include "api_internal.h"
#include "sm100.cuh"

namespace {

__global__ void bounded_wait_kernel(uint32_t limit, int *err) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        kda::sm100::mbar_init(&bar, 1);
        kda::sm100::fence_mbar_init();
        // phase 0 needs one arrival, which never comes
        if (!kda::sm100::mbar_wait(&bar, 0, limit)) kda::set_device_error(err, kda::kErrWaitTimeout);
    }
}

}  // namespace

extern "C" kda_status kda_selftest_bounded_wait(unsigned limit, void *stream) {
    kda::t_msg[0] = 0;
    if (limit == 0 || limit > (1u << 16))
        return kda::fail(KDA_ERR_INVALID_ARG, "kda_selftest_bounded_wait: limit %u out of [1, 65536]",
                         limit);
    int *err = kda::error_word();
    if (!err) return kda::fail(KDA_ERR_CUDA, "kda_selftest_bounded_wait: no device error word");
    bounded_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit, err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return kda::fail(KDA_ERR_CUDA, "kda_selftest_bounded_wait launch: %s", cudaGetErrorString(e));
    return KDA_OK;
}
