// prefill_sm100.cu -- fp16/bf16 prefill on tcgen05 tensor cores (placeholder
// until the TMA + TMEM kernel lands: reports no coverage).
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace sdpa {

bool prefill_tc_supported(int, int64_t, int64_t, const AttnParams&) { return false; }
LaunchPlan prefill_tc_plan(const AttnParams&, int, const DeviceInfo&) { return LaunchPlan{}; }
cudaError_t prefill_tc_launch(const AttnParams&, int, const LaunchPlan&, cudaStream_t) {
    return cudaErrorNotSupported;
}
int take_device_error_prefill_tc(cudaStream_t stream) {
    int code = 0;
    if (cudaMemcpyFromSymbolAsync(&code, g_sdpa_device_error, sizeof(int), 0, cudaMemcpyDeviceToHost, stream) !=
        cudaSuccess)
        return -1;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return -1;
    if (code) {
        const int zero = 0;
        cudaMemcpyToSymbolAsync(g_sdpa_device_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
        cudaStreamSynchronize(stream);
    }
    return code;
}

}  // namespace sdpa
