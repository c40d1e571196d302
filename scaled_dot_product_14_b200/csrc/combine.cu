// combine.cu -- the zero fill for problems with no keys (every row's output is
// 0: a row with no visible key outputs zeros).  The log-sum-exp merge of
// split-key partials runs inside the split kernels themselves (the last split
// of a tile merges it, or the splits of a group meet at a barrier and merge
// slices), so no path launches a separate combine kernel.
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace sdpa {
namespace {

template <typename T>
__global__ void zero_fill_kernel(const AttnParams p) {
    const int64_t total = p.B * p.Hq * p.Lq * p.Dv;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e = idx % p.Dv, row = idx / p.Dv;
        const int64_t i = row % p.Lq, h = (row / p.Lq) % p.Hq, b = row / (p.Lq * p.Hq);
        reinterpret_cast<T*>(p.out)[b * p.so[0] + h * p.so[1] + i * p.so[2] + e] = Elem<T>::from_float(0.f);
    }
}

}  // namespace

cudaError_t zero_fill_launch(const AttnParams& p, int dtype, cudaStream_t stream) {
    const int64_t total = p.B * p.Hq * p.Lq * p.Dv;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 65535) blocks = 65535;
    if (blocks < 1) blocks = 1;
    switch (dtype) {
        case 0: zero_fill_kernel<float><<<(unsigned)blocks, 256, 0, stream>>>(p); break;
        case 1: zero_fill_kernel<__half><<<(unsigned)blocks, 256, 0, stream>>>(p); break;
        case 2: zero_fill_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, stream>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace sdpa
