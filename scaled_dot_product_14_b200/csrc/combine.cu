// combine.cu -- log-sum-exp merge of split-K partial outputs, and the zero
// fill for problems with no keys.
//
// Each split s of a query row left a normalised partial output O_s and the
// log2-domain log-sum-exp lse_s of its keys (-inf when it saw none).  The row's
// output is sum_s w_s O_s / sum_s w_s with w_s = 2^(lse_s - max_s lse_s); a
// split with lse_s = -inf has w_s = 0, and a row whose every split is -inf
// outputs zeros.  This is the second pass of the two-pass decode design that
// MLX issue #3885 ("Metal SDPA: no fused path for head_dim=512 ..."),
// discussion of the sdpa_vector 2-pass kernel, describes for long contexts.
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace sdpa {
namespace {

constexpr int kRowsPerBlock = 4;   // one warp per query row

template <typename T>
__global__ void __launch_bounds__(32 * kRowsPerBlock) combine_kernel(const AttnParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t rows = p.B * p.Hq * p.Lq;
    const int64_t row = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int S = p.splits;
    const float* lse = p.part_lse + row * S;
    float mx = -INFINITY;
    for (int s = lane; s < S; s += 32) mx = fmaxf(mx, lse[s]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));

    const int64_t i = row % p.Lq, h = (row / p.Lq) % p.Hq, b = row / (p.Lq * p.Hq);
    T* og = reinterpret_cast<T*>(p.out) + b * p.so[0] + h * p.so[1] + i * p.so[2];
    const int nv = (int)(p.Dv / 4);   // float4 chunks (Dv % 4 == 0)
    for (int c = lane; c < nv; c += 32) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float wsum = 0.f;
        if (mx != -INFINITY) {
            for (int s = 0; s < S; ++s) {
                const float w = exp2f(lse[s] - mx);   // -inf -> 0
                if (w == 0.f) continue;
                const float4 v = *reinterpret_cast<const float4*>(p.part_o + (row * S + s) * p.Dv + c * 4);
                acc.x += w * v.x;
                acc.y += w * v.y;
                acc.z += w * v.z;
                acc.w += w * v.w;
                wsum += w;
            }
        }
        const float inv = (wsum > 0.f) ? 1.f / wsum : 0.f;
        og[c * 4 + 0] = Elem<T>::from_float(acc.x * inv);
        og[c * 4 + 1] = Elem<T>::from_float(acc.y * inv);
        og[c * 4 + 2] = Elem<T>::from_float(acc.z * inv);
        og[c * 4 + 3] = Elem<T>::from_float(acc.w * inv);
    }
}

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

cudaError_t combine_launch(const AttnParams& p, int dtype, cudaStream_t stream) {
    const int64_t rows = p.B * p.Hq * p.Lq;
    const dim3 grid((unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock));
    const dim3 block(32 * kRowsPerBlock);
    switch (dtype) {
        case 0: combine_kernel<float><<<grid, block, 0, stream>>>(p); break;
        case 1: combine_kernel<__half><<<grid, block, 0, stream>>>(p); break;
        case 2: combine_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

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
