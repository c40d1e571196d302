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

constexpr int kCombineThreads = 128;
constexpr int kMaxSplitsSmem = 1024;

// One CTA per query row: the split weights go to shared memory once, then
// each thread accumulates its float4 columns over the splits with independent
// loads (the loop carries no load-to-load dependency).
template <typename T>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const AttnParams p) {
    __shared__ float w[kMaxSplitsSmem];
    __shared__ float red[kCombineThreads / 32];
    const int64_t row = blockIdx.x;
    const int S = p.splits;
    const float* lse = p.part_lse + row * S;
    float mx = -INFINITY;
    for (int s = threadIdx.x; s < S; s += kCombineThreads) mx = fmaxf(mx, lse[s]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = red[0];
#pragma unroll
    for (int wv = 1; wv < kCombineThreads / 32; ++wv) mx = fmaxf(mx, red[wv]);
    float part = 0.f;
    for (int s = threadIdx.x; s < S; s += kCombineThreads) {
        const float ws = (mx == -INFINITY) ? 0.f : exp2f(lse[s] - mx);   // -inf -> 0
        w[s] = ws;
        part += ws;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = part;
    __syncthreads();
    float wsum = 0.f;
#pragma unroll
    for (int wv = 0; wv < kCombineThreads / 32; ++wv) wsum += red[wv];
    const float inv = (wsum > 0.f) ? 1.f / wsum : 0.f;

    const int64_t i = row % p.Lq, h = (row / p.Lq) % p.Hq, b = row / (p.Lq * p.Hq);
    T* og = reinterpret_cast<T*>(p.out) + b * p.so[0] + h * p.so[1] + i * p.so[2];
    const int nv = (int)(p.Dv / 4);   // float4 chunks (Dv % 4 == 0)
    const float4* po = reinterpret_cast<const float4*>(p.part_o + row * S * p.Dv);
    for (int c = threadIdx.x; c < nv; c += kCombineThreads) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int s = 0; s < S; ++s) {
            const float ws = w[s];
            const float4 v = po[(int64_t)s * nv + c];
            acc.x = fmaf(ws, v.x, acc.x);
            acc.y = fmaf(ws, v.y, acc.y);
            acc.z = fmaf(ws, v.z, acc.z);
            acc.w = fmaf(ws, v.w, acc.w);
        }
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
    if (p.splits > kMaxSplitsSmem || rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)rows);
    const dim3 block(kCombineThreads);
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
