// flash_ffma.cu -- flash attention forward on CUDA cores (FFMA), true fp32.
//
// The fp32 path of both shapes: prefill (one launch over query tiles) and
// decode (the same kernel with the keys split across CTAs, then the
// log-sum-exp combine).  fp32 inputs stay fp32 end to end: products and sums
// are FFMA in fp32, the softmax is fp32, nothing is rounded to TF32 or fp16.
// mlxcel issue #1065 ("f32 matmul and single-query SDPA lose ~fp16 precision
// on M5"), section "Why this is a precision problem": an fp32 result whose
// error sits near 2^-10 betrays reduced internal precision; this kernel is the
// guard against that failure mode.
//
// Tiling: a CTA owns RT = 16 rows of one KV-head group.  A group row r is the
// pair (query head h = g*G + r / Lq, query i = r % Lq), so the G query heads
// that share one KV head (MLX issue #3885, section "Measured impact": scores
// shaped [B, n_kv, n_rep, qL, kL]) share every K/V tile the CTA loads.  Keys
// stream through shared memory in tiles of KT = 32 with an online softmax
// (running max and sum in the log2 domain, fp32).
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace sdpa {
namespace {

constexpr int kRT = 16;       // rows per CTA
constexpr int kKT = 32;       // keys per tile
constexpr int kThreads = 128; // 16 rows x 8 threads

template <int DQK, int DV>
struct FfmaSmem {
    static constexpr int QS = DQK + 1;   // odd strides: conflict-free column walks
    static constexpr int KS = DQK + 1;
    static constexpr int PS = kKT + 1;
    static constexpr size_t bytes =
        sizeof(float) * ((size_t)kRT * QS + (size_t)kKT * KS + (size_t)kKT * DV + (size_t)kRT * PS);
};

// Loads `rows` rows of `cols` elements (cols % 8 == 0 for 16-bit, % 4 for fp32)
// into a float tile with row stride `ld`.  Rows at or past `nvalid` are zero.
template <typename T>
__device__ __forceinline__ void load_rows_to_float(float* dst, int ld, const T* src, int64_t row_stride,
                                                   int rows, int nvalid, int cols, float mul) {
    constexpr int V = 16 / sizeof(T);
    const int chunks = cols / V;
    for (int idx = threadIdx.x; idx < rows * chunks; idx += kThreads) {
        const int r = idx / chunks, c = idx % chunks;
        float* d = dst + r * ld + c * V;
        if (r < nvalid) {
            const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src + r * row_stride + c * V));
            const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
            for (int u = 0; u < V; ++u) d[u] = Elem<T>::to_float(e[u]) * mul;
        } else {
#pragma unroll
            for (int u = 0; u < V; ++u) d[u] = 0.f;
        }
    }
}

template <typename T, int DQK, int DV>
__global__ void __launch_bounds__(kThreads) flash_ffma_kernel(const AttnParams p) {
    using S = FfmaSmem<DQK, DV>;
    extern __shared__ __align__(16) float smem[];
    float* Qs = smem;
    float* Ks = Qs + kRT * S::QS;
    float* Vs = Ks + kKT * S::KS;
    float* Ps = Vs + kKT * DV;

    const int tid = threadIdx.x;
    const int r = tid >> 3;        // row of this thread (both phases)
    const int c8 = tid & 7;        // lane within the row's 8 threads
    const int64_t G = p.group;
    const int64_t R = G * p.Lq;    // rows of one KV-head group
    const int64_t row0 = (int64_t)blockIdx.x * kRT;
    const int hkv = blockIdx.y;
    const int b = blockIdx.z / p.splits;
    const int split = blockIdx.z % p.splits;

    const T* qg = reinterpret_cast<const T*>(p.q);
    const T* kg = reinterpret_cast<const T*>(p.k) + b * p.sk[0] + hkv * p.sk[1];
    const T* vg = reinterpret_cast<const T*>(p.v) + b * p.sv[0] + hkv * p.sv[1];

    // This thread's row.
    const int64_t gr = row0 + r;
    const bool row_ok = gr < R;
    const int64_t hq = hkv * G + (row_ok ? gr / p.Lq : 0);
    const int64_t qi = row_ok ? gr % p.Lq : 0;

    // Q rows, pre-multiplied by scale*log2(e).  Rows of one tile may belong to two heads.
    for (int rr = 0; rr < kRT; ++rr) {
        const int64_t g2 = row0 + rr;
        if (g2 < R) {
            const int64_t h2 = hkv * G + g2 / p.Lq, i2 = g2 % p.Lq;
            load_rows_to_float<T>(Qs + rr * S::QS, S::QS, qg + b * p.sq[0] + h2 * p.sq[1] + i2 * p.sq[2], 0, 1, 1,
                                  DQK, p.scale_log2);
        } else {
            for (int d = tid; d < DQK; d += kThreads) Qs[rr * S::QS + d] = 0.f;
        }
    }

    // Key range of this CTA: its split, cut at the last key any of its rows can see.
    int64_t k_begin = (int64_t)split * p.keys_per_split;
    int64_t k_end = k_begin + p.keys_per_split;
    if (k_end > p.Lk) k_end = p.Lk;
    if (p.mask_kind == 3) {  // causal, bottom-right: key j visible to query i iff j <= i + Lk - Lq
        int64_t max_i = -1;
        for (int rr = 0; rr < kRT; ++rr) {
            const int64_t g2 = row0 + rr;
            if (g2 < R) max_i = max(max_i, g2 % p.Lq);
        }
        const int64_t last = max_i + p.Lk - p.Lq;
        if (k_end > last + 1) k_end = last + 1;
    }

    float m = -INFINITY;   // running max (log2 domain), identical in the row's 8 threads
    float l = 0.f;         // this thread's share of the running sum
    float o[DV / 8];
#pragma unroll
    for (int u = 0; u < DV / 8; ++u) o[u] = 0.f;

    const float log2e = 1.4426950408889634f;
    for (int64_t kt = k_begin; kt < k_end; kt += kKT) {
        const int nvalid = (int)((k_end - kt) < kKT ? (k_end - kt) : kKT);
        __syncthreads();   // previous tile fully consumed
        load_rows_to_float<T>(Ks, S::KS, kg + kt * p.sk[2], p.sk[2], kKT, nvalid, DQK, 1.f);
        load_rows_to_float<T>(Vs, DV, vg + kt * p.sv[2], p.sv[2], kKT, nvalid, DV, 1.f);
        __syncthreads();

        // scores for keys c8, c8+8, c8+16, c8+24
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        const float* qr = Qs + r * S::QS;
#pragma unroll 8
        for (int d = 0; d < DQK; ++d) {
            const float qd = qr[d];
#pragma unroll
            for (int u = 0; u < 4; ++u) s[u] = fmaf(qd, Ks[(c8 + 8 * u) * S::KS + d], s[u]);
        }
        float tmax = -INFINITY;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int jj = c8 + 8 * u;
            const int64_t j = kt + jj;
            bool keep = row_ok && jj < nvalid;
            if (keep && p.mask_kind == 1) {
                const T* mp = reinterpret_cast<const T*>(p.mask);
                s[u] += Elem<T>::to_float(mp[b * p.sm[0] + hq * p.sm[1] + qi * p.sm[2] + j * p.sm[3]]) * log2e;
            } else if (keep && p.mask_kind == 2) {
                const uint8_t* mp = reinterpret_cast<const uint8_t*>(p.mask);
                keep = mp[b * p.sm[0] + hq * p.sm[1] + qi * p.sm[2] + j * p.sm[3]] != 0;
            } else if (keep && p.mask_kind == 3) {
                keep = j <= qi + p.Lk - p.Lq;
            }
            if (!keep) s[u] = -INFINITY;
            tmax = fmaxf(tmax, s[u]);
        }
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
        const float m_new = fmaxf(m, tmax);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = exp2f(m - m_use);   // m = -inf -> 0
        float psum = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float pu = exp2f(s[u] - m_use);   // -inf -> 0
            Ps[r * S::PS + c8 + 8 * u] = pu;
            psum += pu;
        }
        l = l * alpha + psum;
        m = m_new;
#pragma unroll
        for (int u = 0; u < DV / 8; ++u) o[u] *= alpha;
        __syncthreads();   // Ps complete
        const float* pr = Ps + r * S::PS;
#pragma unroll 4
        for (int jj = 0; jj < kKT; ++jj) {
            const float pj = pr[jj];
            const float* vr = Vs + jj * DV + c8;
#pragma unroll
            for (int u = 0; u < DV / 8; ++u) o[u] = fmaf(pj, vr[8 * u], o[u]);
        }
    }

    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    if (!row_ok) return;
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    if (p.splits == 1) {
        T* og = reinterpret_cast<T*>(p.out) + b * p.so[0] + hq * p.so[1] + qi * p.so[2];
#pragma unroll
        for (int u = 0; u < DV / 8; ++u) og[c8 + 8 * u] = Elem<T>::from_float(o[u] * inv);
    } else {
        const int64_t row = ((int64_t)b * p.Hq + hq) * p.Lq + qi;
        float* po = p.part_o + (row * p.splits + split) * DV;
#pragma unroll
        for (int u = 0; u < DV / 8; ++u) po[c8 + 8 * u] = o[u] * inv;
        if (c8 == 0) p.part_lse[row * p.splits + split] = (l > 0.f) ? m + log2f(l) : -INFINITY;
    }
}

template <typename T, int DQK, int DV>
cudaError_t launch_one(const AttnParams& p, const LaunchPlan& plan, cudaStream_t stream) {
    auto kern = flash_ffma_kernel<T, DQK, DV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem_bytes);
    if (e != cudaSuccess) return e;
    kern<<<plan.grid, plan.block, plan.smem_bytes, stream>>>(p);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(const AttnParams& p, const LaunchPlan& plan, cudaStream_t s) {
    switch (p.Dqk * 1000 + p.Dv) {
        case 64064: return launch_one<T, 64, 64>(p, plan, s);
        case 72072: return launch_one<T, 72, 72>(p, plan, s);
        case 80080: return launch_one<T, 80, 80>(p, plan, s);
        case 96096: return launch_one<T, 96, 96>(p, plan, s);
        case 128128: return launch_one<T, 128, 128>(p, plan, s);
        case 192128: return launch_one<T, 192, 128>(p, plan, s);
        case 256256: return launch_one<T, 256, 256>(p, plan, s);
        case 512512: return launch_one<T, 512, 512>(p, plan, s);
        default: return cudaErrorInvalidValue;
    }
}

size_t smem_for(int64_t Dqk, int64_t Dv) {
    switch (Dqk * 1000 + Dv) {
        case 64064: return FfmaSmem<64, 64>::bytes;
        case 72072: return FfmaSmem<72, 72>::bytes;
        case 80080: return FfmaSmem<80, 80>::bytes;
        case 96096: return FfmaSmem<96, 96>::bytes;
        case 128128: return FfmaSmem<128, 128>::bytes;
        case 192128: return FfmaSmem<192, 128>::bytes;
        case 256256: return FfmaSmem<256, 256>::bytes;
        case 512512: return FfmaSmem<512, 512>::bytes;
        default: return 0;
    }
}

}  // namespace

bool ffma_supported(int dtype, int64_t Dqk, int64_t Dv) {
    return dtype >= 0 && dtype <= 2 && smem_for(Dqk, Dv) != 0;
}

LaunchPlan ffma_plan(const AttnParams& p, int dtype, const DeviceInfo& dev, bool split_keys) {
    (void)dtype;
    LaunchPlan plan{};
    const int64_t R = (int64_t)p.group * p.Lq;
    const int64_t row_tiles = (R + kRT - 1) / kRT;
    int splits = 1;
    if (split_keys) {
        // Fill the SMs: split the keys until there are about two CTAs per SM,
        // keeping at least two key tiles per split.
        const int64_t base = row_tiles * p.Hkv * p.B;
        const int64_t tiles = (p.Lk + kKT - 1) / kKT;
        int64_t want = (2 * (int64_t)dev.sm_count + base - 1) / base;
        int64_t cap = (tiles + 1) / 2;
        if (want > cap) want = cap;
        if (want > 64) want = 64;
        if (want < 1) want = 1;
        splits = (int)want;
    }
    int64_t kps = (p.Lk + splits - 1) / splits;
    kps = ((kps + kKT - 1) / kKT) * kKT;            // whole key tiles per split
    if (kps < kKT) kps = kKT;
    splits = (int)((p.Lk + kps - 1) / kps);
    if (splits < 1) splits = 1;
    plan.grid = dim3((unsigned)row_tiles, (unsigned)p.Hkv, (unsigned)(p.B * splits));
    plan.block = dim3(kThreads);
    plan.smem_bytes = smem_for(p.Dqk, p.Dv);
    plan.splits = splits;
    plan.keys_per_split = kps;
    plan.variant = 0;
    return plan;
}

cudaError_t ffma_launch(const AttnParams& p, int dtype, const LaunchPlan& plan, cudaStream_t stream) {
    switch (dtype) {
        case 0: return launch_typed<float>(p, plan, stream);
        case 1: return launch_typed<__half>(p, plan, stream);
        case 2: return launch_typed<__nv_bfloat16>(p, plan, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace sdpa
