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

    // Q rows, pre-multiplied by scale*log2(e).  Rows of one tile may belong to two
    // heads.  One pass over every (row, 16-byte chunk), so all loads are in flight
    // together rather than one row's latency after another.
    {
        constexpr int V = 16 / sizeof(T);
        constexpr int CH = DQK / V;
        for (int idx = tid; idx < kRT * CH; idx += kThreads) {
            const int rr = idx / CH, c = idx % CH;
            const int64_t g2 = row0 + rr;
            float* d = Qs + rr * S::QS + c * V;
            if (g2 < R) {
                const int64_t h2 = hkv * G + g2 / p.Lq, i2 = g2 % p.Lq;
                const uint4 raw =
                    __ldg(reinterpret_cast<const uint4*>(qg + b * p.sq[0] + h2 * p.sq[1] + i2 * p.sq[2] + c * V));
                const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
                for (int u = 0; u < V; ++u) d[u] = Elem<T>::to_float(e[u]) * p.scale_log2;
            } else {
#pragma unroll
                for (int u = 0; u < V; ++u) d[u] = 0.f;
            }
        }
    }

    // Key range of this CTA: its split, cut at the last key any of its rows can see.
    int64_t k_begin = p.key_begin + (int64_t)split * p.keys_per_split;
    int64_t k_end = k_begin + p.keys_per_split;
    if (k_end > p.Lk) k_end = p.Lk;
    if (p.mask_kind == 3 || p.mask_kind == 4) {  // causal, bottom-right: key j visible to query i iff j <= i + Lk - Lq
        int64_t max_i = -1, min_i = p.Lq;
        for (int rr = 0; rr < kRT; ++rr) {
            const int64_t g2 = row0 + rr;
            if (g2 < R) {
                max_i = max(max_i, g2 % p.Lq);
                min_i = min(min_i, g2 % p.Lq);
            }
        }
        const int64_t last = max_i + p.Lk - p.Lq;
        if (k_end > last + 1) k_end = last + 1;
        if (p.mask_kind == 4) {   // sliding window: nothing before the first row's window
            const int64_t first = min_i + p.Lk - p.Lq - p.window + 1;
            if (k_begin < first) k_begin = first;
        }
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
            } else if (keep && p.mask_kind == 4) {
                keep = j <= qi + p.Lk - p.Lq && j > qi + p.Lk - p.Lq - p.window;
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
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    T* og = reinterpret_cast<T*>(p.out) + b * p.so[0] + hq * p.so[1] + qi * p.so[2];
    if (p.splits == 1) {
        if (row_ok)
#pragma unroll
            for (int u = 0; u < DV / 8; ++u) og[c8 + 8 * u] = Elem<T>::from_float(o[u] * inv);
        return;
    }
    const int NS = p.splits;
    const int64_t row = ((int64_t)b * p.Hq + hq) * p.Lq + qi;
    if (row_ok) {
        float* po = p.part_o + (row * NS + split) * DV;
#pragma unroll
        for (int u = 0; u < DV / 8; ++u) po[c8 + 8 * u] = o[u] * inv;
        if (c8 == 0) p.part_lse[row * NS + split] = (l > 0.f) ? m + log2f(l) : -INFINITY;
    }
    if (p.counters == nullptr) return;   // (never with splits > 1: the dispatcher always passes counters)

    // The last split of this (row tile, KV head, batch) to finish merges the
    // tile's rows over all splits; no CTA waits for another, so the grid may
    // run in waves.  Every call adds exactly NS to the tile's 64-bit counter
    // (counters are kept per launch shape), so the last arrival is the one
    // that brings it to a multiple of NS.
    __shared__ int s_last;
    __syncthreads();   // every thread's partial stores precede thread 0's release below
    if (tid == 0) {
        unsigned long long* ctr = reinterpret_cast<unsigned long long*>(p.counters) +
                                  ((int64_t)blockIdx.z / NS * gridDim.y + hkv) * gridDim.x + blockIdx.x;
        unsigned long long old;
        asm volatile("atom.add.acq_rel.gpu.global.u64 %0, [%1], 1;" : "=l"(old) : "l"(ctr) : "memory");
        s_last = ((old + 1) % (unsigned long long)NS) == 0;
    }
    __syncthreads();   // thread 0's acquire orders the other splits' partials before these loads
    if (!s_last || !row_ok) return;
    const float* pl = p.part_lse + row * NS;
    float mx = -INFINITY;
    for (int s2 = 0; s2 < NS; ++s2) mx = fmaxf(mx, __ldcg(pl + s2));
    float acc[DV / 8], wsum = 0.f;
#pragma unroll
    for (int u = 0; u < DV / 8; ++u) acc[u] = 0.f;
    for (int s2 = 0; s2 < NS; ++s2) {
        const float ls = __ldcg(pl + s2);
        const float ws = (mx == -INFINITY || ls == -INFINITY) ? 0.f : exp2f(ls - mx);
        wsum += ws;
        const float* ps = p.part_o + (row * NS + s2) * DV;
#pragma unroll
        for (int u = 0; u < DV / 8; ++u) acc[u] = fmaf(ws, __ldcg(ps + c8 + 8 * u), acc[u]);
    }
    const float winv = (wsum > 0.f) ? 1.f / wsum : 0.f;
#pragma unroll
    for (int u = 0; u < DV / 8; ++u) og[c8 + 8 * u] = Elem<T>::from_float(acc[u] * winv);
}

// ---- register-tiled fp32 prefill ------------------------------------------
//
// The same online softmax, re-tiled so that the FMA units rather than shared
// memory set the pace: a CTA owns TM = 128 group rows and streams the keys in
// tiles of TN = 64.  Thread (ty, tx) of the 32 x 8 grid holds the scores of
// rows 4*ty .. 4*ty+3 against keys tx, tx+8, .., tx+56 (32 accumulators) and,
// for the P.V product, the same 4 rows against Dv/8 output columns.  Per four
// steps along d a thread reads 4 float4 of Q and 8 float4 of K for 128 FMAs;
// P.V runs on packed f32x2 FMAs (fp32 rounding per lane, half the issue slots).
//
// Shared memory (fp32):
//   Qt[d][row]   Q transposed once per CTA, pre-multiplied by scale*log2(e)
//   K[key][d]    row stride DQK+4 (an odd number of 16-byte units: the eight
//                keys tx = 0..7 a quarter-warp reads hit distinct bank groups)
//   V[key][c]    row stride Dv
//   Pt[key][row] P transposed, row stride 128+4 (33 16-byte units): the stores
//                of eight consecutive keys hit distinct bank groups, and the
//                loads of one key are plain offsets
// K and V arrive by cp.async: V of tile j while its scores are computed, K of
// tile j+1 while P.V of tile j runs.
constexpr int kTM = 128;
constexpr int kTN = 64;
constexpr int kTThreads = 256;

template <int DQK, int DV>
struct TiledSmem {
    static_assert(DQK % 8 == 0 && DV % 8 == 0, "head dims are multiples of 8");
    static constexpr int QS = kTM;
    static constexpr int KS = DQK + 4;
    static_assert((KS / 4) % 2 == 1, "K row stride must be an odd number of 16-byte units");
    static constexpr int VS = DV;
    static constexpr int PS = kTM + 4;
    static_assert((PS / 4) % 2 == 1, "Pt row stride must be an odd number of 16-byte units");
    static constexpr int k_off = DQK * QS;
    static constexpr int v_off = k_off + kTN * KS;
    static constexpr int p_off = v_off + kTN * VS;
    static constexpr size_t bytes = sizeof(float) * ((size_t)p_off + (size_t)kTN * PS);
};

// Output columns of thread tx: Dv/32 float4 groups at 32*g + 4*tx, then, for
// the Dv % 32 left over, a float2 at 2*tx (16 columns) and/or one column at tx
// (8 columns).  Every column belongs to exactly one of the 8 threads of a row.
template <int DV>
struct TiledCols {
    static constexpr int F4 = DV / 32;
    static constexpr bool HAS2 = (DV % 32) >= 16;
    static constexpr bool HAS1 = (DV % 16) == 8;
    static constexpr int NC = 4 * F4 + (HAS2 ? 2 : 0) + (HAS1 ? 1 : 0);
    static_assert(NC * 8 == DV, "column split");
    static constexpr int base2 = 32 * F4;
    static constexpr int base1 = 32 * F4 + (HAS2 ? 16 : 0);
};

template <int DV>
__device__ __forceinline__ void tiled_load_v(float (&vv)[TiledCols<DV>::NC], const float* vrow, int tx) {
    using C = TiledCols<DV>;
#pragma unroll
    for (int g = 0; g < C::F4; ++g) {
        const float4 x = *reinterpret_cast<const float4*>(vrow + 32 * g + 4 * tx);
        vv[4 * g] = x.x; vv[4 * g + 1] = x.y; vv[4 * g + 2] = x.z; vv[4 * g + 3] = x.w;
    }
    if constexpr (C::HAS2) {
        const float2 x = *reinterpret_cast<const float2*>(vrow + C::base2 + 2 * tx);
        vv[4 * C::F4] = x.x; vv[4 * C::F4 + 1] = x.y;
    }
    if constexpr (C::HAS1) vv[C::NC - 1] = vrow[C::base1 + tx];
}

template <int DV, typename F>
__device__ __forceinline__ void tiled_for_cols(int tx, F&& f) {   // f(n, column)
    using C = TiledCols<DV>;
#pragma unroll
    for (int g = 0; g < C::F4; ++g)
#pragma unroll
        for (int u = 0; u < 4; ++u) f(4 * g + u, 32 * g + 4 * tx + u);
    if constexpr (C::HAS2) { f(4 * C::F4, C::base2 + 2 * tx); f(4 * C::F4 + 1, C::base2 + 2 * tx + 1); }
    if constexpr (C::HAS1) f(C::NC - 1, C::base1 + tx);
}

// One 64-key tile of K or V (rows kt .. kt+63 of one KV head) into shared
// memory; rows at or past `nvalid` are zero-filled (src-size 0).
template <int D, int LD>
__device__ __forceinline__ void tiled_issue_rows(float* dst, const float* src, int64_t row_stride, int nvalid) {
    constexpr int CH = D / 4;   // 16-byte chunks per row
    for (int it = threadIdx.x; it < kTN * CH; it += kTThreads) {
        const int r = it / CH, c = it % CH;
        const bool ok = r < nvalid;
        const float* g = src + (ok ? (int64_t)r * row_stride : 0) + c * 4;
        cp_async16(smem_u32(dst + r * LD + c * 4), g, ok ? 16 : 0);
    }
    cp_async_commit();
}

template <int DQK, int DV, int MASK, int MINB>
__global__ void __launch_bounds__(kTThreads, MINB) flash_tiled_f32_kernel(const AttnParams p) {
    using S = TiledSmem<DQK, DV>;
    using C = TiledCols<DV>;
    extern __shared__ __align__(16) float smem[];
    float* Qt = smem;
    float* Ks = smem + S::k_off;
    float* Vs = smem + S::v_off;
    float* Pt = smem + S::p_off;

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int tx = lane & 7;
    const int ty = (tid >> 5) * 4 + (lane >> 3);
    const int64_t G = p.group;
    const int64_t R = G * p.Lq;
    const int64_t row0 = (int64_t)blockIdx.x * kTM;
    const int hkv = blockIdx.y;
    const int b = blockIdx.z;

    const float* qg = reinterpret_cast<const float*>(p.q);
    const float* kg = reinterpret_cast<const float*>(p.k) + b * p.sk[0] + hkv * p.sk[1];
    const float* vg = reinterpret_cast<const float*>(p.v) + b * p.sv[0] + hkv * p.sv[1];

    // Key range: all keys, cut for causal (and sliding-window) masks at the
    // last key any row of the CTA sees, and for a sliding window started at
    // the first key any row sees.
    int64_t k_begin = 0, k_end = p.Lk;
    if (MASK == 3 || MASK == 4) {
        const int64_t last_row = min(row0 + kTM, R) - 1;
        // rows of the CTA may span two heads; the largest query index is Lq-1
        // (the smallest 0) unless all rows sit in one head
        const bool one_head = row0 / p.Lq == last_row / p.Lq;
        const int64_t max_i = one_head ? last_row % p.Lq : p.Lq - 1;
        k_end = min(k_end, max_i + p.Lk - p.Lq + 1);
        if (MASK == 4) {
            const int64_t min_i = one_head ? row0 % p.Lq : 0;
            k_begin = max((int64_t)0, min_i + p.Lk - p.Lq - p.window + 1);
        }
    }
    if (k_end > k_begin)
        tiled_issue_rows<DQK, S::KS>(Ks, kg + k_begin * p.sk[2], p.sk[2], (int)min((int64_t)kTN, k_end - k_begin));

    // Qt: 32 consecutive rows per warp and one 4-column chunk, so each
    // transposed store is 32 consecutive floats.
    for (int it = tid; it < kTM * (DQK / 4); it += kTThreads) {
        const int rr = it % kTM, c = it / kTM;
        const int64_t gr = row0 + rr;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (gr < R) {
            const int64_t h = hkv * G + gr / p.Lq, i = gr % p.Lq;
            x = __ldg(reinterpret_cast<const float4*>(qg + b * p.sq[0] + h * p.sq[1] + i * p.sq[2] + c * 4));
        }
        Qt[(4 * c + 0) * S::QS + rr] = x.x * p.scale_log2;
        Qt[(4 * c + 1) * S::QS + rr] = x.y * p.scale_log2;
        Qt[(4 * c + 2) * S::QS + rr] = x.z * p.scale_log2;
        Qt[(4 * c + 3) * S::QS + rr] = x.w * p.scale_log2;
    }

    // This thread's four rows.
    int64_t qi[4], moff[4];
    bool rok[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t gr = row0 + 4 * ty + i;
        rok[i] = gr < R;
        const int64_t h = hkv * G + (rok[i] ? gr / p.Lq : 0);
        qi[i] = rok[i] ? gr % p.Lq : 0;
        moff[i] = (MASK == 1 || MASK == 2) ? b * p.sm[0] + h * p.sm[1] + qi[i] * p.sm[2] : 0;
    }

    float m[4], l[4], o[4][C::NC];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
#pragma unroll
        for (int n = 0; n < C::NC; ++n) o[i][n] = 0.f;
    }
    const float log2e = 1.4426950408889634f;

    for (int64_t kt = k_begin; kt < k_end; kt += kTN) {
        const int nvalid = (int)min((int64_t)kTN, k_end - kt);
        cp_async_wait<0>();   // K of this tile (the only group in flight)
        __syncthreads();      // K (and Qt) visible; the previous P.V is done with V and Pt
        tiled_issue_rows<DV, S::VS>(Vs, vg + kt * p.sv[2], p.sv[2], nvalid);

        float s[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int k = 0; k < 8; ++k) s[i][k] = 0.f;
        const float* kb = Ks + tx * S::KS;
        const float* qb = Qt + 4 * ty;
#pragma unroll 1
        for (int d = 0; d < DQK; d += 4) {
            float4 qf[4];
#pragma unroll
            for (int dd = 0; dd < 4; ++dd) qf[dd] = *reinterpret_cast<const float4*>(qb + (d + dd) * S::QS);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float4 kf = *reinterpret_cast<const float4*>(kb + 8 * k * S::KS + d);
                const float kd[4] = {kf.x, kf.y, kf.z, kf.w};
#pragma unroll
                for (int dd = 0; dd < 4; ++dd) {
                    s[0][k] = fmaf(qf[dd].x, kd[dd], s[0][k]);
                    s[1][k] = fmaf(qf[dd].y, kd[dd], s[1][k]);
                    s[2][k] = fmaf(qf[dd].z, kd[dd], s[2][k]);
                    s[3][k] = fmaf(qf[dd].w, kd[dd], s[3][k]);
                }
            }
        }

        // Rows past the group (zero Q, never stored) need no masking; a full
        // unmasked tile needs none at all.
        if (MASK != 0 || nvalid < kTN) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int jj = tx + 8 * k;
                    const int64_t j = kt + jj;
                    bool keep = jj < nvalid;
                    if (MASK == 1 && keep)
                        s[i][k] += __ldg(reinterpret_cast<const float*>(p.mask) + moff[i] + j * p.sm[3]) * log2e;
                    if (MASK == 2 && keep)
                        keep = __ldg(reinterpret_cast<const uint8_t*>(p.mask) + moff[i] + j * p.sm[3]) != 0;
                    if (MASK == 3 || MASK == 4) keep = keep && j <= qi[i] + p.Lk - p.Lq;
                    if (MASK == 4) keep = keep && j > qi[i] + p.Lk - p.Lq - p.window;
                    if (!keep) s[i][k] = -INFINITY;
                }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float mx = fmaxf(fmaxf(fmaxf(s[i][0], s[i][1]), fmaxf(s[i][2], s[i][3])),
                             fmaxf(fmaxf(s[i][4], s[i][5]), fmaxf(s[i][6], s[i][7])));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            const float m_new = fmaxf(m[i], mx);
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            const float alpha = exp2f(m[i] - m_use);   // m = -inf -> 0
            float ps = 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                s[i][k] = exp2f(s[i][k] - m_use);      // -inf -> 0
                ps += s[i][k];
            }
            l[i] = l[i] * alpha + ps;
            m[i] = m_new;
#pragma unroll
            for (int n = 0; n < C::NC; ++n) o[i][n] *= alpha;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
            *reinterpret_cast<float4*>(Pt + (tx + 8 * k) * S::PS + 4 * ty) =
                make_float4(s[0][k], s[1][k], s[2][k], s[3][k]);

        cp_async_wait<0>();   // V of this tile
        __syncthreads();      // Pt and V visible; every thread is done with K
        if (kt + kTN < k_end)
            tiled_issue_rows<DQK, S::KS>(Ks, kg + (kt + kTN) * p.sk[2], p.sk[2], (int)min((int64_t)kTN, k_end - kt - kTN));

#pragma unroll 8
        for (int j = 0; j < kTN; ++j) {
            const float4 pf = *reinterpret_cast<const float4*>(Pt + j * S::PS + 4 * ty);
            float vv[C::NC];
            tiled_load_v<DV>(vv, Vs + j * S::VS, tx);
            // packed f32x2 FMAs over column pairs (each lane an ordinary fp32 FMA):
            // half the issue slots of scalar FFMA for the same arithmetic
            const uint64_t pp[4] = {f2_pack(pf.x, pf.x), f2_pack(pf.y, pf.y), f2_pack(pf.z, pf.z),
                                    f2_pack(pf.w, pf.w)};
#pragma unroll
            for (int n = 0; n + 1 < C::NC; n += 2) {
                const uint64_t v2 = f2_pack(vv[n], vv[n + 1]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint64_t r = f2_fma(pp[i], v2, f2_pack(o[i][n], o[i][n + 1]));
                    o[i][n] = f2_lo(r);
                    o[i][n + 1] = f2_hi(r);
                }
            }
            if constexpr (C::NC % 2 == 1) {
                constexpr int n = C::NC - 1;
                o[0][n] = fmaf(pf.x, vv[n], o[0][n]);
                o[1][n] = fmaf(pf.y, vv[n], o[1][n]);
                o[2][n] = fmaf(pf.z, vv[n], o[2][n]);
                o[3][n] = fmaf(pf.w, vv[n], o[3][n]);
            }
        }
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float li = l[i];
        li += __shfl_xor_sync(0xffffffffu, li, 1);
        li += __shfl_xor_sync(0xffffffffu, li, 2);
        li += __shfl_xor_sync(0xffffffffu, li, 4);
        if (!rok[i]) continue;
        const float inv = (li > 0.f) ? 1.f / li : 0.f;
        const int64_t gr = row0 + 4 * ty + i;
        const int64_t h = hkv * G + gr / p.Lq;
        float* og = reinterpret_cast<float*>(p.out) + b * p.so[0] + h * p.so[1] + qi[i] * p.so[2];
        tiled_for_cols<DV>(tx, [&](int n, int c) { og[c] = o[i][n] * inv; });
    }
}

template <int DQK, int DV, int MASK>
cudaError_t launch_tiled_mask(const AttnParams& p, const LaunchPlan& plan, cudaStream_t stream) {
    constexpr int MINB = TiledSmem<DQK, DV>::bytes <= 110 * 1024 ? 2 : 1;
    auto kern = flash_tiled_f32_kernel<DQK, DV, MASK, MINB>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem_bytes);
    if (e != cudaSuccess) return e;
    kern<<<plan.grid, plan.block, plan.smem_bytes, stream>>>(p);
    return cudaGetLastError();
}

template <int DQK, int DV>
cudaError_t launch_tiled(const AttnParams& p, const LaunchPlan& plan, cudaStream_t s) {
    switch (p.mask_kind) {
        case 0: return launch_tiled_mask<DQK, DV, 0>(p, plan, s);
        case 1: return launch_tiled_mask<DQK, DV, 1>(p, plan, s);
        case 2: return launch_tiled_mask<DQK, DV, 2>(p, plan, s);
        case 3: return launch_tiled_mask<DQK, DV, 3>(p, plan, s);
        case 4: return launch_tiled_mask<DQK, DV, 4>(p, plan, s);
        default: return cudaErrorInvalidValue;
    }
}

// Head dims of the tiled kernel (Dv <= 128 keeps the accumulators in registers).
size_t tiled_smem_for(int64_t Dqk, int64_t Dv) {
    switch (Dqk * 1000 + Dv) {
        case 40032: return TiledSmem<40, 32>::bytes;
        case 64064: return TiledSmem<64, 64>::bytes;
        case 72072: return TiledSmem<72, 72>::bytes;
        case 80080: return TiledSmem<80, 80>::bytes;
        case 96096: return TiledSmem<96, 96>::bytes;
        case 128128: return TiledSmem<128, 128>::bytes;
        case 192128: return TiledSmem<192, 128>::bytes;
        default: return 0;
    }
}

cudaError_t launch_tiled_dims(const AttnParams& p, const LaunchPlan& plan, cudaStream_t s) {
    switch (p.Dqk * 1000 + p.Dv) {
        case 40032: return launch_tiled<40, 32>(p, plan, s);
        case 64064: return launch_tiled<64, 64>(p, plan, s);
        case 72072: return launch_tiled<72, 72>(p, plan, s);
        case 80080: return launch_tiled<80, 80>(p, plan, s);
        case 96096: return launch_tiled<96, 96>(p, plan, s);
        case 128128: return launch_tiled<128, 128>(p, plan, s);
        case 192128: return launch_tiled<192, 128>(p, plan, s);
        default: return cudaErrorInvalidValue;
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
        case 40032: return launch_one<T, 40, 32>(p, plan, s);
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
        case 40032: return FfmaSmem<40, 32>::bytes;
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
    LaunchPlan plan{};
    const size_t tiled = tiled_smem_for(p.Dqk, p.Dv);
    if (!split_keys && dtype == 0 && tiled != 0) {
        // fp32 prefill: the register-tiled kernel, one CTA per 128 group rows
        const int64_t R = (int64_t)p.group * p.Lq;
        plan.grid = dim3((unsigned)((R + kTM - 1) / kTM), (unsigned)p.Hkv, (unsigned)p.B);
        plan.block = dim3(kTThreads);
        plan.smem_bytes = tiled;
        plan.splits = 1;
        plan.keys_per_split = p.Lk;
        plan.variant = 1;
        return plan;
    }
    const int64_t R = (int64_t)p.group * p.Lq;
    const int64_t row_tiles = (R + kRT - 1) / kRT;
    int splits = 1;
    if (split_keys) {
        // Fill the SMs: split the keys until there are about two CTAs per SM,
        // keeping at least two key tiles per split.
        const int64_t base = row_tiles * p.Hkv * p.B;
        const int64_t tiles = (p.Lk - p.key_begin + kKT - 1) / kKT;
        int64_t want = (2 * (int64_t)dev.sm_count + base - 1) / base;
        int64_t cap = (tiles + 1) / 2;
        if (want > cap) want = cap;
        if (want > 64) want = 64;
        if (want < 1) want = 1;
        splits = (int)want;
    }
    const int64_t span = p.Lk - p.key_begin;        // keys any query may see
    int64_t kps = (span + splits - 1) / splits;
    kps = ((kps + kKT - 1) / kKT) * kKT;            // whole key tiles per split
    if (kps < kKT) kps = kKT;
    splits = (int)((span + kps - 1) / kps);
    if (splits < 1) splits = 1;
    plan.grid = dim3((unsigned)row_tiles, (unsigned)p.Hkv, (unsigned)(p.B * splits));
    plan.block = dim3(kThreads);
    plan.smem_bytes = smem_for(p.Dqk, p.Dv);
    plan.splits = splits;
    plan.keys_per_split = kps;
    plan.variant = 0;
    return plan;
}

size_t ffma_counters(const LaunchPlan& plan) {
    return (size_t)plan.grid.x * plan.grid.y * (plan.grid.z / (plan.splits > 0 ? plan.splits : 1)) * 2;
}

cudaError_t ffma_launch(const AttnParams& p, int dtype, const LaunchPlan& plan, cudaStream_t stream) {
    if (plan.variant == 1) return dtype == 0 ? launch_tiled_dims(p, plan, stream) : cudaErrorInvalidValue;
    switch (dtype) {
        case 0: return launch_typed<float>(p, plan, stream);
        case 1: return launch_typed<__half>(p, plan, stream);
        case 2: return launch_typed<__nv_bfloat16>(p, plan, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace sdpa
