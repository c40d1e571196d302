// decode_mma.cu -- split-K (flash-decoding) attention for short queries,
// fp16 / bf16, on warp-level tensor-core MMA (m16n8k16, fp32 accumulation).
//
// The decode ("vector") path of MLX issue #3885 ("Metal SDPA: no fused path
// for head_dim=512 ..."), section "Current routing": qL <= 8.  Decode is bound
// by reading K and V (same issue, discussion of the bytes-normalised control:
// d * n_kv equal means equal K+V bytes).  Design points:
//
//  * one CTA serves every query row of a KV-head group (the G = Hq/Hkv query
//    heads times the qL queries), so each K/V byte is read once per group
//    (the MLX commit "Read each K/V byte once in gqa-8 decode attention");
//  * keys are split across CTAs (split-K) so that B*Hkv small problems still
//    fill the 148 SMs; each CTA writes a partial output and its log-sum-exp,
//    merged by the combine kernel (combine.cu); the split count scales with
//    1/(B*Hkv) (same issue: the two-pass kernel starves when n_kv is small);
//  * each warp streams its own 16-key blocks of K and V through a 3-stage ring
//    of 16-byte cp.async copies (coalesced, 16-byte vectors), with no
//    CTA-wide barrier in the main loop;
//  * scores are computed transposed, S^T = K Q^T, so the keys fill the
//    16-row side of the MMA and the few query rows the 8-column side (8 rows
//    per n-tile instead of 16: half the padding waste at gqa*qL <= 8);
//    P^T goes from the S^T accumulators to the B operand of O^T += V^T P^T
//    with one movmatrix per 8x8 block, never touching shared memory.
#include <cuda_runtime.h>
#include <math.h>
#include <stdlib.h>

#include "common.cuh"
#include "kernels.h"

namespace sdpa {
namespace {

constexpr int kStages = 3;

__host__ __device__ constexpr int round16(int x) { return (x + 15) / 16 * 16; }

template <int DQK, int DV, int NT, int W>
struct DecodeCfg {
    static constexpr int DQKP = round16(DQK);   // MMA K extent (72 -> 80)
    static constexpr int DVP = round16(DV);
    static constexpr int QS = DQKP + 8;         // smem row strides (elements): +16 B breaks bank conflicts
    static constexpr int KS = DQKP + 8;
    static constexpr int VS = DVP + 8;
    static constexpr int ROWS = 8 * NT;         // query rows per CTA
    static constexpr int STAGE_ELEMS = 16 * KS + 16 * VS;
    static constexpr size_t ring_bytes = (size_t)W * kStages * STAGE_ELEMS * 2;
    static constexpr size_t q_bytes = (size_t)ROWS * QS * 2;
    static constexpr size_t merge_bytes = (size_t)W * ROWS * (DVP + 2) * 4;
    static constexpr size_t smem_bytes = q_bytes + (ring_bytes > merge_bytes ? ring_bytes : merge_bytes);
};

template <typename T, int DQK, int DV, int NT, int W>
__global__ void __launch_bounds__(W * 32) decode_mma_kernel(const AttnParams p, const int RG) {
    using C = DecodeCfg<DQK, DV, NT, W>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    T* Qs = reinterpret_cast<T*>(smem_raw);
    T* ring = reinterpret_cast<T*>(smem_raw + C::q_bytes);
    float* merge = reinterpret_cast<float*>(smem_raw + C::q_bytes);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g8 = lane >> 2, t4 = lane & 3;   // MMA fragment coordinates
    const int split = blockIdx.x;
    const int hkv = blockIdx.y / RG, rg = blockIdx.y % RG;
    const int b = blockIdx.z;
    const int64_t G = p.group, R = G * p.Lq;
    const int64_t row0 = (int64_t)rg * C::ROWS;

    // ---- Q rows of this CTA (zero rows past the group, zero pad columns)
    {
        const T* qg = reinterpret_cast<const T*>(p.q);
        constexpr int CH = C::DQKP / 8;   // 16-byte chunks per padded row
        for (int idx = tid; idx < C::ROWS * CH; idx += W * 32) {
            const int r = idx / CH, c = idx % CH;
            const int64_t gr = row0 + r;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (gr < R && c * 8 < DQK) {
                const int64_t h = hkv * G + gr / p.Lq, i = gr % p.Lq;
                val = *reinterpret_cast<const uint4*>(qg + b * p.sq[0] + h * p.sq[1] + i * p.sq[2] + c * 8);
            }
            *reinterpret_cast<uint4*>(Qs + r * C::QS + c * 8) = val;
        }
        // pad columns of every ring slot (only when the head dim is not a multiple of 16)
        if (C::DQKP != DQK || C::DVP != DV) {
            for (int idx = tid; idx < W * kStages * 16; idx += W * 32) {
                T* st = ring + (size_t)(idx / 16) * C::STAGE_ELEMS;
                const int rr = idx % 16;
                for (int d = DQK; d < C::DQKP; ++d) st[rr * C::KS + d] = Elem<T>::from_float(0.f);
                for (int d = DV; d < C::DVP; ++d) st[16 * C::KS + rr * C::VS + d] = Elem<T>::from_float(0.f);
            }
        }
    }
    __syncthreads();

    // ---- key blocks of this split (16 keys each), cut at the causal horizon
    const int64_t nkb = (p.Lk + 15) / 16;
    const int64_t kbps = p.keys_per_split / 16;
    int64_t kb_begin = (int64_t)split * kbps;
    int64_t kb_end = min(nkb, kb_begin + kbps);
    int64_t max_i = -1;   // largest query index among this CTA's rows
    for (int r = 0; r < C::ROWS; ++r)
        if (row0 + r < R) max_i = max(max_i, (row0 + r) % p.Lq);
    if (p.mask_kind == 3) {
        const int64_t last = max_i + p.Lk - p.Lq;   // last key any row sees
        kb_end = min(kb_end, last < 0 ? (int64_t)0 : last / 16 + 1);
    }
    const int64_t my_first = kb_begin + warp;
    const int n_my = (my_first < kb_end) ? (int)((kb_end - my_first + W - 1) / W) : 0;

    const T* kg = reinterpret_cast<const T*>(p.k) + b * p.sk[0] + hkv * p.sk[1];
    const T* vg = reinterpret_cast<const T*>(p.v) + b * p.sv[0] + hkv * p.sv[1];
    T* my_ring = ring + (size_t)warp * kStages * C::STAGE_ELEMS;

    auto issue = [&](int it) {
        const int64_t kb = my_first + (int64_t)it * W;
        T* st = my_ring + (it % kStages) * C::STAGE_ELEMS;
        constexpr int KCH = DQK / 8, VCH = DV / 8;   // 16-byte chunks per row
        for (int idx = lane; idx < 16 * KCH; idx += 32) {
            const int rr = idx / KCH, c = idx % KCH;
            const int64_t j = kb * 16 + rr;
            const bool ok = j < p.Lk;
            cp_async16(smem_u32(st + rr * C::KS + c * 8), ok ? (const void*)(kg + j * p.sk[2] + c * 8) : (const void*)kg,
                       ok ? 16 : 0);
        }
        T* vs = st + 16 * C::KS;
        for (int idx = lane; idx < 16 * VCH; idx += 32) {
            const int rr = idx / VCH, c = idx % VCH;
            const int64_t j = kb * 16 + rr;
            const bool ok = j < p.Lk;
            cp_async16(smem_u32(vs + rr * C::VS + c * 8), ok ? (const void*)(vg + j * p.sv[2] + c * 8) : (const void*)vg,
                       ok ? 16 : 0);
        }
    };

#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        if (s < n_my) issue(s);
        cp_async_commit();
    }

    // ---- per-thread state: rows (nt*8 + 2*t4 + {0,1}); O^T fragments
    float m_run[NT][2], l_run[NT][2];
    float o[C::DVP / 16][NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        m_run[nt][0] = m_run[nt][1] = -INFINITY;
        l_run[nt][0] = l_run[nt][1] = 0.f;
    }
#pragma unroll
    for (int mt = 0; mt < C::DVP / 16; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 4; ++c) o[mt][nt][c] = 0.f;

    // per-row constants of this thread's rows
    int64_t row_h[NT][2], row_i[NT][2];
    bool row_ok[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int64_t gr = row0 + nt * 8 + 2 * t4 + c;
            row_ok[nt][c] = gr < R;
            row_h[nt][c] = hkv * G + (gr < R ? gr / p.Lq : 0);
            row_i[nt][c] = gr < R ? gr % p.Lq : 0;
        }

    const uint32_t q_base = smem_u32(Qs);
    const float log2e = 1.4426950408889634f;

    for (int it = 0; it < n_my; ++it) {
        if (it + kStages - 1 < n_my) issue(it + kStages - 1);
        cp_async_commit();
        cp_async_wait<kStages - 1>();
        __syncwarp();

        const T* st = my_ring + (it % kStages) * C::STAGE_ELEMS;
        const uint32_t k_base = smem_u32(st);
        const uint32_t v_base = smem_u32(st + 16 * C::KS);
        const int64_t kb = my_first + (int64_t)it * W;

        // S^T[16 keys][8*NT rows] = K_blk . Q^T
        float s[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
        {
            const int mi = lane >> 3;   // which 8x8 matrix this lane addresses
            const uint32_t a_addr = k_base + (uint32_t)((((mi & 1) * 8 + (lane & 7)) * C::KS + (mi >> 1) * 8) * 2);
            const uint32_t b_addr = q_base + (uint32_t)(((lane & 7) * C::QS + ((lane >> 3) & 1) * 8) * 2);
#pragma unroll
            for (int ks = 0; ks < C::DQKP / 16; ++ks) {
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4(a_addr + ks * 32, a0, a1, a2, a3);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    uint32_t b0, b1;
                    ldmatrix_x2(b_addr + (uint32_t)(nt * 8 * C::QS * 2) + ks * 32, b0, b1);
                    mma_16816<T>(s[nt], a0, a1, a2, a3, b0, b1);
                }
            }
        }

        // scale, mask, online softmax (log2 domain).  s[nt][c]: key g8 + 8*(c>>1), row 2*t4 + (c&1)
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float bmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int rc = c & 1;
                const int64_t j = kb * 16 + g8 + 8 * (c >> 1);
                float x = s[nt][c] * p.scale_log2;
                bool keep = row_ok[nt][rc] && j < p.Lk;
                if (keep) {
                    const int64_t moff = b * p.sm[0] + row_h[nt][rc] * p.sm[1] + row_i[nt][rc] * p.sm[2] + j * p.sm[3];
                    if (p.mask_kind == 1) {
                        x += Elem<T>::to_float(reinterpret_cast<const T*>(p.mask)[moff]) * log2e;
                    } else if (p.mask_kind == 2) {
                        keep = reinterpret_cast<const uint8_t*>(p.mask)[moff] != 0;
                    } else if (p.mask_kind == 3) {
                        keep = j <= row_i[nt][rc] + p.Lk - p.Lq;
                    }
                }
                x = keep ? x : -INFINITY;
                s[nt][c] = x;
                bmax[rc] = fmaxf(bmax[rc], x);
            }
            float alpha[2], m_use[2];
#pragma unroll
            for (int rc = 0; rc < 2; ++rc) {
                float v = bmax[rc];
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                const float m_new = fmaxf(m_run[nt][rc], v);
                m_use[rc] = (m_new == -INFINITY) ? 0.f : m_new;
                alpha[rc] = fast_exp2(m_run[nt][rc] - m_use[rc]);
                m_run[nt][rc] = m_new;
            }
            float pr[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) pr[c] = fast_exp2(s[nt][c] - m_use[c & 1]);
            l_run[nt][0] = l_run[nt][0] * alpha[0] + pr[0] + pr[2];
            l_run[nt][1] = l_run[nt][1] * alpha[1] + pr[1] + pr[3];
#pragma unroll
            for (int mt = 0; mt < C::DVP / 16; ++mt) {
                o[mt][nt][0] *= alpha[0];
                o[mt][nt][1] *= alpha[1];
                o[mt][nt][2] *= alpha[0];
                o[mt][nt][3] *= alpha[1];
            }
            pb[nt][0] = movmatrix_trans(pack2<T>(pr[0], pr[1]));   // keys 0-7
            pb[nt][1] = movmatrix_trans(pack2<T>(pr[2], pr[3]));   // keys 8-15
        }

        // O^T[DV][rows] += V^T . P^T
        {
            const int mi = lane >> 3;
            const uint32_t a_addr = v_base + (uint32_t)((((mi >> 1) * 8 + (lane & 7)) * C::VS + (mi & 1) * 8) * 2);
#pragma unroll
            for (int mt = 0; mt < C::DVP / 16; ++mt) {
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4_trans(a_addr + mt * 32, a0, a1, a2, a3);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_16816<T>(o[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();

    // ---- row sums across the 8 lanes that share a row
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int rc = 0; rc < 2; ++rc) {
            float v = l_run[nt][rc];
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            l_run[nt][rc] = v;
        }

    // ---- merge the W warps through shared memory (ring is free now)
    __syncthreads();
    constexpr int MS = C::DVP + 2;   // per row: DVP outputs, then m, l
    float* mw = merge + (size_t)warp * C::ROWS * MS;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int mt = 0; mt < C::DVP / 16; ++mt) {
            const int r0 = nt * 8 + 2 * t4;
            mw[r0 * MS + mt * 16 + g8] = o[mt][nt][0];
            mw[(r0 + 1) * MS + mt * 16 + g8] = o[mt][nt][1];
            mw[r0 * MS + mt * 16 + g8 + 8] = o[mt][nt][2];
            mw[(r0 + 1) * MS + mt * 16 + g8 + 8] = o[mt][nt][3];
        }
        if (g8 == 0) {
            const int r0 = nt * 8 + 2 * t4;
            mw[r0 * MS + C::DVP] = m_run[nt][0];
            mw[r0 * MS + C::DVP + 1] = l_run[nt][0];
            mw[(r0 + 1) * MS + C::DVP] = m_run[nt][1];
            mw[(r0 + 1) * MS + C::DVP + 1] = l_run[nt][1];
        }
    }
    __syncthreads();

    for (int idx = tid; idx < C::ROWS * (DV / 2); idx += W * 32) {
        const int r = idx / (DV / 2), e = (idx % (DV / 2)) * 2;
        const int64_t gr = row0 + r;
        if (gr >= R) continue;
        float mmax = -INFINITY;
#pragma unroll
        for (int w = 0; w < W; ++w) mmax = fmaxf(mmax, merge[((size_t)w * C::ROWS + r) * MS + C::DVP]);
        float L = 0.f, o0 = 0.f, o1 = 0.f;
        if (mmax != -INFINITY) {
#pragma unroll
            for (int w = 0; w < W; ++w) {
                const float* row = merge + ((size_t)w * C::ROWS + r) * MS;
                const float f = fast_exp2(row[C::DVP] - mmax);   // -inf -> 0
                L += row[C::DVP + 1] * f;
                o0 += row[e] * f;
                o1 += row[e + 1] * f;
            }
        }
        const float inv = (L > 0.f) ? 1.f / L : 0.f;
        const int64_t h = hkv * G + gr / p.Lq, i = gr % p.Lq;
        if (p.splits == 1) {
            T* og = reinterpret_cast<T*>(p.out) + b * p.so[0] + h * p.so[1] + i * p.so[2] + e;
            *reinterpret_cast<uint32_t*>(og) = pack2<T>(o0 * inv, o1 * inv);
        } else {
            const int64_t row = ((int64_t)b * p.Hq + h) * p.Lq + i;
            float* po = p.part_o + (row * p.splits + split) * DV + e;
            *reinterpret_cast<float2*>(po) = make_float2(o0 * inv, o1 * inv);
            if (e == 0) p.part_lse[row * p.splits + split] = (L > 0.f) ? mmax + log2f(L) : -INFINITY;
        }
    }
}

// ---------------------------------------------------------------- host side
struct Shape {
    int nt, w;
    size_t smem;
};

template <int DQK, int DV, int NT, int W>
Shape shape_of() {
    return Shape{NT, W, DecodeCfg<DQK, DV, NT, W>::smem_bytes};
}

// NT options per head dim: the O^T accumulators take DVP*NT/4 registers per thread.
Shape pick_shape(int64_t Dqk, int64_t Dv, int64_t rows) {
    const int need = (int)((rows + 7) / 8);
    const int cap = (Dv >= 512) ? 1 : (Dv >= 256 ? 2 : 4);
    int nt = 1;
    while (nt < need && nt < cap) nt *= 2;
    switch (Dqk * 1000 + Dv) {
#define SDPA_DECODE_SHAPE(DQ, DVV, W)                                          \
    case DQ * 1000 + DVV:                                                      \
        if (nt == 1) return shape_of<DQ, DVV, 1, W>();                         \
        if (nt == 2 && (DVV) < 512) return shape_of<DQ, DVV, ((DVV) < 512 ? 2 : 1), W>(); \
        return shape_of<DQ, DVV, ((DVV) < 256 ? 4 : 1), W>();
        SDPA_DECODE_SHAPE(64, 64, 4)
        SDPA_DECODE_SHAPE(72, 72, 4)
        SDPA_DECODE_SHAPE(80, 80, 4)
        SDPA_DECODE_SHAPE(96, 96, 4)
        SDPA_DECODE_SHAPE(128, 128, 4)
        SDPA_DECODE_SHAPE(192, 128, 4)
        SDPA_DECODE_SHAPE(256, 256, 4)
        SDPA_DECODE_SHAPE(512, 512, 2)
#undef SDPA_DECODE_SHAPE
        default: return Shape{0, 0, 0};
    }
}

template <typename T, int DQK, int DV, int NT, int W>
cudaError_t launch_one(const AttnParams& p, const LaunchPlan& plan, cudaStream_t stream) {
    auto kern = decode_mma_kernel<T, DQK, DV, NT, W>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem_bytes);
    if (e != cudaSuccess) return e;
    kern<<<plan.grid, plan.block, plan.smem_bytes, stream>>>(p, plan.variant);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(const AttnParams& p, const LaunchPlan& plan, cudaStream_t s) {
    const int nt = plan.aux;
    const LaunchPlan& pl = plan;
    switch (p.Dqk * 1000 + p.Dv) {
#define SDPA_DECODE_LAUNCH(DQ, DVV, W)                                                  \
    case DQ * 1000 + DVV:                                                               \
        if (nt == 1) return launch_one<T, DQ, DVV, 1, W>(p, pl, s);                     \
        if (nt == 2) return launch_one<T, DQ, DVV, ((DVV) < 512 ? 2 : 1), W>(p, pl, s); \
        return launch_one<T, DQ, DVV, ((DVV) < 256 ? 4 : 1), W>(p, pl, s);
        SDPA_DECODE_LAUNCH(64, 64, 4)
        SDPA_DECODE_LAUNCH(72, 72, 4)
        SDPA_DECODE_LAUNCH(80, 80, 4)
        SDPA_DECODE_LAUNCH(96, 96, 4)
        SDPA_DECODE_LAUNCH(128, 128, 4)
        SDPA_DECODE_LAUNCH(192, 128, 4)
        SDPA_DECODE_LAUNCH(256, 256, 4)
        SDPA_DECODE_LAUNCH(512, 512, 2)
#undef SDPA_DECODE_LAUNCH
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool decode_mma_supported(int dtype, int64_t Dqk, int64_t Dv) {
    return (dtype == 1 || dtype == 2) && pick_shape(Dqk, Dv, 8).smem != 0;
}

LaunchPlan decode_mma_plan(const AttnParams& p, int dtype, const DeviceInfo& dev) {
    (void)dtype;
    LaunchPlan plan{};
    const int64_t rows = (int64_t)p.group * p.Lq;
    const Shape sh = pick_shape(p.Dqk, p.Dv, rows);
    const int64_t RG = (rows + 8 * sh.nt - 1) / (8 * sh.nt);
    const int64_t nkb = (p.Lk + 15) / 16;
    // CTAs one SM holds at once (shared memory bound; registers allow more).
    int per_sm = (int)((228 * 1024) / (sh.smem + 1024));
    if (per_sm < 1) per_sm = 1;
    if (per_sm > 4) per_sm = 4;
    const int64_t base = p.B * p.Hkv * RG;
    const int64_t slots = (int64_t)dev.sm_count * per_sm;
    int64_t splits = slots / base;                        // one wave, no tail
    const int64_t max_splits = (nkb + sh.w - 1) / sh.w;   // at least one block per warp
    if (splits > max_splits) splits = max_splits;
    if (splits > 256) splits = 256;
    if (splits < 1) splits = 1;
    if (const char* env = getenv("SDPA_DECODE_SPLITS")) {
        const long v = strtol(env, nullptr, 10);
        if (v >= 1 && v <= 4096) splits = v;
    }
    int64_t kbps = (nkb + splits - 1) / splits;
    if (kbps < 1) kbps = 1;
    splits = (nkb + kbps - 1) / kbps;
    if (splits < 1) splits = 1;
    plan.grid = dim3((unsigned)splits, (unsigned)(p.Hkv * RG), (unsigned)p.B);
    plan.block = dim3((unsigned)(sh.w * 32), 1, 1);
    plan.smem_bytes = sh.smem;
    plan.splits = (int)splits;
    plan.keys_per_split = kbps * 16;
    plan.variant = (int)RG;
    plan.aux = sh.nt;
    return plan;
}

cudaError_t decode_mma_launch(const AttnParams& p, int dtype, const LaunchPlan& plan, cudaStream_t stream) {
    if (dtype == 1) return launch_typed<__half>(p, plan, stream);
    if (dtype == 2) return launch_typed<__nv_bfloat16>(p, plan, stream);
    return cudaErrorInvalidValue;
}

}  // namespace sdpa
