// prefill_tf32.cu -- fp32 prefill attention on 5th-generation tensor cores
// with a three-term TF32 split, held to fp32 accuracy.
//
// mlxcel issue #1065, section "Root cause: MLX_ENABLE_TF32, not the M5
// neural-accelerator attention route": fp32 attention that lets TF32 (10
// mantissa bits) into its products shows errors near 2^-10.  Here every fp32
// operand x is split into hi = x rounded to TF32 and lo = (x - hi) rounded to
// TF32, and each product is taken as hi*hi + hi*lo + lo*hi on the tensor core
// (tcgen05.mma kind::tf32, fp32 accumulation in TMEM): the dropped lo*lo term
// and the rounding of lo are about 2^-22 of |x||y|, the fp32 class.
//
// One CTA computes a 128-row query tile of one (batch, query head), 64 keys
// per tile:
//   warp 0      TMA producer: Q once, then K(j) and V(j) as fp32 tiles
//               (32-element, 128-byte swizzled chunks) into NSTAGE stages;
//   warp 1      TMEM owner and MMA issuer: S(j) = Qh Kh^T + Qh Kl^T + Ql Kh^T
//               into one of two TMEM S buffers, then O += Ph Vh + Ph Vl + Pl Vh
//               with P read from TMEM (Ph over its S buffer, Pl in columns of
//               its own) and V^T read K-major from shared memory (every tf32
//               operand here is K-major: that is the form the 128-byte swizzle
//               of the tiles describes for 32-bit elements);
//   warps 2-7   split each landed tile: Q and K in place (hi over the raw
//               values, lo into a buffer of the same swizzled layout, so the
//               split is element-wise and both copies take one descriptor
//               form), V transposed into K-major V^T hi and lo tiles;
//   warps 8-11  softmax: thread t owns query row t (TMEM lane t), fp32 running
//               max / sum in the log2 domain, masks (none, additive, boolean,
//               causal, sliding window), P split into hi / lo and written to
//               TMEM, O rescaled in TMEM only when the row maximum grew by more
//               than 2^8, and the epilogue O / l stored through the out strides.
// Head dims: (64, 64) with two stages, (72, 72), (80, 80), (96, 96) with one
// stage (the hi / lo copies of Q, K and V double the shared memory of a tile),
// and the absorbed-MLA pair (40, 32).  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace sdpa {
namespace {

constexpr int kBMf = 128;                 // query rows per CTA (UMMA M)
constexpr int kBNf = 64;                  // keys per tile (UMMA N of S, K of P V)
constexpr int kQChunk = kBMf * 128;       // 128 rows x 32 fp32
constexpr int kKChunk = kBNf * 128;       // 64 rows x 32 fp32
constexpr int kThreadsF = 384;            // 12 warps
constexpr int kSplitThreads = 192;        // warps 2-7 split each landed tile into hi / lo
constexpr float kRescaleThresholdF = 8.0f;

__host__ __device__ constexpr int cdivf(int a, int b) { return (a + b - 1) / b; }

template <int DQK, int DV, int NSTAGE>
struct Tf32Cfg {
    static constexpr int NQ = cdivf(DQK, 32);        // 32-element chunks of a Q / K row
    static constexpr int NV = cdivf(DV, 32);         // chunks of a V row
    static constexpr int KSTEPS = DQK / 8;           // K steps of S (8 tf32 each)
    static constexpr int DVP = cdivf(DV, 16) * 16;   // O columns (N of P V, a multiple of 16)
    static constexpr int Q_BYTES = NQ * kQChunk;
    static constexpr int K_BYTES = NQ * kKChunk;
    static constexpr int V_BYTES = NV * kKChunk;                     // V as loaded: [key][dv]
    static constexpr int VT_CHUNK = DVP * 128;                       // V^T: 32 keys of DVP rows
    static constexpr int VT_BYTES = (kBNf / 32) * VT_CHUNK;
    static constexpr int STAGE_BYTES = 2 * K_BYTES + V_BYTES + 2 * VT_BYTES;   // Kh, Kl, V, V^T h, V^T l
    static constexpr int OFF_QH = 0, OFF_QL = Q_BYTES, OFF_STAGES = 2 * Q_BYTES;
    static constexpr int OFF_BAR = OFF_STAGES + NSTAGE * STAGE_BYTES;
    // q full / conv; per stage K full / conv / empty and V full / conv / empty;
    // S full [2]; P full [2]; O done; drain
    static constexpr int NUM_BARS = 2 + 6 * NSTAGE + 2 + 2 + 1 + 1;
    static constexpr int SMEM = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t S_COL = 0, PL_COL = 2 * kBNf, O_COL = 4 * kBNf;
    static_assert(DQK % 8 == 0, "TF32 K steps of 8");
    static_assert(O_COL + DVP <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct Tf32Params {
    AttnParams p;
    MapAxes q_ax, k_ax, v_ax;
    int q_tiles;
};

__device__ __forceinline__ uint32_t tf32_round(uint32_t bits) {
    // nearest TF32 (10 fraction bits), ties away from zero: sign-magnitude
    // makes the same integer step right for both signs
    return (bits + 0x1000u) & 0xffffe000u;
}

// hi (in place) and lo of `bytes` bytes at `hi`, by `n` threads (thread t of n)
__device__ __forceinline__ void split_tf32(unsigned char* hi, unsigned char* lo, int bytes, int t, int n) {
    for (int i = t; i < bytes / 16; i += n) {
        uint4 x = *reinterpret_cast<const uint4*>(hi + 16 * i);
        uint4 h, l;
        h.x = tf32_round(x.x);
        h.y = tf32_round(x.y);
        h.z = tf32_round(x.z);
        h.w = tf32_round(x.w);
        l.x = tf32_round(__float_as_uint(__uint_as_float(x.x) - __uint_as_float(h.x)));
        l.y = tf32_round(__float_as_uint(__uint_as_float(x.y) - __uint_as_float(h.y)));
        l.z = tf32_round(__float_as_uint(__uint_as_float(x.z) - __uint_as_float(h.z)));
        l.w = tf32_round(__float_as_uint(__uint_as_float(x.w) - __uint_as_float(h.w)));
        *reinterpret_cast<uint4*>(hi + 16 * i) = h;
        *reinterpret_cast<uint4*>(lo + 16 * i) = l;
    }
}

// V(j) as loaded ([key][dv] in NV chunks of 64 keys x 32 dv, 128-byte
// swizzled rows) -> V^T hi and lo as K-major tiles for the P V MMA: for each
// chunk of 32 keys, DVP rows (dv) of 128 bytes (32 keys), 128-byte swizzled.
// Rows dv >= NV * 32 do not exist (DVP <= NV * 32).  By `n` threads, n a
// multiple of 32: the 32 lanes of a warp take 32 consecutive keys of one
// 16-byte unit, so each quarter-warp reads 8 distinct swizzled units and each
// transposed store of the warp hits 32 distinct banks.
template <int NV, int DVP>
__device__ __forceinline__ void split_transpose_v(const unsigned char* raw, unsigned char* th, unsigned char* tl,
                                                  int t, int n) {
    constexpr int VT_CHUNK = DVP * 128;
    for (int i = t; i < NV * 64 * 8; i += n) {   // 16-byte units: chunk c, key chunk kc, logical unit u, key kk
        const int kk = i & 31, u = (i >> 5) & 7, kc = (i >> 8) & 1, c = i >> 9;
        const int r = kc * 32 + kk;
        const uint4 x = *reinterpret_cast<const uint4*>(raw + c * kKChunk + r * 128 + ((u ^ (r & 7)) << 4));
        const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) {
            const int e = c * 32 + u * 4 + e4;   // dv row of V^T
            if (e >= DVP) continue;
            const uint32_t off = kc * VT_CHUNK + e * 128 + ((((kk >> 2) ^ (e & 7)) << 4) | ((kk & 3) << 2));
            const uint32_t h = tf32_round(xs[e4]);
            const uint32_t l = tf32_round(__float_as_uint(__uint_as_float(xs[e4]) - __uint_as_float(h)));
            *reinterpret_cast<uint32_t*>(th + off) = h;
            *reinterpret_cast<uint32_t*>(tl + off) = l;
        }
    }
}

// Instruction descriptor, kind::tf32 with fp32 accumulation (formats TF32 = 2).
__host__ __device__ constexpr uint32_t umma_idesc_tf32(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_tf32_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tmem_ld16f(uint32_t taddr, uint32_t (&o)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]), "=r"(o[4]), "=r"(o[5]), "=r"(o[6]), "=r"(o[7]), "=r"(o[8]),
          "=r"(o[9]), "=r"(o[10]), "=r"(o[11]), "=r"(o[12]), "=r"(o[13]), "=r"(o[14]), "=r"(o[15])
        : "r"(taddr));
}

template <int DQK, int DV, int NSTAGE, int MASK>
__global__ void __launch_bounds__(kThreadsF, 1)
    prefill_tf32_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const Tf32Params tp) {
    using C = Tf32Cfg<DQK, DV, NSTAGE>;
    const AttnParams& p = tp.p;
    extern __shared__ unsigned char smem_dyn[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* bar_q_full = bars;
    uint64_t* bar_q_conv = bars + 1;
    uint64_t* bar_k_full = bars + 2;                 // [NSTAGE]
    uint64_t* bar_k_conv = bar_k_full + NSTAGE;
    uint64_t* bar_k_empty = bar_k_conv + NSTAGE;
    uint64_t* bar_v_full = bar_k_empty + NSTAGE;
    uint64_t* bar_v_conv = bar_v_full + NSTAGE;
    uint64_t* bar_v_empty = bar_v_conv + NSTAGE;
    uint64_t* bar_s_full = bar_v_empty + NSTAGE;     // [2]
    uint64_t* bar_p_full = bar_s_full + 2;           // [2]
    uint64_t* bar_o_done = bar_p_full + 2;
    uint64_t* bar_drain = bar_o_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
    auto kh = [&](int st) { return C::OFF_STAGES + st * C::STAGE_BYTES; };
    auto kl = [&](int st) { return C::OFF_STAGES + st * C::STAGE_BYTES + C::K_BYTES; };
    auto vraw = [&](int st) { return C::OFF_STAGES + st * C::STAGE_BYTES + 2 * C::K_BYTES; };
    auto vth = [&](int st) { return C::OFF_STAGES + st * C::STAGE_BYTES + 2 * C::K_BYTES + C::V_BYTES; };
    auto vtl = [&](int st) {
        return C::OFF_STAGES + st * C::STAGE_BYTES + 2 * C::K_BYTES + C::V_BYTES + C::VT_BYTES;
    };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qt = (MASK == 3) ? (tp.q_tiles - 1 - (int)blockIdx.x) : (int)blockIdx.x;   // heavy tiles first
    const int hq = blockIdx.y, b = blockIdx.z;
    const int hkv = hq / p.group;
    const int64_t q0 = (int64_t)qt * kBMf;

    // key tiles this query tile needs (causal: up to the diagonal; sliding
    // window: from the first row's window start)
    int t0 = 0, n_tiles = 0;
    {
        int64_t k_end = p.Lk, k_begin = 0;
        if (MASK == 3 || MASK == 4) {
            const int64_t last = q0 + kBMf - 1 + p.Lk - p.Lq;
            k_end = last < 0 ? 0 : (last + 1 < p.Lk ? last + 1 : p.Lk);
        }
        if (MASK == 4) {
            const int64_t first = q0 + p.Lk - p.Lq - p.window + 1;
            k_begin = first < 0 ? 0 : first;
        }
        t0 = (int)(k_begin / kBNf);
        const int64_t t_end = (k_end + kBNf - 1) / kBNf;
        n_tiles = t_end > t0 ? (int)(t_end - t0) : 0;
    }

    if (threadIdx.x == 0) {
        mbar_init(bar_q_full, 1);
        mbar_init(bar_q_conv, kSplitThreads);
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(bar_k_full + s, 1);
            mbar_init(bar_k_conv + s, kSplitThreads);
            mbar_init(bar_k_empty + s, 1);
            mbar_init(bar_v_full + s, 1);
            mbar_init(bar_v_conv + s, kSplitThreads);
            mbar_init(bar_v_empty + s, 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_s_full + s, 1);
            mbar_init(bar_p_full + s, 128);
        }
        mbar_init(bar_o_done, 1);
        mbar_init(bar_drain, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && n_tiles > 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(bar_q_full, C::Q_BYTES);
            for (int c = 0; c < C::NQ; ++c)
                tma_load(s_base + C::OFF_QH + c * kQChunk, &tmQ, bar_q_full, tp.q_ax, c * 32, (int)q0, hq, b);
            bool ok = true;
            int j = 0;
            for (; j < n_tiles && ok; ++j) {
                const int st = j % NSTAGE;
                const uint32_t par = ((j / NSTAGE) & 1) ^ 1;
                const int key0 = (t0 + j) * kBNf;
                if (j >= NSTAGE && !(ok = wait_phase(bar_k_empty + st, par, kErrWaitSlot))) break;
                mbar_arrive_expect_tx(bar_k_full + st, C::K_BYTES);
                for (int c = 0; c < C::NQ; ++c)
                    tma_load(s_base + kh(st) + c * kKChunk, &tmK, bar_k_full + st, tp.k_ax, c * 32, key0, hkv, b);
                if (j >= NSTAGE && !(ok = wait_phase(bar_v_empty + st, par, kErrWaitSlot))) {
                    wait_phase(bar_k_full + st, (j / NSTAGE) & 1, kErrWaitTmaLoad);   // K(j) is in flight
                    break;
                }
                mbar_arrive_expect_tx(bar_v_full + st, C::V_BYTES);
                for (int c = 0; c < C::NV; ++c)
                    tma_load(s_base + vraw(st) + c * kKChunk, &tmV, bar_v_full + st, tp.v_ax, c * 32, key0, hkv, b);
            }
            if (!ok) {
                // drain: every issued load lands before the CTA's shared memory goes away
                wait_phase(bar_q_full, 0, kErrWaitTmaLoad);
                for (int x = (j > NSTAGE ? j - NSTAGE : 0); x < j; ++x) {
                    wait_phase(bar_k_full + x % NSTAGE, (x / NSTAGE) & 1, kErrWaitTmaLoad);
                    wait_phase(bar_v_full + x % NSTAGE, (x / NSTAGE) & 1, kErrWaitTmaLoad);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_tiles > 0) {
            constexpr uint32_t idS = umma_idesc_tf32(kBMf, kBNf, 0, 0);
            constexpr uint32_t idPV = umma_idesc_tf32(kBMf, C::DVP, 0, 0);
            bool ok = wait_phase(bar_q_conv, 0, kErrWaitSplit);
            auto issue_s = [&](int j) -> bool {   // S(j) = Qh Kh^T + Qh Kl^T + Ql Kh^T
                const int st = j % NSTAGE;
                if (!wait_phase(bar_k_conv + st, (j / NSTAGE) & 1, kErrWaitSplit)) return false;
                tc_fence_after();
                const uint32_t d = tmem + C::S_COL + (uint32_t)((j & 1) * kBNf);
#pragma unroll
                for (int k = 0; k < C::KSTEPS; ++k) {
                    const uint32_t qo = (uint32_t)((k >> 2) * kQChunk + (k & 3) * 32);
                    const uint32_t ko = (uint32_t)((k >> 2) * kKChunk + (k & 3) * 32);
                    const uint64_t a_h = umma_desc_sw128(s_base + C::OFF_QH + qo, 16, 1024);
                    const uint64_t a_l = umma_desc_sw128(s_base + C::OFF_QL + qo, 16, 1024);
                    const uint64_t b_h = umma_desc_sw128(s_base + kh(st) + ko, 16, 1024);
                    const uint64_t b_l = umma_desc_sw128(s_base + kl(st) + ko, 16, 1024);
                    umma_tf32_ss(d, a_h, b_h, idS, k > 0 ? 1u : 0u);
                    umma_tf32_ss(d, a_h, b_l, idS, 1u);
                    umma_tf32_ss(d, a_l, b_h, idS, 1u);
                }
                umma_commit(bar_k_empty + st);
                umma_commit(bar_s_full + (j & 1));
                return true;
            };
            auto issue_pv = [&](int j) -> bool {   // O += Ph Vh + Ph Vl + Pl Vh
                const int st = j % NSTAGE;
                if (!wait_phase(bar_v_conv + st, (j / NSTAGE) & 1, kErrWaitSplit)) return false;
                tc_fence_after();
                const uint32_t a_h = tmem + C::S_COL + (uint32_t)((j & 1) * kBNf);
                const uint32_t a_l = tmem + C::PL_COL + (uint32_t)((j & 1) * kBNf);
#pragma unroll
                for (int ks = 0; ks < kBNf / 8; ++ks) {   // 8 keys per step, K-major V^T
                    const uint32_t vo = (uint32_t)((ks >> 2) * C::VT_CHUNK + (ks & 3) * 32);
                    const uint64_t b_h = umma_desc_sw128(s_base + vth(st) + vo, 16, 1024);
                    const uint64_t b_l = umma_desc_sw128(s_base + vtl(st) + vo, 16, 1024);
                    umma_tf32_ts(tmem + C::O_COL, a_h + ks * 8, b_h, idPV, (j > 0 || ks > 0) ? 1u : 0u);
                    umma_tf32_ts(tmem + C::O_COL, a_h + ks * 8, b_l, idPV, 1u);
                    umma_tf32_ts(tmem + C::O_COL, a_l + ks * 8, b_h, idPV, 1u);
                }
                umma_commit(bar_v_empty + st);
                umma_commit(bar_o_done);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int j = 0; j < n_tiles && ok; ++j) {
                // S(j+1) goes into the buffer Ph(j-1) was read from; the MMAs of one
                // thread execute in order, so it may follow P(j-1) V(j-1) at once
                if (j + 1 < n_tiles && !(ok = issue_s(j + 1))) break;
                if (!(ok = wait_phase(bar_p_full + (j & 1), (j >> 1) & 1, kErrWaitSoftmax))) break;
                tc_fence_after();
                if (!(ok = issue_pv(j))) break;
            }
            // every MMA issued by this thread completes before TMEM can be freed
            umma_commit(bar_drain);
            wait_phase(bar_drain, 0, kErrWaitMma);
        }
    } else if (warp < 2 + kSplitThreads / 32) {
        // ------------------------------------------------------------ hi / lo split
        const int t = threadIdx.x - 64;
        if (n_tiles > 0) {
            bool ok = wait_phase(bar_q_full, 0, kErrWaitTmaLoad);
            if (ok) {
                split_tf32(smem + C::OFF_QH, smem + C::OFF_QL, C::Q_BYTES, t, kSplitThreads);
                fence_proxy_async();   // the tensor core reads them through the async proxy
                mbar_arrive(bar_q_conv);
            }
            for (int j = 0; j < n_tiles && ok; ++j) {
                const int st = j % NSTAGE;
                const uint32_t par = (j / NSTAGE) & 1;
                if (!(ok = wait_phase(bar_k_full + st, par, kErrWaitTmaLoad))) break;
                split_tf32(smem + kh(st), smem + kl(st), C::K_BYTES, t, kSplitThreads);
                fence_proxy_async();
                mbar_arrive(bar_k_conv + st);
                if (!(ok = wait_phase(bar_v_full + st, par, kErrWaitTmaLoad))) break;
                split_transpose_v<C::NV, C::DVP>(smem + vraw(st), smem + vth(st), smem + vtl(st), t, kSplitThreads);
                fence_proxy_async();
                mbar_arrive(bar_v_conv + st);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax / epilogue
        const int quad = warp & 3;   // warps 8..11 -> TMEM lane quadrants 0..3
        const int r = quad * 32 + lane;
        const int64_t i = q0 + r;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const bool row_ok = i < p.Lq;
        const int64_t own = i + p.Lk - p.Lq;
        const int64_t mrow = (int64_t)b * p.sm[0] + (int64_t)hq * p.sm[1] + i * p.sm[2];
        const float sc = p.scale_log2;
        const float log2e = 1.4426950408889634f;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            const int buf = j & 1;
            ok = __all_sync(0xffffffffu, wait_phase(bar_s_full + buf, (j >> 1) & 1, kErrWaitMma));
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[kBNf];
            tmem_ld32(tmem + lane_off + C::S_COL + buf * kBNf, *reinterpret_cast<uint32_t(*)[32]>(sr));
            tmem_ld32(tmem + lane_off + C::S_COL + buf * kBNf + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
            tmem_wait_ld();
            const int64_t kbase = (int64_t)(t0 + j) * kBNf;
            // keys [lo, vis) of this tile are visible to the row
            int64_t lim = p.Lk - kbase;
            if (MASK == 3 || MASK == 4) lim = min(lim, own - kbase + 1);
            const int vis = row_ok ? (int)max((int64_t)0, min(lim, (int64_t)kBNf)) : 0;
            const int lo = (MASK == 4) ? (int)max((int64_t)0, min(own - p.window + 1 - kbase, (int64_t)kBNf)) : 0;
            float mloc = -INFINITY;
#pragma unroll
            for (int c = 0; c < kBNf; ++c) {
                float x = __uint_as_float(sr[c]) * sc;
                bool keep = c >= lo && c < vis;
                if (MASK == 1 && keep) x += reinterpret_cast<const float*>(p.mask)[mrow + (kbase + c) * p.sm[3]] * log2e;
                if (MASK == 2 && keep) keep = reinterpret_cast<const uint8_t*>(p.mask)[mrow + (kbase + c) * p.sm[3]] != 0;
                x = keep ? x : -INFINITY;
                sr[c] = __float_as_uint(x);
                mloc = fmaxf(mloc, x);
            }
            const float m_new = fmaxf(m_ref, mloc);
            float alpha = 1.f;
            bool rescale = false;
            if (m_new != -INFINITY && (m_ref == -INFINITY || m_new > m_ref + kRescaleThresholdF)) {
                rescale = (m_ref != -INFINITY);   // before the first finite max, O holds nothing yet
                alpha = rescale ? exp2f(m_ref - m_new) : 0.f;
                m_ref = m_new;
            }
            const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
            l *= alpha;
            if (j > 0) {   // P(j-1) V(j-1) done: the P columns of tile j are free and O may be rescaled
                ok = __all_sync(0xffffffffu, wait_phase(bar_o_done, (j - 1) & 1, kErrWaitMma));
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, rescale)) {
                    const float f = rescale ? alpha : 1.f;
#pragma unroll
                    for (int c = 0; c < C::DVP / 16; ++c) {
                        uint32_t o[16];
                        tmem_ld16f(tmem + lane_off + C::O_COL + c * 16, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int u = 0; u < 16; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * f);
                        tmem_st16(tmem + lane_off + C::O_COL + c * 16, o);
                    }
                }
            }
            // P = 2^(x - m), split into hi (over the S columns just read) and lo,
            // 32 keys at a time
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int h = 0; h < kBNf / 32; ++h) {
                uint32_t ph[32], pl[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float pv = exp2f(__uint_as_float(sr[h * 32 + c]) - m_use);   // -inf -> 0
                    acc[c & 3] += pv;
                    ph[c] = tf32_round(__float_as_uint(pv));
                    pl[c] = tf32_round(__float_as_uint(pv - __uint_as_float(ph[c])));
                }
                tmem_st32(tmem + lane_off + C::S_COL + buf * kBNf + h * 32, ph);
                tmem_st32(tmem + lane_off + C::PL_COL + buf * kBNf + h * 32, pl);
                tmem_wait_st();
            }
            l += (acc[0] + acc[1]) + (acc[2] + acc[3]);
            tc_fence_before();
            mbar_arrive(bar_p_full + buf);
        }
        // epilogue: O / l stored through the output strides
        if (ok && n_tiles > 0) ok = __all_sync(0xffffffffu, wait_phase(bar_o_done, (n_tiles - 1) & 1, kErrWaitMma));
        tc_fence_after();
        const bool have = ok && n_tiles > 0;
        const float inv = (have && l > 0.f) ? 1.f / l : 0.f;
        float* og = reinterpret_cast<float*>(p.out) + (int64_t)b * p.so[0] + (int64_t)hq * p.so[1] + i * p.so[2];
#pragma unroll
        for (int c = 0; c < C::DVP / 16; ++c) {
            uint32_t o[16];
            if (have) {
                tmem_ld16f(tmem + lane_off + C::O_COL + c * 16, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int u = 0; u < 16; ++u) o[u] = 0u;
            }
            if (row_ok) {
#pragma unroll
                for (int u4 = 0; u4 < 4; ++u4)
                    if (c * 16 + u4 * 4 < DV)
                        *reinterpret_cast<float4*>(og + c * 16 + u4 * 4) =
                            make_float4(__uint_as_float(o[4 * u4]) * inv, __uint_as_float(o[4 * u4 + 1]) * inv,
                                        __uint_as_float(o[4 * u4 + 2]) * inv, __uint_as_float(o[4 * u4 + 3]) * inv);
            }
        }
    }

    // teardown: every role has drained its asynchronous work
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// (Dqk, Dv, stages)
#define SDPA_TF32_VARIANTS(X) \
    X(40, 32, 2)              \
    X(64, 64, 2)              \
    X(72, 72, 1)              \
    X(80, 80, 1)              \
    X(96, 96, 1)

size_t tf32_smem(int64_t Dqk, int64_t Dv) {
    switch (Dqk * 1000 + Dv) {
#define SDPA_TF32_SMEM(DQ, DVV, NS) \
    case DQ * 1000 + DVV: return (size_t)Tf32Cfg<DQ, DVV, NS>::SMEM;
        SDPA_TF32_VARIANTS(SDPA_TF32_SMEM)
#undef SDPA_TF32_SMEM
        default: return 0;
    }
}

template <int DQK, int DV, int NS, int MASK>
cudaError_t launch_mask(const Tf32Params& tp, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        const LaunchPlan& plan, cudaStream_t stream) {
    auto kern = prefill_tf32_kernel<DQK, DV, NS, MASK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem_bytes);
    if (e != cudaSuccess) return e;
    kern<<<plan.grid, plan.block, plan.smem_bytes, stream>>>(mq, mk, mv, tp);
    return cudaGetLastError();
}

template <int DQK, int DV, int NS>
cudaError_t launch_dims(const Tf32Params& tp, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        const LaunchPlan& plan, cudaStream_t s) {
    switch (tp.p.mask_kind) {
        case 0: return launch_mask<DQK, DV, NS, 0>(tp, mq, mk, mv, plan, s);
        case 1: return launch_mask<DQK, DV, NS, 1>(tp, mq, mk, mv, plan, s);
        case 2: return launch_mask<DQK, DV, NS, 2>(tp, mq, mk, mv, plan, s);
        case 3: return launch_mask<DQK, DV, NS, 3>(tp, mq, mk, mv, plan, s);
        case 4: return launch_mask<DQK, DV, NS, 4>(tp, mq, mk, mv, plan, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool prefill_tf32_supported(int dtype, int64_t Dqk, int64_t Dv) { return dtype == 0 && tf32_smem(Dqk, Dv) != 0; }

int take_device_error_tf32(cudaStream_t stream) {
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

LaunchPlan prefill_tf32_plan(const AttnParams& p, const DeviceInfo& dev) {
    (void)dev;
    LaunchPlan plan{};
    const int64_t q_tiles = (p.Lq + kBMf - 1) / kBMf;
    plan.grid = dim3((unsigned)q_tiles, (unsigned)p.Hq, (unsigned)p.B);
    plan.block = dim3(kThreadsF);
    plan.smem_bytes = tf32_smem(p.Dqk, p.Dv);
    plan.splits = 1;
    plan.keys_per_split = p.Lk;
    plan.aux = (int)q_tiles;
    return plan;
}

cudaError_t prefill_tf32_launch(const AttnParams& p, const LaunchPlan& plan, cudaStream_t stream) {
    Tf32Params tp{};
    tp.p = p;
    tp.q_tiles = plan.aux;
    CUtensorMap mq, mk, mv;
    if (!make_tensor_map(&mq, &tp.q_ax, p.q, 0, p.Dqk, p.Lq, p.Hq, p.B, p.sq, kBMf) ||
        !make_tensor_map(&mk, &tp.k_ax, p.k, 0, p.Dqk, p.Lk, p.Hkv, p.B, p.sk, kBNf) ||
        !make_tensor_map(&mv, &tp.v_ax, p.v, 0, p.Dv, p.Lk, p.Hkv, p.B, p.sv, kBNf))
        return cudaErrorInvalidValue;
    switch (p.Dqk * 1000 + p.Dv) {
#define SDPA_TF32_LAUNCH(DQ, DVV, NS) \
    case DQ * 1000 + DVV: return launch_dims<DQ, DVV, NS>(tp, mq, mk, mv, plan, stream);
        SDPA_TF32_VARIANTS(SDPA_TF32_LAUNCH)
#undef SDPA_TF32_LAUNCH
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace sdpa
