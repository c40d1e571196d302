// decode_mma.cu -- split-K (flash-decoding) attention for short queries,
// fp16 / bf16, one launch: TMA loads, warp-level tensor-core MMA (m16n8k16,
// fp32 accumulation) and the log-sum-exp merge of the splits.
//
// The decode ("vector") path of MLX issue #3885 ("Metal SDPA: no fused path
// for head_dim=512 ..."), section "Current routing": qL <= 8.  Decode is bound
// by reading K and V (same issue, the bytes-normalised control: d * n_kv equal
// means equal K+V bytes).  Design points:
//
//  * one CTA serves every query row of a KV-head group (the G = Hq/Hkv query
//    heads times the qL queries), so each K/V byte is read once per group
//    (the MLX commit "Read each K/V byte once in gqa-8 decode attention");
//  * keys are split across CTAs (split-K) so that B*Hkv small problems still
//    occupy every SM: one CTA per SM, and when the SM count is not a multiple
//    of the group count the first groups take one split more, so no SM is left
//    idle (same issue: its two-pass kernel starves the grid when n_kv is small);
//  * one producer thread streams slots of SK keys of K and V with TMA (128-byte
//    swizzle, zero fill past Lk; one whole-row box per tensor and slot for head
//    dims that are multiples of 64) into a CTA-wide ring of ~192 KB, so most of
//    a CTA's share is requested at once and the consumer warps issue no load
//    instructions for K and V;
//  * consumer warp w takes the 16-key sub-blocks w, w+W, ... of the slots; the
//    additive / boolean mask values of its next sub-block are loaded while it
//    computes the current one; scores are computed transposed, S^T = K Q^T, so
//    the keys fill the 16-row side of the MMA and the few query rows the
//    8-column side; P^T reaches the B operand of O^T += V^T P^T with one
//    movmatrix per 8x8 block;
//  * each CTA merges its warps and writes its split's normalised partial and
//    log-sum-exp; the grid is a cooperative launch (all CTAs resident at once),
//    so the splits of a (batch, KV head, row group) meet at a bounded barrier
//    and then each CTA merges its own slice of the group's output, loading
//    every split's partial of its slice in one round trip.  The barrier is a
//    64-bit arrival counter per group that only grows: every call adds exactly
//    S (the group's split count; the workspace keeps separate counters per
//    launch shape), so a call's target is the next multiple of S above the
//    value it reads at start.  Arrivals are fire-and-forget reductions and no
//    CTA needs a second round trip to reset anything.
#include <cuda_runtime.h>
#include <math.h>
#include <stdlib.h>

#include "common.cuh"
#include "kernels.h"

namespace sdpa {
namespace {

constexpr int kMaxSplits = 256;

__host__ __device__ constexpr int round16(int x) { return (x + 15) / 16 * 16; }
__host__ __device__ constexpr int cdiv(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ constexpr int align1k(int x) { return (x + 1023) / 1024 * 1024; }
__host__ __device__ constexpr int imin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int imax(int a, int b) { return a > b ? a : b; }

// SK keys per ring slot; a slot holds K then V, each as 64-element column chunks
// of SK rows x 128 bytes (128-byte swizzle).
template <int DQK, int DV, int NT, int W, int NSLOT, int SK>
struct DecodeCfg {
    static constexpr int NSUB = SK / 16;         // 16-key sub-blocks per slot
    static constexpr int CHUNK = SK * 128;       // one 64-element column chunk of a slot
    static constexpr int DQKP = round16(DQK);    // MMA K extent (72 -> 80; TMA zero-fills the pad)
    static constexpr int DVP = round16(DV);
    static constexpr int NBK = cdiv(DQK, 64);    // 64-element chunks per K row block
    static constexpr int NBV = cdiv(DV, 64);
    static constexpr int SLOT = (NBK + NBV) * CHUNK;
    static constexpr int QS = DQKP + 8;          // Q smem row stride (elements): +16 B breaks bank conflicts
    static constexpr int ROWS = 8 * NT;          // query rows per CTA
    static constexpr int OFF_RING = align1k(ROWS * QS * 2);
    static constexpr int OFF_BAR = OFF_RING + NSLOT * SLOT;
    static constexpr int MS = DVP + 4;           // merge row: DVP outputs, then m, l (16-byte aligned rows)
    static constexpr int MERGE_FLOATS = W * ROWS * MS;
    static constexpr int OFF_ROWS = OFF_BAR + 2 * NSLOT * 8 + 16;
    static constexpr int OFF_COEF = OFF_ROWS + 2 * ROWS * 8;   // [ROWS][W + 1]: merge weights, then lse
    static constexpr int OFF_MPRE = (OFF_COEF + ROWS * (W + 1) * 4 + 127) / 128 * 128;
    static constexpr int MPRE = 8192;            // mask values of the CTA's keys, copied up front
    static constexpr int SMEM = OFF_MPRE + MPRE + 1024;
    // slots the producer keeps in flight: about 96 KB per SM (a deeper queue
    // only delays the first slot of every CTA, and every other load behind it)
    static constexpr int INFLIGHT = imin(imax(98304 / SLOT, 3), NSLOT);
    static constexpr int THREADS = (W + 1) * 32;
    static_assert(MERGE_FLOATS * 4 <= NSLOT * SLOT, "merge area must fit in the ring");
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct DecParams {
    AttnParams p;
    MapAxes k_ax, v_ax;
    int RG;          // row groups per KV head
    int s_lo;        // splits of a group (the first `extra` groups take one more)
    int extra;
    int s_max;       // row stride of the partials (s_lo, or s_lo + 1 when extra > 0)
    int* counters;   // [B * Hkv * RG] 64-bit arrival counters, multiples of the group's S between calls
};

// ldmatrix address of 16-byte unit `u` of row `row` in a 128-byte-swizzled chunk.
__device__ __forceinline__ uint32_t swz(uint32_t chunk, int row, int u) {
    return chunk + (uint32_t)(row * 128 + ((u ^ (row & 7)) << 4));
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// The splits of a group meet here (thread 0 of each CTA; the caller's CTA
// barrier has ordered every thread's partial stores before it): one
// fire-and-forget arrival, then a bounded wait for `target` arrivals.  The
// release (cumulative) publishes this CTA's partials with its arrival; the
// acquire load that sees the target makes every split's partials visible.
// Returns false if the wait ran out (device error flag set).
__device__ __forceinline__ bool split_barrier(unsigned long long* counter, unsigned long long target,
                                              uint64_t limit_ns) {
    asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(counter) : "memory");
    if (ld_acquire_u64(counter) >= target) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        if (ld_acquire_u64(counter) >= target) return true;
        if (globaltimer() - t0 > limit_ns) {
            atomicCAS(&g_sdpa_device_error, 0, (int)kErrWaitSplits);
            return false;
        }
    }
}

// untiled bulk copy global -> this CTA's shared memory, completing on `bar`
// (16-byte aligned addresses, a multiple of 16 bytes)
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

template <int NT>
struct MaskFrag {
    float add[NT][4];
    bool keep[NT][4];
};

template <typename T, int DQK, int DV, int NT, int W, int NSLOT, int SK>
__global__ void __launch_bounds__((W + 1) * 32, 1)
    decode_mma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const DecParams dp) {
    using C = DecodeCfg<DQK, DV, NT, W, NSLOT, SK>;
    constexpr int kNSUB = C::NSUB, kChunk = C::CHUNK;
    const AttnParams& p = dp.p;
    extern __shared__ unsigned char smem_dyn[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    T* Qs = reinterpret_cast<T*>(smem);
    const uint32_t ring = smem_u32(smem + C::OFF_RING);
    float* merge = reinterpret_cast<float*>(smem + C::OFF_RING);   // reused after the key loop
    uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* bar_empty = bar_full + NSLOT;
    int* s_flag = reinterpret_cast<int*>(bar_empty + NSLOT);
    uint64_t* bar_mask = bar_empty + NSLOT + 1;   // the mask values copied up front
    const unsigned char* mpre = smem + C::OFF_MPRE;
    int64_t* row_out = reinterpret_cast<int64_t*>(smem + C::OFF_ROWS);     // [ROWS] output element offset
    int64_t* row_part = row_out + C::ROWS;                                  // [ROWS] partial row index, -1 = none

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g8 = lane >> 2, t4 = lane & 3;   // MMA fragment coordinates

    // ---- which group and split this CTA serves
    int grp, split, S;
    {
        const int c = (int)blockIdx.x;
        const int big = dp.extra * (dp.s_lo + 1);
        if (c < big) {
            grp = c / (dp.s_lo + 1);
            split = c - grp * (dp.s_lo + 1);
            S = dp.s_lo + 1;
        } else {
            const int c2 = c - big;
            grp = dp.extra + c2 / dp.s_lo;
            split = c2 - (c2 / dp.s_lo) * dp.s_lo;
            S = dp.s_lo;
        }
    }
    const int rg = grp % dp.RG;
    const int hkv = (grp / dp.RG) % (int)p.Hkv;
    const int b = grp / (dp.RG * (int)p.Hkv);
    const int64_t G = p.group, R = G * p.Lq;
    const int64_t row0 = (int64_t)rg * C::ROWS;

    // Let the next kernel of the stream start its own launch now; nothing of
    // this grid is read by it before its griddepcontrol.wait.
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    if (tid == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(bar_full + s, 1);
            mbar_init(bar_empty + s, W);   // every consumer warp arrives once per slot
        }
        mbar_init(bar_mask, 1);
        fence_barrier_init();
        tma_prefetch_desc(&tmK);   // kernel parameters: safe before the wait below
        tma_prefetch_desc(&tmV);
    }

    // ---- slots of this split (SK keys each): the keys any row of the CTA can
    // see (all of them; up to the causal horizon; inside the sliding window)
    // are divided among the group's S splits
    int64_t key_first = 0, key_last = p.Lk - 1;
    if (p.mask_kind == 3 || p.mask_kind == 4) {
        int64_t max_i = -1, min_i = p.Lq;   // query indices among this CTA's rows
        for (int r = 0; r < C::ROWS; ++r)
            if (row0 + r < R) {
                max_i = max(max_i, (row0 + r) % p.Lq);
                min_i = min(min_i, (row0 + r) % p.Lq);
            }
        key_last = min(key_last, max_i + p.Lk - p.Lq);   // last key any row sees
        if (p.mask_kind == 4) key_first = max(key_first, min_i + p.Lk - p.Lq - p.window + 1);
    }
    int64_t sl_begin = 0, sl_end = 0;
    if (key_last >= key_first) {
        const int64_t sl_first = key_first / SK, nv = key_last / SK + 1 - sl_first;
        sl_begin = sl_first + nv * split / S;
        sl_end = sl_first + nv * (split + 1) / S;
    }
    const int n_slots = sl_end > sl_begin ? (int)(sl_end - sl_begin) : 0;
    const int n_rows = (int)min((int64_t)C::ROWS, R - row0);   // real query rows of this CTA

    // ---- additive / boolean mask values of this CTA's keys go to shared memory
    // up front, one bulk copy per distinct mask row issued right behind the
    // first K/V slot (ahead of it, it delayed that slot; after several slots,
    // it would queue behind the CTA's K/V stream), when each row's run is
    // contiguous and 16-byte aligned and all of them fit.  Keys [pre_k0,
    // pre_end) are then read from shared memory (the ragged last bytes of the
    // run, if any, from global memory).
    const int64_t esz = p.mask_kind == 1 ? (int64_t)sizeof(T) : 1;
    auto mask_row = [&](int r) -> int64_t {   // element offset of CTA row r's mask row
        const int64_t gr = row0 + r;
        return b * p.sm[0] + (hkv * G + gr / p.Lq) * p.sm[1] + (gr % p.Lq) * p.sm[2];
    };
    int64_t pre_k0 = 0, pre_end = 0;
    int pre_rows = 0;
    uint32_t pre_pitch = 0;
    if ((p.mask_kind == 1 || p.mask_kind == 2) && p.sm[3] == 1 && n_slots > 0) {
        const int64_t k0 = sl_begin * SK, k1 = min(sl_end * SK, p.Lk);
        const uint32_t nb = (uint32_t)(((k1 - k0) * esz) & ~(int64_t)15);
        const int rows = (p.sm[1] == 0 && (p.sm[2] == 0 || p.Lq == 1)) ? 1 : n_rows;
        bool ok = nb > 0 && (int64_t)rows * nb <= C::MPRE;
        for (int r = 0; r < rows && ok; ++r)
            ok = ((reinterpret_cast<uintptr_t>(p.mask) + (uint64_t)((mask_row(r) + k0) * esz)) & 15) == 0;
        if (ok) {
            pre_k0 = k0;
            pre_end = k0 + nb / esz;
            pre_rows = rows;
            pre_pitch = nb;
        }
    }

    // Inputs and the split counters may come from the previous kernel of the
    // stream: wait for it to complete before the first global access.
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    // the group's arrival counter, read now (its round trip is then off the
    // path after the partials): every call on it adds exactly S, and no CTA of
    // this call can have arrived S times yet, so this call's target is the next
    // multiple of S
    unsigned long long* ctr = reinterpret_cast<unsigned long long*>(dp.counters) + grp;
    unsigned long long target = 0;
    if (tid == 0 && S > 1) {
        const unsigned long long c0 = ld_relaxed_u64(ctr);
        target = c0 - c0 % (unsigned long long)S + (unsigned long long)S + (unsigned long long)p.barrier_extra;
    }
    __syncthreads();   // barriers initialised; the producer starts streaming K/V right away

    // per-thread state: rows (nt*8 + 2*t4 + {0,1}); O^T fragments (consumer warps)
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

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && n_slots > 0) {
            int t = 0;
            bool ok = true;
            for (; t < n_slots; ++t) {
                const int slot = t % NSLOT;
                if (C::INFLIGHT < NSLOT && t >= C::INFLIGHT &&
                    !(ok = wait_phase(bar_full + (t - C::INFLIGHT) % NSLOT, ((t - C::INFLIGHT) / NSLOT) & 1,
                                      kErrWaitTmaLoad, p.wait_limit_ns)))
                    break;
                if (t >= NSLOT &&
                    !(ok = wait_phase(bar_empty + slot, ((t / NSLOT) & 1) ^ 1, kErrWaitSlot, p.wait_limit_ns)))
                    break;
                mbar_arrive_expect_tx(bar_full + slot, C::SLOT);
                const int key0 = (int)((sl_begin + t) * SK);
                const uint32_t base = ring + slot * C::SLOT;
                // head dims that are multiples of 64 come as one whole-row box per
                // tensor (one thread issuing one box per chunk cannot keep HBM busy)
                if (DQK % 64 == 0)
                    tma_load_rows(base, &tmK, bar_full + slot, dp.k_ax, key0, hkv, b);
                else
#pragma unroll
                    for (int c = 0; c < C::NBK; ++c)
                        tma_load(base + c * kChunk, &tmK, bar_full + slot, dp.k_ax, c * 64, key0, hkv, b);
                if (DV % 64 == 0)
                    tma_load_rows(base + C::NBK * kChunk, &tmV, bar_full + slot, dp.v_ax, key0, hkv, b);
                else
#pragma unroll
                    for (int c = 0; c < C::NBV; ++c)
                        tma_load(base + (C::NBK + c) * kChunk, &tmV, bar_full + slot, dp.v_ax, c * 64, key0, hkv,
                                 b);
                // the mask values right behind the first slot (pre_rows > 0 implies
                // n_slots > 0, and slot 0 is issued without a wait, so this always runs)
                if (t == 0 && pre_rows > 0) {
                    mbar_arrive_expect_tx(bar_mask, (uint32_t)pre_rows * pre_pitch);
                    for (int r = 0; r < pre_rows; ++r)
                        bulk_load(smem_u32(mpre) + r * pre_pitch,
                                  static_cast<const unsigned char*>(p.mask) + (mask_row(r) + pre_k0) * esz, pre_pitch,
                                  bar_mask);
                }
            }
            if (!ok)   // every issued load must land before shared memory is reused or released
                for (int x = (t > NSLOT ? t - NSLOT : 0); x < t; ++x)
                    wait_phase(bar_full + x % NSLOT, (x / NSLOT) & 1, kErrWaitTmaLoad, p.wait_limit_ns);
        }
        if (lane == 0 && pre_rows > 0) wait_phase(bar_mask, 0, kErrWaitTmaLoad, p.wait_limit_ns);
    } else {
        // ------------------------------------------------------------ consumer warps
        // Q rows of this CTA (zero rows past the group and zero pad columns)
        const T* qg = reinterpret_cast<const T*>(p.q);
        constexpr int CH = C::DQKP / 8;   // 16-byte chunks per padded row
        for (int idx = tid - 32; idx < C::ROWS * CH; idx += C::THREADS - 32) {
            const int r = idx / CH, c = idx % CH;
            const int64_t gr = row0 + r;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (gr < R && c * 8 < DQK) {
                const int64_t h = hkv * G + gr / p.Lq, i = gr % p.Lq;
                val = *reinterpret_cast<const uint4*>(qg + b * p.sq[0] + h * p.sq[1] + i * p.sq[2] + c * 8);
            }
            *reinterpret_cast<uint4*>(Qs + r * C::QS + c * 8) = val;
        }
        for (int r = tid - 32; r < C::ROWS; r += C::THREADS - 32) {   // per-row output / partial offsets
            const int64_t gr = row0 + r;
            if (gr < R) {
                const int64_t h = hkv * G + gr / p.Lq, i = gr % p.Lq;
                row_out[r] = b * p.so[0] + h * p.so[1] + i * p.so[2];
                row_part[r] = ((int64_t)b * p.Hq + h) * p.Lq + i;
            } else {
                row_out[r] = 0;
                row_part[r] = -1;
            }
        }

        const int w = warp - 1;
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
        const float log2e = 1.4426950408889634f;
        // mask values of one 16-key sub-block; s[nt][c] holds key g8 + 8*(c>>1), row 2*t4 + (c&1)
        auto load_mask = [&](int item, MaskFrag<NT>& mf) {
            const int64_t kb = (sl_begin + item / kNSUB) * kNSUB + item % kNSUB;   // global 16-key block
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int rc = c & 1;
                    const int64_t j = kb * 16 + g8 + 8 * (c >> 1);
                    bool keep = row_ok[nt][rc] && j < p.Lk;
                    float add = 0.f;
                    if (keep && (p.mask_kind == 1 || p.mask_kind == 2)) {   // a mask tensor to read
                        if (j >= pre_k0 && j < pre_end) {
                            const int rr = pre_rows == 1 ? 0 : nt * 8 + 2 * t4 + rc;
                            const unsigned char* src = mpre + rr * pre_pitch + (j - pre_k0) * esz;
                            if (p.mask_kind == 1)
                                add = Elem<T>::to_float(*reinterpret_cast<const T*>(src)) * log2e;
                            else
                                keep = *src != 0;
                        } else {
                            const int64_t moff =
                                b * p.sm[0] + row_h[nt][rc] * p.sm[1] + row_i[nt][rc] * p.sm[2] + j * p.sm[3];
                            if (p.mask_kind == 1)
                                add = Elem<T>::to_float(reinterpret_cast<const T*>(p.mask)[moff]) * log2e;
                            else
                                keep = reinterpret_cast<const uint8_t*>(p.mask)[moff] != 0;
                        }
                    } else if (keep && p.mask_kind == 3) {
                        keep = j <= row_i[nt][rc] + p.Lk - p.Lq;
                    } else if (keep && p.mask_kind == 4) {
                        const int64_t own = row_i[nt][rc] + p.Lk - p.Lq;
                        keep = j <= own && j > own - p.window;
                    }
                    mf.add[nt][c] = add;
                    mf.keep[nt][c] = keep;
                }
        };
        // (if the mask copy never lands, the wait sets the error flag and this
        // warp takes no sub-block: the producer's own waits then run out too)
        const bool mask_ok =
            pre_rows == 0 || __all_sync(0xffffffffu, wait_phase(bar_mask, 0, kErrWaitTmaLoad, p.wait_limit_ns));
        const int n_items = mask_ok ? n_slots * kNSUB : 0;
        // one sub-block ahead where the registers allow (NT <= 2); with 32 rows
        // per CTA the values load right before the wait for the sub-block's data
        constexpr bool kAhead = NT <= 2;
        MaskFrag<NT> mnext;
        if (kAhead && w < n_items) load_mask(w, mnext);
        asm volatile("bar.sync 1, %0;\n" ::"n"(W * 32) : "memory");   // Q and row offsets written (consumers)

        const uint32_t q_base = smem_u32(Qs);
        const int mi = lane >> 3;   // which 8x8 matrix this lane addresses in an x4 ldmatrix

        // Every consumer warp waits on every slot in order and releases it
        // (bar_empty counts W arrivals), doing its own sub-blocks of the slot in
        // between.  A parity wait is only unambiguous when the barrier has
        // already completed the phase before the awaited one; a warp that
        // waited only on the slots of its own sub-blocks could run two uses
        // of a ring position ahead (with 7 warps and 3 slots of 2 sub-blocks,
        // a warp's first sub-block already sits in a position's second use)
        // and pass a wait on the wrong phase.
        int item = w;   // this warp's next sub-block: w, w + W, ...
        for (int t = 0; t < n_slots; ++t) {
            const int slot = t % NSLOT;
            if (!__all_sync(0xffffffffu, wait_phase(bar_full + slot, (t / NSLOT) & 1, kErrWaitTmaLoad,
                                                    p.wait_limit_ns)))
                break;
            for (; item < n_items && item < (t + 1) * kNSUB; item += W) {
                const int u = item - t * kNSUB;   // 16-key sub-block u of slot t
                MaskFrag<NT> mcur;
                if (kAhead) {
                    mcur = mnext;
                    // the next sub-block's mask values load while this one computes
                    if (item + W < n_items) load_mask(item + W, mnext);
                } else {
                    load_mask(item, mcur);
                }
                const uint32_t kbase = ring + slot * C::SLOT;
                const uint32_t vbase = kbase + C::NBK * kChunk;
                const int rsub = u * 16;   // first row of this sub-block inside the slot

                // S^T[16 keys][8*NT rows] = K_blk . Q^T
                float s[NT][4], s2[NT][4];   // even / odd K steps: two independent MMA chains
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) s[nt][c] = s2[nt][c] = 0.f;
                {
                    const int arow = rsub + (mi & 1) * 8 + (lane & 7);
                    const uint32_t b_addr = q_base + (uint32_t)(((lane & 7) * C::QS + ((lane >> 3) & 1) * 8) * 2);
#pragma unroll
                    for (int ks = 0; ks < C::DQKP / 16; ++ks) {
                        uint32_t a0, a1, a2, a3;
                        ldmatrix_x4(swz(kbase + (ks >> 2) * kChunk, arow, ((ks & 3) << 1) + (mi >> 1)), a0, a1, a2, a3);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            uint32_t b0, b1;
                            ldmatrix_x2(b_addr + (uint32_t)(nt * 8 * C::QS * 2) + ks * 32, b0, b1);
                            if (ks & 1)
                                mma_16816<T>(s2[nt], a0, a1, a2, a3, b0, b1);
                            else
                                mma_16816<T>(s[nt], a0, a1, a2, a3, b0, b1);
                        }
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int c = 0; c < 4; ++c) s[nt][c] += s2[nt][c];
                }

                // scale, mask, online softmax (log2 domain)
                uint32_t pb[NT][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float bmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float x = mcur.keep[nt][c] ? fmaf(s[nt][c], p.scale_log2, mcur.add[nt][c]) : -INFINITY;
                        s[nt][c] = x;
                        bmax[c & 1] = fmaxf(bmax[c & 1], x);
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
                    const int vrow = rsub + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
                    for (int mt = 0; mt < C::DVP / 16; ++mt) {
                        uint32_t a0, a1, a2, a3;
                        ldmatrix_x4_trans(swz(vbase + (mt >> 2) * kChunk, vrow, ((mt & 3) << 1) + (mi & 1)), a0, a1, a2,
                                          a3);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) mma_16816<T>(o[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_empty + slot);
        }

        // row sums across the 8 lanes that share a row
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
    }

    // ---- merge the consumer warps through shared memory (the ring is drained)
    __syncwarp();   // the producer warp reconverges (its lane 0 ran the TMA loop) before the CTA barrier
    __syncthreads();
    if (warp > 0) {
        float* mw = merge + (size_t)(warp - 1) * C::ROWS * C::MS;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int r0 = nt * 8 + 2 * t4;
#pragma unroll
            for (int mt = 0; mt < C::DVP / 16; ++mt) {
                mw[r0 * C::MS + mt * 16 + g8] = o[mt][nt][0];
                mw[(r0 + 1) * C::MS + mt * 16 + g8] = o[mt][nt][1];
                mw[r0 * C::MS + mt * 16 + g8 + 8] = o[mt][nt][2];
                mw[(r0 + 1) * C::MS + mt * 16 + g8 + 8] = o[mt][nt][3];
            }
            if (g8 == 0) {
                mw[r0 * C::MS + C::DVP] = m_run[nt][0];
                mw[r0 * C::MS + C::DVP + 1] = l_run[nt][0];
                mw[(r0 + 1) * C::MS + C::DVP] = m_run[nt][1];
                mw[(r0 + 1) * C::MS + C::DVP + 1] = l_run[nt][1];
            }
        }
    }
    __syncthreads();

    float* coef = reinterpret_cast<float*>(smem + C::OFF_COEF);   // [ROWS][W + 1]
    for (int r = tid; r < n_rows; r += C::THREADS) {            // per row: weights of the W warps, lse
        float mmax = -INFINITY;
#pragma unroll
        for (int w = 0; w < W; ++w) mmax = fmaxf(mmax, merge[((size_t)w * C::ROWS + r) * C::MS + C::DVP]);
        float f[W], L = 0.f;
#pragma unroll
        for (int w = 0; w < W; ++w) {
            const float* row = merge + ((size_t)w * C::ROWS + r) * C::MS;
            f[w] = (mmax == -INFINITY) ? 0.f : fast_exp2(row[C::DVP] - mmax);   // -inf -> 0
            L += row[C::DVP + 1] * f[w];
        }
        const float inv = (L > 0.f) ? 1.f / L : 0.f;
#pragma unroll
        for (int w = 0; w < W; ++w) coef[r * (W + 1) + w] = f[w] * inv;
        coef[r * (W + 1) + W] = (L > 0.f) ? mmax + log2f(L) : -INFINITY;
    }
    __syncthreads();
    const int SM = dp.s_max;
    for (int idx = tid; idx < n_rows * (DV / 4); idx += C::THREADS) {
        const int r = idx / (DV / 4), c4 = idx % (DV / 4);
        const int64_t row = row_part[r];
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < W; ++w) {
            const float cw = coef[r * (W + 1) + w];
            const float4 v = *reinterpret_cast<const float4*>(merge + ((size_t)w * C::ROWS + r) * C::MS + c4 * 4);
            acc.x = fmaf(cw, v.x, acc.x);
            acc.y = fmaf(cw, v.y, acc.y);
            acc.z = fmaf(cw, v.z, acc.z);
            acc.w = fmaf(cw, v.w, acc.w);
        }
        if (S == 1) {
            uint2 pk;
            pk.x = pack2<T>(acc.x, acc.y);
            pk.y = pack2<T>(acc.z, acc.w);
            *reinterpret_cast<uint2*>(reinterpret_cast<T*>(p.out) + row_out[r] + c4 * 4) = pk;
        } else {
            __stcg(reinterpret_cast<float4*>(p.part_o + (row * SM + split) * DV) + c4, acc);
            if (c4 == 0) __stcg(p.part_lse + row * SM + split, coef[r * (W + 1) + W]);
        }
    }
    if (S == 1) return;

    // ---- the S splits of this group meet (every CTA of the grid is resident:
    // cooperative launch), then each CTA merges its slice of the group's rows x
    // columns.  The CTA barrier orders every thread's partial stores before
    // thread 0's arrival, whose release (cumulative) makes them visible with it.
    __syncthreads();
    if (tid == 0)
        *s_flag = split_barrier(ctr, target, p.wait_limit_ns) ? 1 : 0;
    __syncthreads();
    if (!*s_flag) return;
    // this split's share of the (row, 4-column) items; each thread merges its
    // items online over the splits, 32 splits (their log-sum-exps and
    // partials) in flight per round trip
    const int items = n_rows * (DV / 4);
    const int per = (items + S - 1) / S;
    const int i_end = min(items, (split + 1) * per);
    for (int idx = split * per + tid; idx < i_end; idx += C::THREADS) {
        const int r = idx / (DV / 4), c4 = idx % (DV / 4);
        const int64_t row = row_part[r];
        const float4* po = reinterpret_cast<const float4*>(p.part_o + row * SM * DV) + c4;
        const float* pl = p.part_lse + row * SM;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float mx = -INFINITY, sum = 0.f;
        for (int s0 = 0; s0 < S; s0 += 32) {
            float lse[32];
            float4 v[32];
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const bool in = s0 + u < S;
                lse[u] = in ? __ldcg(pl + s0 + u) : -INFINITY;
                v[u] = in ? __ldcg(po + (int64_t)(s0 + u) * (DV / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            float cm = mx;
#pragma unroll
            for (int u = 0; u < 32; ++u) cm = fmaxf(cm, lse[u]);
            if (cm == -INFINITY) continue;   // no key of these splits is visible
            const float f = (mx == -INFINITY) ? 0.f : fast_exp2(mx - cm);
            acc.x *= f;
            acc.y *= f;
            acc.z *= f;
            acc.w *= f;
            sum *= f;
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const float ws = (lse[u] == -INFINITY) ? 0.f : fast_exp2(lse[u] - cm);
                sum += ws;
                acc.x = fmaf(ws, v[u].x, acc.x);
                acc.y = fmaf(ws, v[u].y, acc.y);
                acc.z = fmaf(ws, v[u].z, acc.z);
                acc.w = fmaf(ws, v[u].w, acc.w);
            }
            mx = cm;
        }
        const float inv = (sum > 0.f) ? 1.f / sum : 0.f;
        uint2 pk;
        pk.x = pack2<T>(acc.x * inv, acc.y * inv);
        pk.y = pack2<T>(acc.z * inv, acc.w * inv);
        *reinterpret_cast<uint2*>(reinterpret_cast<T*>(p.out) + row_out[r] + c4 * 4) = pk;
    }
}

// ---------------------------------------------------------------- host side
struct Shape {
    int nt, w, nslot, sk;
    size_t smem;
};

template <int DQK, int DV, int NT, int W, int NSLOT, int SK>
Shape shape_of() {
    return Shape{NT, W, NSLOT, SK, (size_t)DecodeCfg<DQK, DV, NT, W, NSLOT, SK>::SMEM};
}

// (Dqk, Dv, W, NSLOT, SK) per head dim: about 192 KB of K/V in flight per SM
// in slots of SK keys (32 at Dv >= 256, so that the ring keeps several slots);
// NT in {1, 2, 4} with the O^T accumulators at DVP*NT/4 registers per
// thread (NT = 1 only at Dv = 512, NT <= 2 at Dv = 256).
#define SDPA_DECODE_DIMS(X) \
    X(64, 64, 7, 12, 64)    \
    X(72, 72, 7, 6, 64)     \
    X(80, 80, 7, 6, 64)     \
    X(96, 96, 7, 6, 64)     \
    X(128, 128, 7, 6, 64)   \
    X(192, 128, 7, 5, 64)   \
    X(256, 256, 7, 6, 32)   \
    X(512, 512, 7, 3, 32)

// Head dim 512 has a second variant with 16-key slots (a ring of 6): when the
// CTAs of a call hold more slots than the 3-slot ring, its deeper ring keeps
// more loads queued behind the in-order slot releases (measured at kL = 4096:
// 14.4 us against 16.6); with one or two slots per CTA the 32-key variant is
// faster (10.7 us against 11.9 at kL = 1024).
#define SDPA_DECODE_D512_DEEP 7, 6, 16

constexpr int nt_cap(int dv) { return dv >= 512 ? 1 : (dv >= 256 ? 2 : 4); }
constexpr int nt_fix(int want, int dv) { return want < nt_cap(dv) ? want : nt_cap(dv); }

Shape pick_shape(int64_t Dqk, int64_t Dv, int64_t rows, bool deep = false) {
    if (deep && Dqk == 512 && Dv == 512) return shape_of<512, 512, 1, SDPA_DECODE_D512_DEEP>();
    const int need = (int)((rows + 7) / 8);
    int nt = 1;
    while (nt < need && nt < nt_cap((int)Dv)) nt *= 2;
    switch (Dqk * 1000 + Dv) {
#define SDPA_DECODE_SHAPE(DQ, DVV, W, NS, SK)                                \
    case DQ * 1000 + DVV:                                                    \
        if (nt == 1) return shape_of<DQ, DVV, 1, W, NS, SK>();               \
        if (nt == 2) return shape_of<DQ, DVV, nt_fix(2, DVV), W, NS, SK>();  \
        return shape_of<DQ, DVV, nt_fix(4, DVV), W, NS, SK>();
        SDPA_DECODE_DIMS(SDPA_DECODE_SHAPE)
#undef SDPA_DECODE_SHAPE
        default: return Shape{0, 0, 0, 0, 0};
    }
}

// Splits > 1 meet at a barrier in the workspace, so every CTA of the grid must be
// resident at once: a cooperative launch (which fails rather than run the grid
// in waves).
template <typename T, int DQK, int DV, int NT, int W, int NS, int SK>
cudaError_t launch_one(const DecParams& dp, const CUtensorMap& mk, const CUtensorMap& mv, const LaunchPlan& plan,
                       cudaStream_t stream) {
    auto kern = decode_mma_kernel<T, DQK, DV, NT, W, NS, SK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem_bytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = plan.grid;
    cfg.blockDim = plan.block;
    cfg.dynamicSmemBytes = plan.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    // The grid may be launched while the kernel before it in the stream is
    // still finishing; it waits (griddepcontrol.wait) before its first global
    // read, so stream order holds for every input and for the workspace.
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (plan.splits > 1) {
        attr[n].id = cudaLaunchAttributeCooperative;
        attr[n].val.cooperative = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, mk, mv, dp);
}

template <typename T>
cudaError_t launch_typed(const DecParams& dp, const CUtensorMap& mk, const CUtensorMap& mv, const LaunchPlan& plan,
                         cudaStream_t s) {
    const int nt = plan.aux;
    if (plan.slot_keys == 16 && dp.p.Dqk == 512 && dp.p.Dv == 512)
        return launch_one<T, 512, 512, 1, SDPA_DECODE_D512_DEEP>(dp, mk, mv, plan, s);
    switch (dp.p.Dqk * 1000 + dp.p.Dv) {
#define SDPA_DECODE_LAUNCH(DQ, DVV, W, NS, SK)                                                       \
    case DQ * 1000 + DVV:                                                                            \
        if (nt == 1) return launch_one<T, DQ, DVV, 1, W, NS, SK>(dp, mk, mv, plan, s);               \
        if (nt == 2) return launch_one<T, DQ, DVV, nt_fix(2, DVV), W, NS, SK>(dp, mk, mv, plan, s);  \
        return launch_one<T, DQ, DVV, nt_fix(4, DVV), W, NS, SK>(dp, mk, mv, plan, s);
        SDPA_DECODE_DIMS(SDPA_DECODE_LAUNCH)
#undef SDPA_DECODE_LAUNCH
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool decode_mma_supported(int dtype, int64_t Dqk, int64_t Dv) {
    return (dtype == 1 || dtype == 2) && pick_shape(Dqk, Dv, 8).smem != 0;
}

// Work split.  A (batch, KV head, row group) is a group; its slots of keys are
// split across CTAs, at most one CTA per SM (the kernel takes most of the
// shared memory), every group the same number of splits, each split at most one
// slot short of the others.  More groups than SMs: one CTA per group, in waves.  A head-dim pair this kernel does not cover gets an empty grid,
// which every caller refuses.
LaunchPlan decode_mma_plan(const AttnParams& p, int dtype, const DeviceInfo& dev) {
    (void)dtype;
    LaunchPlan plan{};
    const int64_t rows = (int64_t)p.group * p.Lq;
    Shape sh = pick_shape(p.Dqk, p.Dv, rows);
    if (sh.smem == 0 || rows <= 0 || p.B <= 0 || p.Hkv <= 0) return plan;
    const int base_sk = sh.sk;   // the split count is chosen in slots of this size
    {   // more slots per CTA than the ring holds: the deeper-ring variant (head dim 512)
        const Shape deep = pick_shape(p.Dqk, p.Dv, rows, true);
        const int64_t groups0 = p.B * p.Hkv * ((rows + 8 * sh.nt - 1) / (8 * sh.nt));
        const int64_t splits0 = groups0 < dev.sm_count ? dev.sm_count / groups0 : 1;
        const int64_t slots0 = (p.Lk + sh.sk - 1) / sh.sk;
        if (deep.sk != sh.sk && (slots0 + splits0 - 1) / splits0 > sh.nslot) sh = deep;
    }
    const int64_t RG = (rows + 8 * sh.nt - 1) / (8 * sh.nt);
    // slots of sk keys per group that some row may see (a sliding window
    // covers at most window + Lq - 1 keys, which may straddle one more slot)
    auto visible_slots = [&](int64_t sk) {
        int64_t n = (p.Lk + sk - 1) / sk;
        if (p.mask_kind == 4) {
            const int64_t vis = p.window + p.Lq - 1 < p.Lk ? p.window + p.Lq - 1 : p.Lk;
            const int64_t n_vis = (vis + sk - 1) / sk + 1;
            if (n_vis < n) n = n_vis;
        }
        return n;
    };
    const int64_t nsl = visible_slots(sh.sk);
    // the split count is chosen on the head dim's base slot, so that the
    // deeper ring (half-size slots) changes only how a split streams its keys
    const int64_t nsb = visible_slots(base_sk);
    const int64_t groups = p.B * p.Hkv * RG;
    int64_t lo = 1, extra = 0;
    if (groups < dev.sm_count) {
        // Every group takes the same number of splits: the slowest split sets
        // the launch time, so a group given one split more than the others
        // gains nothing.  The cap is the SMs' share per group, and half the
        // slots (each split adds a partial to merge, and a one-slot split is
        // mostly fixed cost).  Under the cap, the fewest splits that reach the
        // smallest largest share of slots.
        int64_t cap = dev.sm_count / groups;
        if (cap > nsb / 2) cap = nsb / 2 > 1 ? nsb / 2 : 1;
        if (cap > kMaxSplits - 1) cap = kMaxSplits - 1;
        const int64_t m = (nsb + cap - 1) / cap;   // base slots of the largest split
        lo = m > 0 ? (nsb + m - 1) / m : 1;
    }
    // debugging override: the same number of splits for every group; a grid
    // that cannot be resident at once makes the cooperative launch fail
    if (const char* env = getenv("SDPA_DECODE_SPLITS")) {
        const long v = strtol(env, nullptr, 10);
        if (v >= 1) {
            lo = v < kMaxSplits - 1 ? v : kMaxSplits - 1;
            extra = 0;
        }
    }
    const int64_t ctas = groups * lo + extra;
    if (ctas > 0x7fffffff) return plan;
    plan.grid = dim3((unsigned)ctas, 1, 1);
    plan.block = dim3((unsigned)((sh.w + 1) * 32), 1, 1);
    plan.smem_bytes = sh.smem;
    plan.splits = (int)(lo + (extra > 0));
    plan.split_lo = (int)lo;
    plan.split_extra = (int)extra;
    plan.keys_per_split = ((nsl + lo - 1) / lo) * sh.sk;   // the largest split (informational)
    plan.variant = (int)RG;
    plan.aux = sh.nt;
    plan.slot_keys = sh.sk;
    return plan;
}

// ints of counter space (one 64-bit counter per group)
size_t decode_mma_counters(const AttnParams& p, const LaunchPlan& plan) {
    return (size_t)p.B * p.Hkv * plan.variant * 2;
}

cudaError_t decode_mma_launch(const AttnParams& p, int dtype, const LaunchPlan& plan, int* counters,
                              cudaStream_t stream) {
    if (plan.splits > 1 && (plan.splits >= kMaxSplits || counters == nullptr)) return cudaErrorInvalidValue;
    if (plan.split_lo < 1 || plan.splits != plan.split_lo + (plan.split_extra > 0 ? 1 : 0))
        return cudaErrorInvalidValue;
    DecParams dp{};
    dp.p = p;
    dp.RG = plan.variant;
    dp.s_lo = plan.split_lo;
    dp.extra = plan.split_extra;
    dp.s_max = plan.splits;
    dp.counters = counters;
    const int sk = plan.slot_keys;
    CUtensorMap mk, mv;
    const bool ok_k = p.Dqk % 64 == 0
                          ? make_tensor_map_rows(&mk, &dp.k_ax, p.k, dtype, p.Dqk, p.Lk, p.Hkv, p.B, p.sk, sk)
                          : make_tensor_map(&mk, &dp.k_ax, p.k, dtype, p.Dqk, p.Lk, p.Hkv, p.B, p.sk, sk);
    const bool ok_v = p.Dv % 64 == 0
                          ? make_tensor_map_rows(&mv, &dp.v_ax, p.v, dtype, p.Dv, p.Lk, p.Hkv, p.B, p.sv, sk)
                          : make_tensor_map(&mv, &dp.v_ax, p.v, dtype, p.Dv, p.Lk, p.Hkv, p.B, p.sv, sk);
    if (!ok_k || !ok_v) return cudaErrorInvalidValue;
    if (dtype == 1) return launch_typed<__half>(dp, mk, mv, plan, stream);
    if (dtype == 2) return launch_typed<__nv_bfloat16>(dp, mk, mv, plan, stream);
    return cudaErrorInvalidValue;
}

int take_device_error_decode(cudaStream_t stream) {
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
