// prefill_sm100.cu -- fp16/bf16 prefill attention on 5th-generation tensor
// cores: TMA tile loads, tcgen05.mma with TMEM accumulators, fused online
// softmax (fp32) with masks, causal tile skipping.
//
// The "full" (qL > 8) path of MLX issue #3885 ("Metal SDPA: no fused path for
// head_dim=512 ..."), section "Current routing", for every head dim of that
// section plus 72 (MLX PR #4330, "Support head dimension 72 in Metal full
// attention").  The pages' kernels tile the head dim on 8x8 simdgroup
// fragments (Steel, TD=9 at d=72) or kU=16 (NAX, which needs d % 32 == 0).
// Here the MMA K step is 16, so d=72 is padded to 80 inside the MMA only: the
// TMA descriptors keep the true extent and the hardware zero-fills columns
// 72..79, costing no memory traffic (that PR's section "Benchmarks" shows why
// head dim 72 must not fall back to the unfused path).
//
// One CTA computes a 128-row query tile of one (batch, query head):
//   warp 0      TMA producer: Q once, then K and V as 16 KB chunks (128 keys
//               x 64 head-dim elements, 128-byte swizzle) into one ring, in
//               the order the MMAs consume them;
//   warp 1      TMEM owner and MMA issuer: S = Q K^T into one of two TMEM
//               S buffers (double-buffered), then O += P V with P read from
//               TMEM (it overwrites its own S buffer) and O kept in TMEM;
//   warps 2..5  softmax: thread t owns query row t (its TMEM lane), scales,
//               masks, keeps the running max / sum in fp32 (log2 domain),
//               writes P as 16-bit pairs back to TMEM, rescales O in TMEM
//               only when its row maximum grew by more than 2^8 (the result
//               is exact either way after the final 1/l), and finally
//               normalises O and stores it through the output strides.
// Head dim 512 (MLX issue #3885, section "Requests": a split-D variant):
// O for 128 rows x 512 fp32 columns would fill all of TMEM, so two CTAs share
// a query tile and each produces 256 of the value columns (S is computed by
// both; the tensor work is 1.5x the algorithmic count for that head dim).
// Every mbarrier wait is bounded (globaltimer); on expiry the kernel records
// an error code, drains its TMA loads and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace sdpa {
namespace {

constexpr int kBM = 128;               // query rows per CTA (UMMA M)
constexpr int kBN = 128;               // keys per tile (UMMA N of S)
constexpr int kChunk = kBN * 128;      // one ring slot: 128 rows x 64 head-dim elements (128-byte swizzle)
constexpr int kThreads = 192;          // 6 warps
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O only when the max grows by > 2^8

__host__ __device__ constexpr int cdiv(int a, int b) { return (a + b - 1) / b; }

// The single-tile kernel's ring order: K(0), then per key tile j K(j+1) (not
// after the last tile) and V(j).  True when, with ring positions mapped to slots
// as (position + shift) % nslot, the NBV chunks of every V(j) occupy consecutive
// slots for every tile count: then one MMA with N = Dv can read all of them
// (consecutive slots are kChunk bytes apart).  The producer's position sequence
// is replayed for up to 2 * nslot + 1 tiles, which covers every residue.
__host__ __device__ constexpr bool v_contiguous(int nbq, int nbv, int nslot, int shift) {
    for (int n = 1; n <= 2 * nslot + 1; ++n) {
        int pos = nbq;   // after K(0)
        for (int j = 0; j < n; ++j) {
            if (j + 1 < n) pos += nbq;   // K(j+1)
            if ((pos + shift) % nslot + nbv > nslot) return false;
            pos += nbv;   // V(j)
        }
    }
    return true;
}

// The smallest slot shift that keeps every V(j) contiguous, or 0 if none does.
__host__ __device__ constexpr int ring_shift(int nbq, int nbv, int nslot) {
    for (int sh = 0; sh < nslot; ++sh)
        if (v_contiguous(nbq, nbv, nslot, sh)) return sh;
    return 0;
}

// DQK: q/k head dim; DVC: value columns this CTA produces (Dv, or Dv/2 when the
// pair of CTAs splits Dv: head dim 512); NSLOT: ring slots; SPLIT: CTAs per query tile.
template <int DQK, int DVC, int NSLOT, int SPLIT>
struct TcCfg {
    static constexpr int NBQ = cdiv(DQK, 64);        // Q / K chunks
    static constexpr int NBV = cdiv(DVC, 64);        // V chunks per CTA
    static constexpr int KSTEPS = cdiv(DQK, 16);     // K steps of S = Q K^T
    static constexpr int DVP = cdiv(DVC, 16) * 16;   // O columns in TMEM
    static constexpr int Q_BYTES = NBQ * kBM * 128;
    static constexpr int OFF_RING = Q_BYTES;
    static constexpr int OFF_BAR = OFF_RING + NSLOT * kChunk;
    static constexpr int NUM_BARS = 1 + 2 * NSLOT + 2 + 2 + 1 + 1;
    static constexpr int SMEM = OFF_BAR + NUM_BARS * 8 + 16 + 1024;   // + TMEM slot + alignment slack
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int O_COL = 2 * kBN;
    static constexpr int SHIFT = ring_shift(NBQ, NBV, NSLOT);   // ring position -> slot offset
    static constexpr bool V_CONTIG = v_contiguous(NBQ, NBV, NSLOT, SHIFT);
    static_assert(O_COL + DVP <= 512, "TMEM budget: two S buffers and O");
    static_assert(NSLOT >= 2, "ring depth");
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct TcParams {
    AttnParams p;
    MapAxes q_ax, k_ax, v_ax;
    int q_tiles;
};

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&o)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]), "=r"(o[4]), "=r"(o[5]), "=r"(o[6]), "=r"(o[7]), "=r"(o[8]),
          "=r"(o[9]), "=r"(o[10]), "=r"(o[11]), "=r"(o[12]), "=r"(o[13]), "=r"(o[14]), "=r"(o[15])
        : "r"(taddr));
}


// Key tiles [t0, t0 + n) of `bn` keys that query rows [r_first, r_last] need:
// causal and sliding-window masks end at the last row's own (bottom-right
// aligned) key; a sliding window starts at the first row's window.  Tiles
// outside that range are never loaded.
template <int MASK>
__device__ __forceinline__ void key_tiles(const AttnParams& p, int64_t r_first, int64_t r_last, int bn, int& t0,
                                          int& n) {
    int64_t k_end = p.Lk, k_begin = 0;
    if (MASK == 3 || MASK == 4) {
        const int64_t last = r_last + p.Lk - p.Lq;
        k_end = last < 0 ? 0 : (last + 1 < p.Lk ? last + 1 : p.Lk);
    }
    if (MASK == 4) {
        const int64_t first = r_first + p.Lk - p.Lq - p.window + 1;
        k_begin = first < 0 ? 0 : first;
    }
    t0 = (int)(k_begin / bn);
    const int64_t t_end = (k_end + bn - 1) / bn;
    n = t_end > t0 ? (int)(t_end - t0) : 0;
}

// ---------------------------------------------------------------- per-row softmax (shared by the kernels)
// Thread t of a softmax warpgroup owns query row t of its 128-row tile, which
// is TMEM lane t.  For a key tile of NK keys it loads that row of S, applies
// scale, masks and the causal / sequence limits, updates the running max (log2
// domain) and sum, and writes P as 16-bit pairs to TMEM: keys [64h, 64h+64) at
// p_taddr + h * 32 (a last block of NK % 64 keys at the end).  P may overwrite
// the S buffer itself (p_taddr = s_taddr) or go to columns of its own.  The
// caller rescales O by `alpha` when `rescale` is set, once the previous P V
// has completed, before the first P block is written.
template <typename T, int MASK, int NK = kBN>
struct RowSoftmax {
    static_assert(NK % 32 == 0 && NK >= 64 && NK <= kBN, "key tile of 64 to 128 keys, a multiple of 32");
    static constexpr int NBLK = (NK + 63) / 64;   // P blocks of 64 keys (the last may hold 32)
    float m_ref, l;
    bool row_ok, pos_scale;
    float sc;
    int64_t Lk, causal_lim, win_lo, mrow, msm3;
    const T* mask_t;
    const uint8_t* mask_b;
    // The row's mask values of the next key tile, loaded as 16-byte vectors
    // while the current tile is processed (additive: NK 16-bit values; boolean:
    // NK bytes).  Used when the row's tile is contiguous (key stride 1),
    // 16-byte aligned and inside the row (not the ragged last tile); otherwise
    // the tile's values are read one by one.
    static constexpr int MV = MASK == 1 ? NK * 2 / 16 : MASK == 2 ? NK / 16 : 1;
    uint4 mvec[MV];
    int64_t mvec_kbase;   // the tile mvec holds, or -1

    __device__ __forceinline__ void init(const AttnParams& p, int64_t b, int64_t hq, int64_t i) {
        m_ref = -INFINITY;
        l = 0.f;
        row_ok = i < p.Lq;
        sc = p.scale_log2;
        pos_scale = sc > 0.f;
        Lk = p.Lk;
        causal_lim = i + p.Lk - p.Lq;
        win_lo = causal_lim - p.window + 1;   // sliding window: first visible key
        mrow = b * p.sm[0] + hq * p.sm[1] + i * p.sm[2];
        msm3 = p.sm[3];
        mask_t = reinterpret_cast<const T*>(p.mask);
        mask_b = reinterpret_cast<const uint8_t*>(p.mask);
        mvec_kbase = -1;
    }

    // Issue the vector loads of the mask tile at kbase (no-op when the tile
    // cannot take them: it is then read element by element in tile()).
    __device__ __forceinline__ void fetch_mask(int64_t kbase) {
        mvec_kbase = -1;
        if (MASK != 1 && MASK != 2) return;
        if (MASK == 1 && NK > 96) return;   // 64 more registers next to 128 scores would spill
        if (!row_ok || msm3 != 1 || kbase < 0 || kbase + NK > Lk) return;
        const void* src = MASK == 1 ? static_cast<const void*>(mask_t + mrow + kbase)
                                    : static_cast<const void*>(mask_b + mrow + kbase);
        if ((reinterpret_cast<uintptr_t>(src) & 15u) != 0) return;
        const uint4* v = reinterpret_cast<const uint4*>(src);
#pragma unroll
        for (int u = 0; u < MV; ++u) mvec[u] = __ldg(v + u);
        mvec_kbase = kbase;
    }

    // NP pairs: p = 2^(x * mul - m) (MUFU), summed into acc, packed into pr.
    template <int NP>
    __device__ __forceinline__ static void exp_pairs(const uint32_t* sr, uint64_t mul2, uint64_t negm2,
                                                     uint64_t (&acc)[4], uint32_t* pr) {
#pragma unroll
        for (int c = 0; c < NP; ++c) {
            const uint64_t x = f2_fma(f2_bits(sr[2 * c], sr[2 * c + 1]), mul2, negm2);
            const uint64_t pp = f2_pack(fast_exp2(f2_lo(x)), fast_exp2(f2_hi(x)));
            acc[c & 3] = f2_add(acc[c & 3], pp);
            pr[c] = pack2<T>(f2_lo(pp), f2_hi(pp));
        }
    }

    // Hooks: loaded() once S is in registers (its TMEM columns may then be
    // overwritten), before_store(h, alpha, rescale) before P block h is written,
    // after_store(h, alpha, rescale) once that store has completed.
    __device__ __forceinline__ void tile(uint32_t s_taddr, int64_t kbase, float& alpha, bool& rescale) {
        auto none = [](int, float, bool) {};
        tile(s_taddr, s_taddr, kbase, alpha, rescale, [] {}, none, none);
    }
    template <typename HalfDone>
    __device__ __forceinline__ void tile(uint32_t s_taddr, int64_t kbase, float& alpha, bool& rescale,
                                         HalfDone&& half_done) {
        auto none = [](int, float, bool) {};
        tile(s_taddr, s_taddr, kbase, alpha, rescale, [] {}, none, half_done);
    }
    template <typename Loaded, typename Before, typename After>
    __device__ __forceinline__ void tile(uint32_t s_taddr, uint32_t p_taddr, int64_t kbase, float& alpha,
                                         bool& rescale, Loaded&& loaded, Before&& before_store,
                                         After&& after_store) {
        const float log2e = 1.4426950408889634f;
        uint32_t sr[NK];
#pragma unroll
        for (int c = 0; c < NK / 32; ++c)
            tmem_ld32(s_taddr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sr + c * 32));
        tmem_wait_ld();
        loaded();

        // keys of this tile that the row may see: [lo, vis) (sequence end, causal
        // limit; a sliding window also hides the keys before its start)
        int64_t lim = Lk - kbase;
        if (MASK == 3 || MASK == 4) lim = min(lim, causal_lim - kbase + 1);
        const int vis = row_ok ? (int)max((int64_t)0, min(lim, (int64_t)NK)) : 0;
        const int lo = (MASK == 4) ? (int)max((int64_t)0, min(win_lo - kbase, (int64_t)NK)) : 0;
        const bool partial = __any_sync(0xffffffffu, vis < NK || lo > 0);   // some key of the tile is hidden
        // values stay raw where possible and are scaled inside the exponent's FFMA
        float mul = sc;
        if (MASK == 1 || MASK == 2) {
            // this tile's values: the vectors requested during the previous tile
            // (or now); they are applied first, and then the next tile's vectors
            // are requested, so one set is live at a time (an additive mask at
            // 128-key tiles is read element by element: its 64 registers next to
            // the 128 scores would spill)
            if (mvec_kbase != kbase) fetch_mask(kbase);
            const bool vec = mvec_kbase == kbase;
            if (__all_sync(0xffffffffu, vec) && !partial && (MASK == 1 || pos_scale)) {
                // every key of the tile visible and the values in registers: no
                // branch per key
                if (MASK == 2) {
                    // boolean: hidden keys become -inf on the raw score; the scale
                    // stays in the exponent's multiplier (positive scale)
                    const uint32_t* w = reinterpret_cast<const uint32_t*>(mvec);
#pragma unroll
                    for (int g = 0; g < NK / 4; ++g) {
                        const uint32_t keepb = __vcmpne4(w[g], 0u);   // 0xff per visible key
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            // byte e's sign replicated over the word (byte-permute selector 8 + e)
                            const uint32_t m = __byte_perm(keepb, 0u, (8u + e) * 0x1111u);
                            sr[4 * g + e] = (sr[4 * g + e] & m) | (0xff800000u & ~m);
                        }
                    }
                } else {
                    // additive: s * scale + m in natural-log units; log2(e) moves
                    // into the exponent's multiplier
                    mul = log2e;
                    const float scn = sc / log2e;
                    const T* mv = reinterpret_cast<const T*>(mvec);
#pragma unroll
                    for (int c = 0; c < NK; ++c)
                        sr[c] = __float_as_uint(fmaf(__uint_as_float(sr[c]), scn, Elem<T>::to_float(mv[c])));
                }
            } else {
                mul = 1.f;
                const T* mt_row = mask_t + mrow + kbase * msm3;
                const uint8_t* mb_row = mask_b + mrow + kbase * msm3;
#pragma unroll
                for (int c = 0; c < NK; ++c) {
                    float x = __uint_as_float(sr[c]) * sc;
                    bool keep = c < vis && c >= lo;
                    if (MASK == 1 && keep) {
                        const T mv = vec ? reinterpret_cast<const T*>(mvec)[c] : mt_row[(int64_t)c * msm3];
                        x += Elem<T>::to_float(mv) * log2e;
                    }
                    if (MASK == 2 && keep) {
                        const uint8_t mb =
                            vec ? reinterpret_cast<const uint8_t*>(mvec)[c] : mb_row[(int64_t)c * msm3];
                        keep = mb != 0;
                    }
                    sr[c] = __float_as_uint(keep ? x : -INFINITY);
                }
            }
            fetch_mask(kbase + NK);
        } else if (!pos_scale) {
            mul = 1.f;
#pragma unroll
            for (int c = 0; c < NK; ++c) {
                const float x = __uint_as_float(sr[c]) * sc;
                sr[c] = __float_as_uint((c < vis && c >= lo) ? x : -INFINITY);
            }
        } else if (partial) {
#pragma unroll
            for (int c = 0; c < NK; ++c) sr[c] = (c < vis && c >= lo) ? sr[c] : __float_as_uint(-INFINITY);
        }
        float mx8[8];   // eight independent chains of three-input maxima
#pragma unroll
        for (int u = 0; u < 8; ++u) mx8[u] = __uint_as_float(sr[u]);
#pragma unroll
        for (int c = 8; c < NK; c += 2)
            mx8[(c >> 1) & 7] = fmax3(mx8[(c >> 1) & 7], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
        const float mloc = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                                 fmaxf(mx8[6], mx8[7])) * mul;   // scaled max
        const float m_new = fmaxf(m_ref, mloc);
        alpha = 1.f;
        rescale = false;
        if (m_new != -INFINITY && (m_ref == -INFINITY || m_new > m_ref + kRescaleThreshold)) {
            rescale = (m_ref != -INFINITY);   // before the first finite max, O holds zeros
            alpha = rescale ? fast_exp2(m_ref - m_new) : 0.f;
            m_ref = m_new;
        }
        const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
        l *= alpha;
        // p = 2^(s * mul - m) on pairs (f32x2); P goes to TMEM 64 keys at a time.
        const uint64_t mul2 = f2_pack(mul, mul), negm2 = f2_pack(-m_use, -m_use);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};   // four independent sum chains
#pragma unroll
        for (int h = 0; h < NBLK; ++h) {
            uint32_t pr[32];
            if (h * 64 + 64 <= NK) {
                exp_pairs<32>(sr + h * 64, mul2, negm2, acc, pr);
                before_store(h, alpha, rescale);
                tmem_st32(p_taddr + h * 32, pr);
            } else {   // a last block of 32 keys
                exp_pairs<16>(sr + h * 64, mul2, negm2, acc, pr);
                before_store(h, alpha, rescale);
                tmem_st16(p_taddr + h * 32, pr);
            }
            tmem_wait_st();
            after_store(h, alpha, rescale);
        }
        const uint64_t acc2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
        l += f2_lo(acc2) + f2_hi(acc2);
    }
};

// O *= f (one row, DVP fp32 columns starting at o_taddr); warp-collective.
template <int DVP>
__device__ __forceinline__ void rescale_o(uint32_t o_taddr, float f) {
#pragma unroll
    for (int c = 0; c < DVP / 16; ++c) {
        uint32_t o[16];
        tmem_ld16(o_taddr + c * 16, o);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * f);
        tmem_st16(o_taddr + c * 16, o);
    }
    tmem_wait_st();
}

// out row = O * inv (zeros when `have` is false), converted and stored; warp-collective.
template <typename T, int DVC, int DVP>
__device__ __forceinline__ void store_o(uint32_t o_taddr, bool have, float inv, T* og, bool row_ok) {
#pragma unroll
    for (int c = 0; c < DVP / 16; ++c) {
        uint32_t o[16];
        if (have) {
            tmem_ld16(o_taddr + c * 16, o);
            tmem_wait_ld();
        } else {
#pragma unroll
            for (int u = 0; u < 16; ++u) o[u] = 0u;
        }
        uint4 w[2];
        uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
        for (int u = 0; u < 8; ++u)
            wp[u] = pack2<T>(__uint_as_float(o[2 * u]) * inv, __uint_as_float(o[2 * u + 1]) * inv);
        if (row_ok) {
            if (c * 16 < DVC) *reinterpret_cast<uint4*>(og + c * 16) = w[0];
            if (c * 16 + 8 < DVC) *reinterpret_cast<uint4*>(og + c * 16 + 8) = w[1];
        }
    }
}

template <typename T, int DQK, int DVC, int NSLOT, int SPLIT, int MASK>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const TcParams tp) {
    using C = TcCfg<DQK, DVC, NSLOT, SPLIT>;
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
    const AttnParams& p = tp.p;

    extern __shared__ unsigned char smem_dyn[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t ring = s_base + C::OFF_RING;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* bar_q = bars;
    uint64_t* bar_full = bars + 1;              // [NSLOT]
    uint64_t* bar_empty = bar_full + NSLOT;     // [NSLOT]
    uint64_t* bar_s_full = bar_empty + NSLOT;   // [2]
    uint64_t* bar_p_full = bar_s_full + 2;      // [2]
    uint64_t* bar_o_done = bar_p_full + 2;
    uint64_t* bar_drain = bar_o_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // causal work is heaviest for the last query tiles: run them first
    const int tile_idx = (int)blockIdx.x / SPLIT;
    const int half = (int)blockIdx.x % SPLIT;
    const int qt = (MASK == 3) ? (tp.q_tiles - 1 - tile_idx) : tile_idx;
    const int hq = blockIdx.y, b = blockIdx.z;
    const int hkv = hq / p.group;
    const int64_t q0 = (int64_t)qt * kBM;
    const int dv0 = half * DVC;   // first value column of this CTA

    // key tiles this query tile needs (causal: up to the diagonal; sliding
    // window: from the first row's window start)
    int t0, n_tiles;
    key_tiles<MASK>(p, q0, q0 + kBM - 1, kBN, t0, n_tiles);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(bar_full + s, 1);
            mbar_init(bar_empty + s, 1);
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
        // Chunks go through the ring in exactly the order the MMA warp consumes
        // them: K(0), then per tile j: K(j+1), V(j).
        if (lane == 0 && n_tiles > 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
            for (int c = 0; c < C::NBQ; ++c) tma_load(s_base + c * kChunk, &tmQ, bar_q, tp.q_ax, c * 64, (int)q0, hq, b);
            int seq = 0;
            bool ok = true;
            auto put = [&](const CUtensorMap* map, const MapAxes& ax, int d0, int j) -> bool {
                const int slot = (seq + C::SHIFT) % NSLOT;
                if (!wait_phase(bar_empty + slot, ((seq / NSLOT) & 1) ^ 1, kErrWaitSlot)) return false;
                mbar_arrive_expect_tx(bar_full + slot, kChunk);
                tma_load(ring + slot * kChunk, map, bar_full + slot, ax, d0, (t0 + j) * kBN, hkv, b);
                ++seq;
                return true;
            };
            for (int c = 0; c < C::NBQ && ok; ++c) ok = put(&tmK, tp.k_ax, c * 64, 0);
            for (int j = 0; j < n_tiles && ok; ++j) {
                if (j + 1 < n_tiles)
                    for (int c = 0; c < C::NBQ && ok; ++c) ok = put(&tmK, tp.k_ax, c * 64, j + 1);
                for (int c = 0; c < C::NBV && ok; ++c) ok = put(&tmV, tp.v_ax, dv0 + c * 64, j);
            }
            if (!ok) {
                // drain: every issued load must land before the CTA's shared memory goes away
                wait_phase(bar_q, 0, kErrWaitTmaLoad);
                for (int x = (seq > NSLOT ? seq - NSLOT : 0); x < seq; ++x)
                    wait_phase(bar_full + (x + C::SHIFT) % NSLOT, (x / NSLOT) & 1, kErrWaitTmaLoad);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_tiles > 0) {
            constexpr uint32_t idS = umma_idesc_f16(kBF16 ? 1 : 0, kBM, kBN, 0, 0);
            int seq = 0;
            bool ok = wait_phase(bar_q, 0, kErrWaitTmaLoad);
            tc_fence_after();
            // The tensor pipe queues few MMAs, so a barrier round trip between two
            // groups of MMAs idles it: the next chunk's barrier is polled before the
            // current chunk's MMAs are issued, and waited on only if it was not ready.
            auto full_ready = [&](int sq) { return mbar_test(bar_full + (sq + C::SHIFT) % NSLOT, (sq / NSLOT) & 1); };
            auto issue_s = [&](int j) -> bool {   // S_j = Q K_j^T into TMEM buffer j & 1
                const uint32_t d = tmem + (uint32_t)((j & 1) * kBN);
                bool ready = full_ready(seq);
#pragma unroll
                for (int c = 0; c < C::NBQ; ++c) {
                    const int slot = (seq + C::SHIFT) % NSLOT;
                    if (!ready && !wait_phase(bar_full + slot, (seq / NSLOT) & 1, kErrWaitTmaLoad)) return false;
                    tc_fence_after();
                    ready = (c + 1 < C::NBQ) ? full_ready(seq + 1) : true;
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        if (c * 4 + k4 >= C::KSTEPS) break;
                        const uint64_t da = umma_desc_sw128(s_base + c * kChunk + k4 * 32, 16, 1024);
                        const uint64_t db = umma_desc_sw128(ring + slot * kChunk + k4 * 32, 16, 1024);
                        umma_ss(d, da, db, idS, (c > 0 || k4 > 0) ? 1u : 0u);
                    }
                    umma_commit(bar_empty + slot);
                    ++seq;
                }
                umma_commit(bar_s_full + (j & 1));
                return true;
            };
            constexpr bool kContig = C::V_CONTIG;
            auto issue_pv = [&](int j, bool ready) -> bool {   // O += P_j V_j, P_j read from TMEM
                const uint32_t a_tmem = tmem + (uint32_t)((j & 1) * kBN);
                if (kContig) {   // one MMA per 16 keys covers every value column
                    const int slot0 = (seq + C::SHIFT) % NSLOT;
                    if (slot0 + C::NBV > NSLOT) {   // excluded by v_contiguous; checked, never read past the ring
                        atomicCAS(&g_sdpa_device_error, 0, kErrRingLayout);
                        return false;
                    }
                    if (!ready)
#pragma unroll
                        for (int c = 0; c < C::NBV; ++c)
                            if (!wait_phase(bar_full + (seq + c + C::SHIFT) % NSLOT, ((seq + c) / NSLOT) & 1, kErrWaitTmaLoad))
                                return false;
                    tc_fence_after();
                    constexpr uint32_t idPV = umma_idesc_f16(kBF16 ? 1 : 0, kBM, C::DVP, 0, 1);
#pragma unroll
                    for (int kk = 0; kk < kBN / 16; ++kk) {
                        const uint64_t db = umma_desc_sw128(ring + slot0 * kChunk + kk * 2048, kChunk, 1024);
                        umma_ts(tmem + C::O_COL, a_tmem + kk * 8, db, idPV, (j > 0 || kk > 0) ? 1u : 0u);
                    }
#pragma unroll
                    for (int c = 0; c < C::NBV; ++c) umma_commit(bar_empty + (seq + c + C::SHIFT) % NSLOT);
                    seq += C::NBV;
                } else {
                    ready = ready || full_ready(seq);
#pragma unroll
                    for (int c = 0; c < C::NBV; ++c) {
                        const int slot = (seq + C::SHIFT) % NSLOT;
                        if (!ready && !wait_phase(bar_full + slot, (seq / NSLOT) & 1, kErrWaitTmaLoad)) return false;
                        tc_fence_after();
                        ready = (c + 1 < C::NBV) ? full_ready(seq + 1) : true;
                        constexpr int kLastN = C::DVP - 64 * (C::NBV - 1);
                        const uint32_t idPV =
                            umma_idesc_f16(kBF16 ? 1 : 0, kBM, (c == C::NBV - 1) ? kLastN : 64, 0, 1);
#pragma unroll
                        for (int kk = 0; kk < kBN / 16; ++kk) {
                            const uint64_t db = umma_desc_sw128(ring + slot * kChunk + kk * 2048, kChunk, 1024);
                            umma_ts(tmem + C::O_COL + c * 64, a_tmem + kk * 8, db, idPV,
                                    (j > 0 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit(bar_empty + slot);
                        ++seq;
                    }
                }
                umma_commit(bar_o_done);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int j = 0; j < n_tiles && ok; ++j) {
                // S_{j+1} goes into the TMEM buffer that P_{j-1} was read from.  The
                // MMAs of one thread execute in order, so it is issued right after
                // P_{j-1} V_{j-1} without waiting for that to complete.
                if (j + 1 < n_tiles && !(ok = issue_s(j + 1))) break;
                // V(j)'s chunks are polled while the softmax of tile j still runs
                bool v_ready = true;
                if (kContig)
#pragma unroll
                    for (int c = 0; c < C::NBV; ++c) v_ready = full_ready(seq + c) && v_ready;
                else
                    v_ready = false;
                if (!(ok = wait_phase(bar_p_full + (j & 1), (j >> 1) & 1, kErrWaitSoftmax))) break;
                tc_fence_after();
                if (!(ok = issue_pv(j, v_ready))) break;
            }
            // every MMA issued by this thread completes before TMEM can be freed
            umma_commit(bar_drain);
            wait_phase(bar_drain, 0, kErrWaitMma);
        }
    } else {
        // ------------------------------------------------------------ softmax / correction / epilogue
        const int quad = warp & 3;   // warps 2,3,4,5 -> TMEM lane quadrants 2,3,0,1
        const int r = quad * 32 + lane;
        const int64_t i = q0 + r;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        RowSoftmax<T, MASK> rs;
        rs.init(p, b, hq, i);
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            const int buf = j & 1;
            ok = __all_sync(0xffffffffu, wait_phase(bar_s_full + buf, (j >> 1) & 1, kErrWaitMma));
            if (!ok) break;
            tc_fence_after();
            float alpha;
            bool rescale;
            rs.tile(tmem + lane_off + buf * kBN, (int64_t)(t0 + j) * kBN, alpha, rescale);
            if (j > 0) {
                ok = __all_sync(0xffffffffu, wait_phase(bar_o_done, (j - 1) & 1, kErrWaitMma));
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, rescale)) rescale_o<C::DVP>(tmem + lane_off + C::O_COL, rescale ? alpha : 1.f);
            }
            tc_fence_before();
            mbar_arrive(bar_p_full + buf);
        }
        // epilogue: O / l -> dtype, stored through the output strides
        if (ok && n_tiles > 0)
            ok = __all_sync(0xffffffffu, wait_phase(bar_o_done, (n_tiles - 1) & 1, kErrWaitMma));
        tc_fence_after();
        T* og = reinterpret_cast<T*>(p.out) + (int64_t)b * p.so[0] + (int64_t)hq * p.so[1] + i * p.so[2] + dv0;
        store_o<T, DVC, C::DVP>(tmem + lane_off + C::O_COL, n_tiles > 0 && ok, rs.l > 0.f ? 1.f / rs.l : 0.f, og,
                                rs.row_ok);
    }

    // teardown: every role has drained its asynchronous work
    __syncwarp();   // producer / MMA warps reconverge (lane 0 ran their loops) before the CTA barrier
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}


// ---------------------------------------------------------------- two query tiles per CTA (ping-pong)
// For Dv <= 128 per CTA: 256 query rows of one (batch, head) as tiles A and B
// that share every K/V chunk.  TMEM: S_A [0,128), S_B [128,256), O_A from 256,
// O_B from 384.  Warpgroup 0 holds the TMA producer (warp 0) and the MMA
// issuer (warp 1); warpgroups 1 and 2 are the softmax of tiles A and B.  The
// two take turns on the tensor core: while one computes its exponentials the
// MMA warp runs the other tile's P V and next S.  MMAs issued by one thread
// execute in order, so S_X(j+1) may be issued right after PV_X(j), which reads
// P_X(j) from the same TMEM columns.  Warpgroup 0 hands registers to the
// softmax warpgroups (setmaxnreg), which hold a 128-wide row of S each.
constexpr int kThreads2 = 384;     // 12 warps
constexpr int kRegsLaunch2 = 168;  // registers per thread at launch (65536 / 384, rounded down to 8)
constexpr int kRegsCtl2 = 88;      // warpgroup 0 after the split
constexpr int kRegsSoftmax2 = 208; // each softmax warpgroup after the split
static_assert(128 * kRegsCtl2 + 256 * kRegsSoftmax2 <= kThreads2 * kRegsLaunch2, "register split exceeds the pool");

template <int DQK, int DVC, int NSLOT>
struct Tc2Cfg {
    static constexpr int NBQ = cdiv(DQK, 64);
    static constexpr int NBV = cdiv(DVC, 64);
    static constexpr int KSTEPS = cdiv(DQK, 16);
    static constexpr int DVP = cdiv(DVC, 16) * 16;
    static constexpr int PER_TILE = NBQ + NBV;        // ring chunks per key tile: K(j) then V(j)
    static constexpr int NSTAGE = NSLOT / PER_TILE;   // key tiles the ring holds
    static constexpr int Q_TILE = NBQ * kBM * 128;
    static constexpr int OFF_RING = 2 * Q_TILE;
    static constexpr int OFF_BAR = OFF_RING + NSLOT * kChunk;
    // q, K full/empty and V full/empty per stage, S full / P full / O done per tile, drain
    static constexpr int NUM_BARS = 1 + 4 * NSTAGE + 2 + 4 + 2 + 1;
    static constexpr int SMEM = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(DVP <= 128, "two O tiles of at most 128 columns");
    static_assert(NSLOT % PER_TILE == 0 && NSTAGE >= 2, "the ring holds whole key tiles, at least two");
    static_assert(SMEM <= 232448, "shared memory budget");
};

template <typename T, int DQK, int DVC, int NSLOT, int MASK>
__global__ void __launch_bounds__(kThreads2, 1)
    prefill_tc2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const TcParams tp) {
    using C = Tc2Cfg<DQK, DVC, NSLOT>;
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
    const AttnParams& p = tp.p;

    extern __shared__ unsigned char smem_dyn[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t ring = s_base + C::OFF_RING;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* bar_q = bars;
    uint64_t* bar_kfull = bars + 1;                   // [NSTAGE]: K(j) landed
    uint64_t* bar_kempty = bar_kfull + C::NSTAGE;     // [NSTAGE]: both tiles' S(j) done with K(j)
    uint64_t* bar_vfull = bar_kempty + C::NSTAGE;     // [NSTAGE]: V(j) landed
    uint64_t* bar_vempty = bar_vfull + C::NSTAGE;     // [NSTAGE]: both tiles' P V(j) done with V(j)
    uint64_t* bar_s_full = bar_vempty + C::NSTAGE;    // [2]: tile A, tile B
    uint64_t* bar_p_full = bar_s_full + 2;            // [2][2]: tile, half of P (keys 0-63, 64-127)
    uint64_t* bar_o_done = bar_p_full + 4;            // [2]
    uint64_t* bar_drain = bar_o_done + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = (MASK == 3) ? (tp.q_tiles - 1 - (int)blockIdx.x) : (int)blockIdx.x;
    const int hq = blockIdx.y, b = blockIdx.z;
    const int hkv = hq / p.group;
    const int64_t q0 = (int64_t)pair * 2 * kBM;   // tile A rows [q0, q0+128), tile B the next 128

    // key tiles the pair needs (tile B sees the last keys under causal masking,
    // tile A the first ones under a sliding window)
    int t0, n_tiles;
    key_tiles<MASK>(p, q0, q0 + 2 * kBM - 1, kBN, t0, n_tiles);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(bar_kfull + s, 1);
            mbar_init(bar_kempty + s, 1);
            mbar_init(bar_vfull + s, 1);
            mbar_init(bar_vempty + s, 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_s_full + s, 1);
            mbar_init(bar_p_full + 2 * s, 128);
            mbar_init(bar_p_full + 2 * s + 1, 128);
            mbar_init(bar_o_done + s, 1);
        }
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
    // Each warpgroup sets its register budget inside its own branch, so that the
    // compiler allots registers per role.
    if (warp < 4) {
        regs_dec<kRegsCtl2>();
        if (warp == 0) {
            // -------------------------------------------------------- TMA producer: K(j), V(j), ...
            // K(j) and V(j) each arrive on one barrier of stage j % NSTAGE; a stage is
            // refilled once both MMA issuers have released it.
            if (lane == 0 && n_tiles > 0) {
                tma_prefetch_desc(&tmQ);
                tma_prefetch_desc(&tmK);
                tma_prefetch_desc(&tmV);
                mbar_arrive_expect_tx(bar_q, 2 * C::Q_TILE);
                for (int t2 = 0; t2 < 2; ++t2)
                    for (int c = 0; c < C::NBQ; ++c)
                        tma_load(s_base + t2 * C::Q_TILE + c * kChunk, &tmQ, bar_q, tp.q_ax, c * 64,
                                 (int)(q0 + t2 * kBM), hq, b);
                bool ok = true;
                int j = 0;
                for (; j < n_tiles && ok; ++j) {
                    const int st = j % C::NSTAGE;
                    const uint32_t par = ((j / C::NSTAGE) & 1) ^ 1;
                    const uint32_t slot0 = ring + (uint32_t)(st * C::PER_TILE) * kChunk;
                    if (!(ok = wait_phase(bar_kempty + st, par, kErrWaitSlot))) break;
                    mbar_arrive_expect_tx(bar_kfull + st, C::NBQ * kChunk);
                    for (int c = 0; c < C::NBQ; ++c)
                        tma_load(slot0 + c * kChunk, &tmK, bar_kfull + st, tp.k_ax, c * 64, (t0 + j) * kBN, hkv,
                                 b);
                    if (!(ok = wait_phase(bar_vempty + st, par, kErrWaitSlot))) {
                        // K(j) is in flight: land it before the drain below
                        wait_phase(bar_kfull + st, (j / C::NSTAGE) & 1, kErrWaitTmaLoad);
                        break;
                    }
                    mbar_arrive_expect_tx(bar_vfull + st, C::NBV * kChunk);
                    for (int c = 0; c < C::NBV; ++c)
                        tma_load(slot0 + (C::NBQ + c) * kChunk, &tmV, bar_vfull + st, tp.v_ax, c * 64, (t0 + j) * kBN,
                                 hkv,
                                 b);
                }
                if (!ok) {
                    // drain: every issued load lands before the CTA's shared memory goes away
                    wait_phase(bar_q, 0, kErrWaitTmaLoad);
                    for (int x = (j > C::NSTAGE ? j - C::NSTAGE : 0); x < j; ++x) {
                        wait_phase(bar_kfull + x % C::NSTAGE, (x / C::NSTAGE) & 1, kErrWaitTmaLoad);
                        wait_phase(bar_vfull + x % C::NSTAGE, (x / C::NSTAGE) & 1, kErrWaitTmaLoad);
                    }
                }
            }
        } else if (warp == 1) {
            // -------------------------------------------------------- MMA issuer
            // Per key tile j: P V and then S(j+1) of tile A, then the same of tile B,
            // so one tile's MMAs run while the other tile's softmax computes.  MMAs
            // issued by one thread execute in order, so S_X(j+1) may overwrite P_X(j)
            // right after P_X(j) V(j) was issued.  The tensor pipe queues few MMAs:
            // the readiness of V(j) and K(j+1) is polled while P(j) is still being
            // computed, so that no barrier round trip sits between the MMAs.
            if (lane == 0 && n_tiles > 0) {
                constexpr uint32_t idS = umma_idesc_f16(kBF16 ? 1 : 0, kBM, kBN, 0, 0);
                constexpr uint32_t idPV = umma_idesc_f16(kBF16 ? 1 : 0, kBM, C::DVP, 0, 1);
                const uint64_t dsc_k = umma_desc_sw128(0, 16, 1024);       // K-major (Q, K)
                const uint64_t dsc_v = umma_desc_sw128(0, kChunk, 1024);   // MN-major (V)
                bool ok = wait_phase(bar_q, 0, kErrWaitTmaLoad);
                auto issue_s = [&](int x, int j) {   // S_X(j) = Q_X K(j)^T
                    const int st = j % C::NSTAGE;
                    const uint32_t kb = ring + (uint32_t)(st * C::PER_TILE) * kChunk;
                    const uint32_t qx = s_base + x * C::Q_TILE;
#pragma unroll
                    for (int k = 0; k < C::KSTEPS; ++k) {
                        const uint32_t off = (uint32_t)((k >> 2) * kChunk + (k & 3) * 32);
                        umma_ss(tmem + (uint32_t)(x * kBN), dsc_k + ((qx + off) >> 4), dsc_k + ((kb + off) >> 4), idS,
                                k > 0 ? 1u : 0u);
                    }
                    if (x == 1) umma_commit(bar_kempty + st);   // tile B is K(j)'s last reader
                    umma_commit(bar_s_full + x);
                };
                // O_X += P_X(j) V(j) over keys [64h, 64h+64), P_X(j) read from TMEM
                auto issue_pv = [&](int x, int j, int h) {
                    const int st = j % C::NSTAGE;
                    const uint32_t v0 = ring + (uint32_t)(st * C::PER_TILE + C::NBQ) * kChunk;
                    const uint32_t a_tmem = tmem + (uint32_t)(x * kBN);
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {   // one MMA per 16 keys covers every value column
                        const int kk = h * 4 + k4;
                        umma_ts(tmem + (uint32_t)(2 * kBN + x * 128), a_tmem + kk * 8, dsc_v + ((v0 + kk * 2048) >> 4),
                                idPV, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                    if (h == 1) {
                        if (x == 1) umma_commit(bar_vempty + st);   // tile B is V(j)'s last reader
                        umma_commit(bar_o_done + x);
                    }
                };
                if (ok) ok = wait_phase(bar_kfull, 0, kErrWaitTmaLoad);
                if (ok) {
                    tc_fence_after();
                    issue_s(0, 0);
                    issue_s(1, 0);
                }
                for (int j = 0; j < n_tiles && ok; ++j) {
                    const int stv = j % C::NSTAGE, stk = (j + 1) % C::NSTAGE;
                    const bool more = j + 1 < n_tiles;
                    // non-blocking polls, answered while tile A's softmax still runs
                    bool v_ok = mbar_test(bar_vfull + stv, (j / C::NSTAGE) & 1);
                    bool k_ok = !more || mbar_test(bar_kfull + stk, ((j + 1) / C::NSTAGE) & 1);
                    for (int x = 0; x < 2 && ok; ++x) {
                        // the first half of P_X(j) goes into the tensor pipe while the
                        // softmax still computes the second
                        if (!(ok = wait_phase(bar_p_full + 2 * x, j & 1, kErrWaitSoftmax))) break;
                        if (!v_ok && !(ok = v_ok = wait_phase(bar_vfull + stv, (j / C::NSTAGE) & 1, kErrWaitTmaLoad)))
                            break;
                        tc_fence_after();
                        issue_pv(x, j, 0);
                        if (!(ok = wait_phase(bar_p_full + 2 * x + 1, j & 1, kErrWaitSoftmax))) break;
                        tc_fence_after();
                        issue_pv(x, j, 1);
                        if (more) {
                            if (!k_ok &&
                                !(ok = k_ok = wait_phase(bar_kfull + stk, ((j + 1) / C::NSTAGE) & 1, kErrWaitTmaLoad)))
                                break;
                            tc_fence_after();
                            issue_s(x, j + 1);
                        }
                    }
                }
                // every MMA issued by this thread completes before TMEM can be freed
                umma_commit(bar_drain);
                wait_phase(bar_drain, 0, kErrWaitMma);
            }
        }
    } else {
        regs_inc<kRegsSoftmax2>();
        // ------------------------------------------------------------ softmax warpgroups (A: warps 4-7, B: 8-11)
        const int x = (warp - 4) >> 2;         // tile of this warpgroup
        const int quad = warp & 3;             // TMEM lane quadrant
        const int r = quad * 32 + lane;
        const int64_t i = q0 + x * kBM + r;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t s_taddr = tmem + lane_off + x * kBN;
        const uint32_t o_taddr = tmem + lane_off + 2 * kBN + x * 128;
        RowSoftmax<T, MASK> rs;
        rs.init(p, b, hq, i);
        bool ok = true;
        for (int j = 0; j < n_tiles && ok; ++j) {
            ok = __all_sync(0xffffffffu, wait_phase(bar_s_full + x, j & 1, kErrWaitMma));
            if (!ok) break;
            tc_fence_after();
            float alpha;
            bool rescale;
            // After each half of P: O is rescaled (before the first half, once
            // P(j-1) V(j-1) has completed) and the MMA issuer is signalled.
            rs.tile(s_taddr, (int64_t)(t0 + j) * kBN, alpha, rescale, [&](int h, float a, bool rs_needed) {
                if (h == 0 && j > 0 && __any_sync(0xffffffffu, rs_needed)) {
                    ok = __all_sync(0xffffffffu, wait_phase(bar_o_done + x, (j - 1) & 1, kErrWaitMma));
                    tc_fence_after();
                    if (ok) rescale_o<C::DVP>(o_taddr, rs_needed ? a : 1.f);
                }
                tc_fence_before();
                mbar_arrive(bar_p_full + 2 * x + h);
            });
        }
        if (ok && n_tiles > 0)
            ok = __all_sync(0xffffffffu, wait_phase(bar_o_done + x, (n_tiles - 1) & 1, kErrWaitMma));
        tc_fence_after();
        T* og = reinterpret_cast<T*>(p.out) + (int64_t)b * p.so[0] + (int64_t)hq * p.so[1] + i * p.so[2];
        store_o<T, DVC, C::DVP>(o_taddr, n_tiles > 0 && ok, rs.l > 0.f ? 1.f / rs.l : 0.f, og, rs.row_ok);
    }

    __syncwarp();   // producer / MMA warps reconverge before the CTA barrier
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- two query tiles, 96-key tiles, P apart (Dv <= 96)
// Same roles and register split as prefill_tc2_kernel, but the key tile is 96
// keys, which leaves TMEM room for everything: S_A [0,96), S_B [96,192),
// O_A [192,288), O_B [288,384), P_A [384,432), P_B [448,496).  P never
// overwrites S, so S_X(j+1) is issued as soon as the softmax of tile X has read
// S_X(j) into registers: it is ready when that softmax finishes, and the softmax
// warpgroups, which the exponentials bind, never wait for the tensor core.  One
// MMA issuer per tile (warps 1 and 2), so the two tiles never wait for each
// other; K(j) and V(j) are released once both tiles' MMAs have read them.
constexpr int kBN3 = 96;                 // keys per tile
constexpr int kChunk3 = kBN3 * 128;      // one ring chunk: 96 rows x 64 head-dim elements (12 KB)

template <int DQK, int DVC, int NSTAGE>
struct Tc3Cfg {
    static constexpr int NBQ = cdiv(DQK, 64);
    static constexpr int NBV = cdiv(DVC, 64);
    static constexpr int KSTEPS = cdiv(DQK, 16);
    static constexpr int DVP = cdiv(DVC, 16) * 16;
    static constexpr int PER_TILE = NBQ + NBV;        // ring chunks per key tile: K(j) then V(j)
    static constexpr int STAGE_BYTES = PER_TILE * kChunk3;
    static constexpr int Q_TILE = NBQ * kBM * 128;    // Q chunks hold 128 rows
    static constexpr int OFF_RING = 2 * Q_TILE;
    static constexpr int OFF_BAR = OFF_RING + NSTAGE * STAGE_BYTES;
    // q; K full/empty and V full/empty per stage; S full, S read, P full, P V done per tile; drain
    static constexpr int NUM_BARS = 1 + 4 * NSTAGE + 2 + 2 + 2 + 2 + 1;
    static constexpr int SMEM = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t S_COL0 = 0, S_COL1 = kBN3, O_COL0 = 2 * kBN3, O_COL1 = 2 * kBN3 + 96;
    static constexpr uint32_t P_COL0 = 384, P_COL1 = 448;   // kBN3 / 2 columns of 16-bit pairs each
    static_assert(DVP <= 96, "O tiles of at most 96 columns");
    static_assert(O_COL1 + 96 <= P_COL0 && P_COL1 + kBN3 / 2 <= TMEM_COLS, "TMEM layout");
    static_assert(NSTAGE >= 2, "the ring holds at least two key tiles");
    static_assert(SMEM <= 232448, "shared memory budget");
};

template <typename T, int DQK, int DVC, int NSTAGE, int MASK>
__global__ void __launch_bounds__(kThreads2, 1)
    prefill_tc3_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const TcParams tp) {
    using C = Tc3Cfg<DQK, DVC, NSTAGE>;
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
    const AttnParams& p = tp.p;

    extern __shared__ unsigned char smem_dyn[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t ring = s_base + C::OFF_RING;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* bar_q = bars;
    uint64_t* bar_kfull = bars + 1;                 // [NSTAGE]: K(j) landed
    uint64_t* bar_kempty = bar_kfull + NSTAGE;      // [NSTAGE]: both tiles' S(j) done with K(j)
    uint64_t* bar_vfull = bar_kempty + NSTAGE;      // [NSTAGE]: V(j) landed
    uint64_t* bar_vempty = bar_vfull + NSTAGE;      // [NSTAGE]: both tiles' P V(j) done with V(j)
    uint64_t* bar_s_full = bar_vempty + NSTAGE;     // [2]: S_X(j) computed
    uint64_t* bar_s_read = bar_s_full + 2;          // [2]: S_X(j) read by the softmax
    uint64_t* bar_p_full = bar_s_read + 2;          // [2]: P_X(j) written
    uint64_t* bar_pv = bar_p_full + 2;              // [2]: P_X(j) V(j) completed
    uint64_t* bar_drain = bar_pv + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = (MASK == 3) ? (tp.q_tiles - 1 - (int)blockIdx.x) : (int)blockIdx.x;
    const int hq = blockIdx.y, b = blockIdx.z;
    const int hkv = hq / p.group;
    const int64_t q0 = (int64_t)pair * 2 * kBM;   // tile A rows [q0, q0+128), tile B the next 128

    // key tiles the pair needs (tile B sees the last keys under causal masking,
    // tile A the first ones under a sliding window)
    int t0, n_tiles;
    key_tiles<MASK>(p, q0, q0 + 2 * kBM - 1, kBN3, t0, n_tiles);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(bar_kfull + s, 1);
            mbar_init(bar_kempty + s, 2);   // one commit per MMA issuer
            mbar_init(bar_vfull + s, 1);
            mbar_init(bar_vempty + s, 2);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_s_full + s, 1);
            mbar_init(bar_s_read + s, 4);   // one arrival per softmax warp
            mbar_init(bar_p_full + s, 128);
            mbar_init(bar_pv + s, 1);
        }
        mbar_init(bar_drain, 2);
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
    if (warp < 4) {
        regs_dec<kRegsCtl2>();
        if (warp == 0) {
            // -------------------------------------------------------- TMA producer: K(j), V(j), ...
            if (lane == 0 && n_tiles > 0) {
                tma_prefetch_desc(&tmQ);
                tma_prefetch_desc(&tmK);
                tma_prefetch_desc(&tmV);
                mbar_arrive_expect_tx(bar_q, 2 * C::Q_TILE);
                for (int t2 = 0; t2 < 2; ++t2)
                    for (int c = 0; c < C::NBQ; ++c)
                        tma_load(s_base + t2 * C::Q_TILE + c * kChunk, &tmQ, bar_q, tp.q_ax, c * 64,
                                 (int)(q0 + t2 * kBM), hq, b);
                bool ok = true;
                int j = 0;
                for (; j < n_tiles && ok; ++j) {
                    const int st = j % NSTAGE;
                    const uint32_t par = ((j / NSTAGE) & 1) ^ 1;
                    const uint32_t stage = ring + (uint32_t)st * C::STAGE_BYTES;
                    if (!(ok = wait_phase(bar_kempty + st, par, kErrWaitSlot))) break;
                    mbar_arrive_expect_tx(bar_kfull + st, C::NBQ * kChunk3);
                    for (int c = 0; c < C::NBQ; ++c)
                        tma_load(stage + c * kChunk3, &tmK, bar_kfull + st, tp.k_ax, c * 64, (t0 + j) * kBN3, hkv,
                                 b);
                    if (!(ok = wait_phase(bar_vempty + st, par, kErrWaitSlot))) {
                        wait_phase(bar_kfull + st, (j / NSTAGE) & 1, kErrWaitTmaLoad);   // K(j) is in flight
                        break;
                    }
                    mbar_arrive_expect_tx(bar_vfull + st, C::NBV * kChunk3);
                    for (int c = 0; c < C::NBV; ++c)
                        tma_load(stage + (C::NBQ + c) * kChunk3, &tmV, bar_vfull + st, tp.v_ax, c * 64,
                                 (t0 + j) * kBN3,
                                 hkv, b);
                }
                if (!ok) {
                    // drain: every issued load lands before the CTA's shared memory goes away
                    wait_phase(bar_q, 0, kErrWaitTmaLoad);
                    for (int x = (j > NSTAGE ? j - NSTAGE : 0); x < j; ++x) {
                        wait_phase(bar_kfull + x % NSTAGE, (x / NSTAGE) & 1, kErrWaitTmaLoad);
                        wait_phase(bar_vfull + x % NSTAGE, (x / NSTAGE) & 1, kErrWaitTmaLoad);
                    }
                }
            }
        } else if (warp <= 2) {
            // -------------------------------------------------------- MMA issuer of tile x
            const int x = warp - 1;
            if (lane == 0 && n_tiles > 0) {
                constexpr uint32_t idS = umma_idesc_f16(kBF16 ? 1 : 0, kBM, kBN3, 0, 0);
                constexpr uint32_t idPV = umma_idesc_f16(kBF16 ? 1 : 0, kBM, C::DVP, 0, 1);
                const uint64_t dsc_k = umma_desc_sw128(0, 16, 1024);        // K-major (Q, K)
                const uint64_t dsc_v = umma_desc_sw128(0, kChunk3, 1024);   // MN-major (V)
                const uint32_t d_s = tmem + (x ? C::S_COL1 : C::S_COL0);
                const uint32_t d_o = tmem + (x ? C::O_COL1 : C::O_COL0);
                const uint32_t a_p = tmem + (x ? C::P_COL1 : C::P_COL0);
                const uint32_t qx = s_base + x * C::Q_TILE;
                auto issue_s = [&](int j) {   // S_X(j) = Q_X K(j)^T
                    const int st = j % NSTAGE;
                    const uint32_t kb = ring + (uint32_t)st * C::STAGE_BYTES;
#pragma unroll
                    for (int k = 0; k < C::KSTEPS; ++k) {
                        const uint32_t qo = (uint32_t)((k >> 2) * kChunk + (k & 3) * 32);
                        const uint32_t ko = (uint32_t)((k >> 2) * kChunk3 + (k & 3) * 32);
                        umma_ss(d_s, dsc_k + ((qx + qo) >> 4), dsc_k + ((kb + ko) >> 4), idS, k > 0 ? 1u : 0u);
                    }
                    umma_commit(bar_kempty + st);
                    umma_commit(bar_s_full + x);
                };
                auto issue_pv = [&](int j) {   // O_X += P_X(j) V(j), one MMA per 16 keys
                    const int st = j % NSTAGE;
                    const uint32_t v0 = ring + (uint32_t)st * C::STAGE_BYTES + C::NBQ * kChunk3;
#pragma unroll
                    for (int kk = 0; kk < kBN3 / 16; ++kk)
                        umma_ts(d_o, a_p + kk * 8, dsc_v + ((v0 + kk * 2048) >> 4), idPV, (j > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(bar_vempty + st);
                    umma_commit(bar_pv + x);
                };
                bool ok = wait_phase(bar_q, 0, kErrWaitTmaLoad) && wait_phase(bar_kfull, 0, kErrWaitTmaLoad);
                if (ok) {
                    tc_fence_after();
                    issue_s(0);
                }
                for (int j = 0; j < n_tiles && ok; ++j) {
                    const int stv = j % NSTAGE, stk = (j + 1) % NSTAGE;
                    const bool more = j + 1 < n_tiles;
                    // non-blocking polls, answered while the softmax still runs
                    const bool v_ok = mbar_test(bar_vfull + stv, (j / NSTAGE) & 1);
                    const bool k_ok = !more || mbar_test(bar_kfull + stk, ((j + 1) / NSTAGE) & 1);
                    if (more) {   // S_X(j+1) as soon as the softmax has read S_X(j)
                        if (!(ok = wait_phase(bar_s_read + x, j & 1, kErrWaitSoftmax))) break;
                        if (!k_ok && !(ok = wait_phase(bar_kfull + stk, ((j + 1) / NSTAGE) & 1, kErrWaitTmaLoad)))
                            break;
                        tc_fence_after();
                        issue_s(j + 1);
                    }
                    if (!(ok = wait_phase(bar_p_full + x, j & 1, kErrWaitSoftmax))) break;
                    if (!v_ok && !(ok = wait_phase(bar_vfull + stv, (j / NSTAGE) & 1, kErrWaitTmaLoad))) break;
                    tc_fence_after();
                    issue_pv(j);
                }
                // every MMA issued by this thread completes before TMEM can be freed
                umma_commit(bar_drain);
                wait_phase(bar_drain, 0, kErrWaitMma);
            }
        }
    } else {
        regs_inc<kRegsSoftmax2>();
        // ------------------------------------------------------------ softmax warpgroups (A: warps 4-7, B: 8-11)
        const int x = (warp - 4) >> 2;
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int64_t i = q0 + x * kBM + r;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t s_taddr = tmem + lane_off + (x ? C::S_COL1 : C::S_COL0);
        const uint32_t p_taddr = tmem + lane_off + (x ? C::P_COL1 : C::P_COL0);
        const uint32_t o_taddr = tmem + lane_off + (x ? C::O_COL1 : C::O_COL0);
        using RS = RowSoftmax<T, MASK, kBN3>;
        RS rs;
        rs.init(p, b, hq, i);
        bool ok = true;
        for (int j = 0; j < n_tiles && ok; ++j) {
            ok = __all_sync(0xffffffffu, wait_phase(bar_s_full + x, j & 1, kErrWaitMma));
            if (!ok) break;
            tc_fence_after();
            float alpha;
            bool rescale;
            auto loaded = [&] {   // S_X(j) is in registers: its columns may take S_X(j+1)
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_s_read + x);
            };
            // Before P(j) is written: P_X(j-1) V(j-1) has completed, which frees the P
            // columns and lets O be rescaled (one wait per key tile, in order).
            auto before_store = [&](int h, float a, bool rs_needed) {
                if (h != 0 || j == 0) return;
                ok = __all_sync(0xffffffffu, wait_phase(bar_pv + x, (j - 1) & 1, kErrWaitMma)) && ok;
                tc_fence_after();
                if (ok && __any_sync(0xffffffffu, rs_needed)) rescale_o<C::DVP>(o_taddr, rs_needed ? a : 1.f);
            };
            auto after_store = [&](int h, float, bool) {
                if (h != RS::NBLK - 1) return;
                tc_fence_before();
                mbar_arrive(bar_p_full + x);
            };
            rs.tile(s_taddr, p_taddr, (int64_t)(t0 + j) * kBN3, alpha, rescale, loaded, before_store, after_store);
        }
        if (ok && n_tiles > 0)
            ok = __all_sync(0xffffffffu, wait_phase(bar_pv + x, (uint32_t)(n_tiles - 1) & 1, kErrWaitMma));
        tc_fence_after();
        T* og = reinterpret_cast<T*>(p.out) + (int64_t)b * p.so[0] + (int64_t)hq * p.so[1] + i * p.so[2];
        store_o<T, DVC, C::DVP>(o_taddr, n_tiles > 0 && ok, rs.l > 0.f ? 1.f / rs.l : 0.f, og, rs.row_ok);
    }

    __syncwarp();   // producer / MMA warps reconverge before the CTA barrier
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side
struct Variant {
    int split, smem, pair;   // pair: two query tiles per CTA (the two-tile kernels)
    int kv_rows;             // keys per K/V box (key tile)
};

template <int DQK, int DVC, int NSLOT, int SPLIT>
Variant variant_of() {
    return Variant{SPLIT, TcCfg<DQK, DVC, NSLOT, SPLIT>::SMEM, 0, kBN};
}
template <int DQK, int DVC, int NSLOT>
Variant variant2_of() {
    return Variant{1, Tc2Cfg<DQK, DVC, NSLOT>::SMEM, 1, kBN};
}
template <int DQK, int DVC, int NSTAGE>
Variant variant3_of() {
    return Variant{1, Tc3Cfg<DQK, DVC, NSTAGE>::SMEM, 1, kBN3};
}

// One query tile per CTA: (Dqk, Dv, Dv per CTA, ring slots, CTAs per query tile).
#define SDPA_TC_VARIANTS(X)             \
    X(192, 128, 128, 10, 1)             \
    X(256, 256, 256, 8, 1)              \
    X(512, 512, 256, 6, 2)
// Two query tiles per CTA, 128-key tiles, P over S: (Dqk, Dv, ring slots), slots a
// multiple of the chunks per key tile.
#define SDPA_TC2_VARIANTS(X)  \
    X(128, 128, 8)
// Two query tiles per CTA, 96-key tiles, P apart: (Dqk, Dv, key tiles in the ring).
#define SDPA_TC3_VARIANTS(X)  \
    X(64, 64, 4)              \
    X(72, 72, 3)              \
    X(80, 80, 3)              \
    X(96, 96, 3)

Variant pick(int64_t Dqk, int64_t Dv) {
    switch (Dqk * 1000 + Dv) {
#define SDPA_TC_PICK(DQ, DVV, DVC, NSL, SP) \
    case DQ * 1000 + DVV: return variant_of<DQ, DVC, NSL, SP>();
        SDPA_TC_VARIANTS(SDPA_TC_PICK)
#undef SDPA_TC_PICK
#define SDPA_TC2_PICK(DQ, DVV, NSL) \
    case DQ * 1000 + DVV: return variant2_of<DQ, DVV, NSL>();
        SDPA_TC2_VARIANTS(SDPA_TC2_PICK)
#undef SDPA_TC2_PICK
#define SDPA_TC3_PICK(DQ, DVV, NST) \
    case DQ * 1000 + DVV: return variant3_of<DQ, DVV, NST>();
        SDPA_TC3_VARIANTS(SDPA_TC3_PICK)
#undef SDPA_TC3_PICK
        default: return Variant{0, 0, 0, 0};
    }
}

template <typename Kern>
cudaError_t launch_kernel(Kern kern, const TcParams& tp, const CUtensorMap& mq, const CUtensorMap& mk,
                          const CUtensorMap& mv, const LaunchPlan& plan, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem_bytes);
    if (e != cudaSuccess) return e;
    kern<<<plan.grid, plan.block, plan.smem_bytes, stream>>>(mq, mk, mv, tp);
    return cudaGetLastError();
}

template <typename T, int DQK, int DVC, int NSLOT, int SPLIT>
cudaError_t launch_one(const TcParams& tp, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const LaunchPlan& plan, cudaStream_t stream) {
    switch (tp.p.mask_kind) {
        case 0: return launch_kernel(prefill_tc_kernel<T, DQK, DVC, NSLOT, SPLIT, 0>, tp, mq, mk, mv, plan, stream);
        case 1: return launch_kernel(prefill_tc_kernel<T, DQK, DVC, NSLOT, SPLIT, 1>, tp, mq, mk, mv, plan, stream);
        case 2: return launch_kernel(prefill_tc_kernel<T, DQK, DVC, NSLOT, SPLIT, 2>, tp, mq, mk, mv, plan, stream);
        case 3: return launch_kernel(prefill_tc_kernel<T, DQK, DVC, NSLOT, SPLIT, 3>, tp, mq, mk, mv, plan, stream);
        case 4: return launch_kernel(prefill_tc_kernel<T, DQK, DVC, NSLOT, SPLIT, 4>, tp, mq, mk, mv, plan, stream);
        default: return cudaErrorInvalidValue;
    }
}

// The pair kernel's register split (setmaxnreg) waits until the increase fits in
// the CTA's launch registers: refuse to launch a build whose register count
// would leave the split waiting.
template <typename Kern>
cudaError_t launch_split_regs(Kern kern, const TcParams& tp, const CUtensorMap& mq, const CUtensorMap& mk,
                              const CUtensorMap& mv, const LaunchPlan& plan, cudaStream_t stream) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if ((int64_t)fa.numRegs * kThreads2 < 128 * kRegsCtl2 + 256 * kRegsSoftmax2 || (int)plan.block.x != kThreads2)
        return cudaErrorInvalidConfiguration;
    return launch_kernel(kern, tp, mq, mk, mv, plan, stream);
}

template <typename T, int DQK, int DVC, int NSLOT>
cudaError_t launch_two(const TcParams& tp, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const LaunchPlan& plan, cudaStream_t stream) {
    switch (tp.p.mask_kind) {
        case 0: return launch_split_regs(prefill_tc2_kernel<T, DQK, DVC, NSLOT, 0>, tp, mq, mk, mv, plan, stream);
        case 1: return launch_split_regs(prefill_tc2_kernel<T, DQK, DVC, NSLOT, 1>, tp, mq, mk, mv, plan, stream);
        case 2: return launch_split_regs(prefill_tc2_kernel<T, DQK, DVC, NSLOT, 2>, tp, mq, mk, mv, plan, stream);
        case 3: return launch_split_regs(prefill_tc2_kernel<T, DQK, DVC, NSLOT, 3>, tp, mq, mk, mv, plan, stream);
        case 4: return launch_split_regs(prefill_tc2_kernel<T, DQK, DVC, NSLOT, 4>, tp, mq, mk, mv, plan, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T, int DQK, int DVC, int NSTAGE>
cudaError_t launch_three(const TcParams& tp, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const LaunchPlan& plan, cudaStream_t stream) {
    switch (tp.p.mask_kind) {
        case 0: return launch_split_regs(prefill_tc3_kernel<T, DQK, DVC, NSTAGE, 0>, tp, mq, mk, mv, plan, stream);
        case 1: return launch_split_regs(prefill_tc3_kernel<T, DQK, DVC, NSTAGE, 1>, tp, mq, mk, mv, plan, stream);
        case 2: return launch_split_regs(prefill_tc3_kernel<T, DQK, DVC, NSTAGE, 2>, tp, mq, mk, mv, plan, stream);
        case 3: return launch_split_regs(prefill_tc3_kernel<T, DQK, DVC, NSTAGE, 3>, tp, mq, mk, mv, plan, stream);
        case 4: return launch_split_regs(prefill_tc3_kernel<T, DQK, DVC, NSTAGE, 4>, tp, mq, mk, mv, plan, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t launch_typed(const TcParams& tp, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const LaunchPlan& plan, cudaStream_t s) {
    switch (tp.p.Dqk * 1000 + tp.p.Dv) {
#define SDPA_TC_LAUNCH(DQ, DVV, DVC, NSL, SP) \
    case DQ * 1000 + DVV: return launch_one<T, DQ, DVC, NSL, SP>(tp, mq, mk, mv, plan, s);
        SDPA_TC_VARIANTS(SDPA_TC_LAUNCH)
#undef SDPA_TC_LAUNCH
#define SDPA_TC2_LAUNCH(DQ, DVV, NSL) \
    case DQ * 1000 + DVV: return launch_two<T, DQ, DVV, NSL>(tp, mq, mk, mv, plan, s);
        SDPA_TC2_VARIANTS(SDPA_TC2_LAUNCH)
#undef SDPA_TC2_LAUNCH
#define SDPA_TC3_LAUNCH(DQ, DVV, NST) \
    case DQ * 1000 + DVV: return launch_three<T, DQ, DVV, NST>(tp, mq, mk, mv, plan, s);
        SDPA_TC3_VARIANTS(SDPA_TC3_LAUNCH)
#undef SDPA_TC3_LAUNCH
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool prefill_tc_supported(int dtype, int64_t Dqk, int64_t Dv, const AttnParams& p) {
    (void)p;
    return (dtype == 1 || dtype == 2) && pick(Dqk, Dv).split != 0;
}

LaunchPlan prefill_tc_plan(const AttnParams& p, int dtype, const DeviceInfo& dev) {
    (void)dtype;
    (void)dev;
    const Variant v = pick(p.Dqk, p.Dv);
    LaunchPlan plan{};
    const int64_t rows_per_cta = v.pair ? 2 * kBM : kBM;
    const int64_t q_tiles = (p.Lq + rows_per_cta - 1) / rows_per_cta;
    plan.grid = dim3((unsigned)(q_tiles * v.split), (unsigned)p.Hq, (unsigned)p.B);
    plan.block = dim3(v.pair ? kThreads2 : kThreads);
    // at least 120 KB: one CTA per SM, so a CTA never waits on another CTA's TMEM
    plan.smem_bytes = (size_t)(v.smem > 120 * 1024 ? v.smem : 120 * 1024);
    plan.splits = 1;
    plan.keys_per_split = p.Lk;
    plan.variant = v.split;
    plan.aux = (int)q_tiles;
    return plan;
}

cudaError_t prefill_tc_launch(const AttnParams& p, int dtype, const LaunchPlan& plan, cudaStream_t stream) {
    TcParams tp{};
    tp.p = p;
    tp.q_tiles = plan.aux;
    CUtensorMap mq, mk, mv;
    const int kv_rows = pick(p.Dqk, p.Dv).kv_rows;
    if (!make_tensor_map(&mq, &tp.q_ax, p.q, dtype, p.Dqk, p.Lq, p.Hq, p.B, p.sq, kBM) ||
        !make_tensor_map(&mk, &tp.k_ax, p.k, dtype, p.Dqk, p.Lk, p.Hkv, p.B, p.sk, kv_rows) ||
        !make_tensor_map(&mv, &tp.v_ax, p.v, dtype, p.Dv, p.Lk, p.Hkv, p.B, p.sv, kv_rows))
        return cudaErrorInvalidValue;
    if (dtype == 2) return launch_typed<__nv_bfloat16>(tp, mq, mk, mv, plan, stream);
    return launch_typed<__half>(tp, mq, mk, mv, plan, stream);
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
