// kernels.h -- internal interface between the host dispatcher (api.cu) and the
// kernel translation units.  Not part of the public ABI (include/sdpa.h is).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sdpa {

// Each kernel translation unit holds its own copy of this flag (internal
// linkage, no relocatable device code).  A bounded wait that gives up writes a
// nonzero code here; the host reads and clears it through the unit's
// take_device_error_* function.
static __device__ int g_sdpa_device_error = 0;

enum DeviceErrorCode : int {
    kErrNone = 0,
    kErrWaitTmaLoad = 1,     // producer-side data never arrived
    kErrWaitMma = 2,         // an MMA completion never arrived
    kErrWaitSoftmax = 3,     // the softmax warps never released a buffer
    kErrWaitSlot = 4,        // a ring slot was never freed
    kErrWaitSplits = 5,      // the splits of a decode group never all arrived
    kErrRingLayout = 6,      // a V block would have read past the ring (never expected)
    kErrWaitSplit = 7,       // the hi / lo split of an fp32 tile never completed
};

// Everything a kernel needs to address one attention problem.  Strides are in
// elements; the dispatcher has already validated them.
struct AttnParams {
    const void* q;
    const void* k;
    const void* v;
    void* out;
    const void* mask;
    int64_t B, Hq, Hkv, Lq, Lk, Dqk, Dv;
    int64_t sq[4], sk[4], sv[4], so[4], sm[4];   // (b, h, l, d); sm = mask (b, h, lq, lk)
    int64_t window;       // sliding-window mask: keys each query sees (0 unless mask_kind == 4)
    int64_t key_begin;    // first key any query may see: max(0, Lk - Lq - window + 1) for a sliding
                          // window, else 0 (split-key plans divide [key_begin, Lk))
    float scale;          // as given
    float scale_log2;     // scale * log2(e): scores are kept in the log2 domain
    int mask_kind;        // sdpa_mask_kind (4 = causal sliding window of `window` keys)
    int group;            // Hq / Hkv
    // split-K (decode path, and the fp32 flash kernel when it splits keys)
    int splits;           // 1 = write the output directly
    int64_t keys_per_split;
    float* part_o;        // [rows][splits][Dv]   rows = B*Hq*Lq, row = (b*Hq + h)*Lq + i
    float* part_lse;      // [rows][splits]       log2-domain log-sum-exp, -inf = no key
    // CUDA-core split-key decode: one 64-bit arrival counter per (row tile, KV
    // head, batch); with it the last split to finish merges the tile in the
    // same launch (nullptr: a separate combine launch merges)
    int* counters;
    // bounded in-kernel waits of the decode kernel give up after this many
    // nanoseconds (the dispatcher passes about 2 s unless a test hook asks for less)
    uint64_t wait_limit_ns;
    // added to the decode split barrier's arrival target; 0 in normal use, > 0
    // only from the test hook that makes the barrier wait run out
    int barrier_extra;
};

// Default limit of every bounded in-kernel wait (about 2 s).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Launch shapes chosen by a plan function; the dispatcher checks them against
// device limits before any launch.
struct LaunchPlan {
    dim3 grid;
    dim3 block;
    size_t smem_bytes;
    int splits;
    int64_t keys_per_split;
    int variant;          // kernel-specific (decode: row groups per KV head)
    int aux;              // kernel-specific (decode: 8-row n-tiles per CTA)
    // decode: the first split_extra groups take split_lo + 1 splits, the others
    // split_lo (splits = the larger, the row stride of the partials)
    int split_lo;
    int split_extra;
    int slot_keys;        // decode: keys per ring slot of the chosen variant
};

struct DeviceInfo {
    int device;
    int sm_count;
    int max_smem_optin;   // bytes per block
    int cc_major, cc_minor;
};

// Which tensor-map dimension carries the sequence, head and batch index
// (the host orders the three by stride); pos 0 means "always coordinate 0".
struct MapAxes {
    int l_pos, h_pos, b_pos;
};

// A 4-D tiled TMA map of a tensor given by (b, h, l, d) element strides `st`:
// dim 0 = d (extent D), then the sequence / head / batch axes ordered by
// stride (an extent-1 or zero-stride axis is pinned to coordinate 0); box =
// 128 bytes of d (64 16-bit or 32 fp32 elements) x box_rows sequence rows;
// 128-byte swizzle; zero fill out of bounds.  tma_map.cu.
bool make_tensor_map(CUtensorMap* map, MapAxes* ax, const void* base, int dtype, int64_t D, int64_t L, int64_t H,
                     int64_t B, const int64_t* st, int box_rows);

// A 5-D map for D a multiple of 64 whose box is box_rows whole rows: dims 64
// elements, sequence, D / 64 chunks (stride 128 bytes), head, batch; shared
// memory gets [chunk][row][64]; 128-byte swizzle; zero fill out of bounds.
// ax->h_pos / b_pos are 3 / 4, or 0 where the axis is pinned.  tma_map.cu.
bool make_tensor_map_rows(CUtensorMap* map, MapAxes* ax, const void* base, int dtype, int64_t D, int64_t L,
                          int64_t H, int64_t B, const int64_t* st, int box_rows);

// ---- fp32 (and generic) flash kernel on CUDA cores: flash_ffma.cu
bool ffma_supported(int dtype, int64_t Dqk, int64_t Dv);
LaunchPlan ffma_plan(const AttnParams& p, int dtype, const DeviceInfo& dev, bool split_keys);
// ints of counter space the split-key plan's in-launch merge needs
size_t ffma_counters(const LaunchPlan& plan);
cudaError_t ffma_launch(const AttnParams& p, int dtype, const LaunchPlan& plan, cudaStream_t stream);

// ---- fp16/bf16 split-K decode (TMA + mma.sync, combine fused): decode_mma.cu
// With plan.splits > 1 the kernel needs p.part_o / p.part_lse and
// decode_mma_counters(p, plan) ints of `counters`: one 64-bit arrival counter
// per group, zero when first used with this launch shape and, between calls,
// a multiple of the group's split count (each call adds exactly that count).
bool decode_mma_supported(int dtype, int64_t Dqk, int64_t Dv);
LaunchPlan decode_mma_plan(const AttnParams& p, int dtype, const DeviceInfo& dev);
size_t decode_mma_counters(const AttnParams& p, const LaunchPlan& plan);
cudaError_t decode_mma_launch(const AttnParams& p, int dtype, const LaunchPlan& plan, int* counters,
                              cudaStream_t stream);

// ---- zero fill of the output of a problem with no keys: combine.cu
cudaError_t zero_fill_launch(const AttnParams& p, int dtype, cudaStream_t stream);

// ---- fp16/bf16 prefill on tcgen05 / TMEM / TMA: prefill_sm100.cu
bool prefill_tc_supported(int dtype, int64_t Dqk, int64_t Dv, const AttnParams& p);
LaunchPlan prefill_tc_plan(const AttnParams& p, int dtype, const DeviceInfo& dev);
cudaError_t prefill_tc_launch(const AttnParams& p, int dtype, const LaunchPlan& plan, cudaStream_t stream);

// api.cu: stores cudaGetErrorString(e) as this thread's sdpa_last_cuda_error
// text, clears the runtime's pending error, and returns SDPA_ERR_CUDA.
int record_cuda_error(cudaError_t e);
// empties this thread's last-error text (every entry point does on entry)
void clear_last_cuda_error();

// ---- fp32 prefill on tcgen05 kind::tf32 with a three-term split: prefill_tf32.cu
bool prefill_tf32_supported(int dtype, int64_t Dqk, int64_t Dv);
LaunchPlan prefill_tf32_plan(const AttnParams& p, const DeviceInfo& dev);
cudaError_t prefill_tf32_launch(const AttnParams& p, const LaunchPlan& plan, cudaStream_t stream);

// Device error flags of each unit (read and clear; synchronous on `stream`).
int take_device_error_prefill_tc(cudaStream_t stream);
int take_device_error_decode(cudaStream_t stream);
int take_device_error_tf32(cudaStream_t stream);

}  // namespace sdpa
