// api.cu -- the C ABI (include/sdpa.h): validation, path selection, split-K
// workspace, counters and launches.
//
// Shapes come only from the explicit integer arguments and every tensor is
// addressed through its own (b, h, l, d) strides, so no dimension is ever read
// from a tensor's position.  That rules out by construction the failure of
// MLX issue #3585 ("mx.fast.scaled_dot_product_attention produces incorrect
// attention scores"), section "Root cause analysis", where a dispatcher read
// H and L from the wrong axes of a [B, L, H, D] tensor.
//
// Path selection follows MLX issue #3885 ("Metal SDPA: no fused path for
// head_dim=512 ..."), section "Current routing": Lq <= 8 is the decode
// ("vector") path, longer queries the prefill ("full") path.  Unlike the
// routing that issue describes, every supported head dim has a fused kernel on
// both paths, there is no composite fallback that materialises scores, and a
// case no kernel covers is an error status (its request for a queryable
// predicate is sdpa_supported, which calls the very same validation).
// Launch shapes are checked against the device's limits before launching, so
// a launch is never silently dropped (same issue, the missing
// check_kernel_threadgroup_size that produced all-zero outputs).
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <map>
#include <mutex>
#include <set>
#include <string>
#include <tuple>
#include <utility>
#include <vector>

#include "../../include/sdpa.h"
#include "kernels.h"

namespace sdpa {
namespace {

std::atomic<uint64_t> c_calls{0}, c_prefill{0}, c_decode{0}, c_empty{0}, c_rejected{0};
std::atomic<uint64_t> c_tc{0}, c_pffma{0}, c_dmma{0}, c_dffma{0}, c_combine{0}, c_tf32{0};

thread_local std::string t_last_cuda_error;
thread_local int t_last_launches = 0;

// test hooks (sdpa_debug_set)
std::atomic<int64_t> g_dbg_wait_limit_ns{0};    // <= 0: the default limit
std::atomic<int64_t> g_dbg_barrier_extra{0};
std::atomic<int64_t> g_dbg_fail_allocs{0};

bool env_flag(const char* name) {
    const char* v = getenv(name);
    return v && v[0] && strcmp(v, "0") != 0;
}

int elem_size(int dtype) { return dtype == SDPA_F32 ? 4 : 2; }

bool dims_supported(int64_t Dqk, int64_t Dv) {
    switch (Dqk) {
        case 64: case 72: case 80: case 96: case 128: case 256: case 512: return Dv == Dqk;
        case 192: return Dv == 128;
        // absorbed multi-head latent attention on the small MLA fixture of mlxcel
        // issue #1065 ("Why this is a precision problem": kv_lora_rank 32,
        // qk_rope_head_dim 8): keys are [latent | rope] = 40 wide, values are
        // the 32 latent columns (V may alias K through its strides)
        case 40: return Dv == 32;
        default: return false;
    }
}

// Strides of one tensor: d-stride 1, others >= 0 and 16-byte multiples
// (a dimension of extent 1 is exempt from the multiple rule).
int check_tensor_strides(const int64_t* s, int64_t nb, int64_t nh, int64_t nl, int esz) {
    if (s[3] != 1) return SDPA_ERR_UNSUPPORTED_STRIDE;
    const int64_t ext[3] = {nb, nh, nl};
    for (int a = 0; a < 3; ++a) {
        if (s[a] < 0) return SDPA_ERR_UNSUPPORTED_STRIDE;
        if (ext[a] > 1 && ((s[a] * esz) % 16 != 0 || s[a] * esz >= (int64_t(1) << 40)))
            return SDPA_ERR_UNSUPPORTED_STRIDE;
    }
    return SDPA_OK;
}

int validate(int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk, int64_t Dqk, int64_t Dv,
             const int64_t* strides, int mask_kind, const int64_t* mask_strides, int dtype, int* path) {
    *path = SDPA_PATH_NONE;
    if (dtype < SDPA_F32 || dtype > SDPA_BF16) return SDPA_ERR_INVALID_ARG;
    if (mask_kind < SDPA_MASK_NONE || mask_kind > SDPA_MASK_SLIDING) return SDPA_ERR_INVALID_ARG;
    if (B < 0 || Hq < 0 || Hkv <= 0 || Lq < 0 || Lk < 0) return SDPA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return SDPA_ERR_INVALID_ARG;
    if (!dims_supported(Dqk, Dv)) return SDPA_ERR_UNSUPPORTED_DIM;
    if (!strides) return SDPA_ERR_INVALID_ARG;
    // index-range limits: TMA coordinates and grid dimensions are 32-bit
    const int64_t lim = (int64_t(1) << 31) - 1;
    if (Lq > lim || Lk > lim || Hq > 65535 || B > 65535) return SDPA_ERR_TOO_LARGE;
    const int esz = elem_size(dtype);
    int st;
    if ((st = check_tensor_strides(strides + 0, B, Hq, Lq, esz)) != SDPA_OK) return st;
    if ((st = check_tensor_strides(strides + 4, B, Hkv, Lk, esz)) != SDPA_OK) return st;
    if ((st = check_tensor_strides(strides + 8, B, Hkv, Lk, esz)) != SDPA_OK) return st;
    if ((st = check_tensor_strides(strides + 12, B, Hq, Lq, esz)) != SDPA_OK) return st;
    if (mask_kind == SDPA_MASK_ADDITIVE || mask_kind == SDPA_MASK_BOOL) {
        if (!mask_strides) return SDPA_ERR_INVALID_ARG;
        for (int a = 0; a < 4; ++a)
            if (mask_strides[a] < 0) return SDPA_ERR_UNSUPPORTED_STRIDE;
    }
    if (B == 0 || Hq == 0 || Lq == 0) return SDPA_OK;   // empty
    *path = (Lq <= 8) ? SDPA_PATH_DECODE : SDPA_PATH_PREFILL;
    return SDPA_OK;
}

// ---------------------------------------------------------------- device info
std::mutex g_mu;
std::map<int, DeviceInfo> g_devices;

int device_info(DeviceInfo* out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) { t_last_cuda_error = cudaGetErrorString(e); return SDPA_ERR_CUDA; }
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_devices.find(dev);
    if (it == g_devices.end()) {
        DeviceInfo d{};
        d.device = dev;
        if ((e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
                cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) {
            t_last_cuda_error = cudaGetErrorString(e);
            return SDPA_ERR_CUDA;
        }
        it = g_devices.emplace(dev, d).first;
    }
    *out = it->second;
    return SDPA_OK;
}

// ---------------------------------------------------------------- split-K workspace
// Per (device, stream): the split-K partials (contents do not outlive a call)
// and the decode kernel's arrival counters.  A grown partial buffer does not
// free the smaller one (a CUDA graph captured earlier may still point at it):
// retired buffers are kept until sdpa_shutdown.  The counters come in one
// zero-initialised region per launch shape (groups, splits): every call of a
// shape adds exactly its split count to each of its groups' counters, which is
// what the kernel's barrier relies on, so shapes never share counters.
struct Workspace {
    void* ptr = nullptr;
    size_t bytes = 0;
    std::vector<std::pair<void*, size_t>> retired;
    std::map<std::tuple<int64_t, int, int>, std::pair<int*, size_t>> counters;
};
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;

int workspace(int dev, cudaStream_t stream, size_t bytes, void** out) {
    std::lock_guard<std::mutex> lk(g_mu);
    // test hook: behave as if the allocator had no memory, before touching anything
    for (int64_t n = g_dbg_fail_allocs.load(); n > 0;)
        if (g_dbg_fail_allocs.compare_exchange_weak(n, n - 1)) {
            t_last_cuda_error = "workspace allocation failed (forced by SDPA_DEBUG_FAIL_ALLOCS)";
            return SDPA_ERR_NO_MEMORY;
        }
    Workspace& w = g_ws[{dev, stream}];
    if (w.bytes < bytes) {
        const size_t want = bytes + bytes / 4 + 4096;
        void* ptr = nullptr;
        cudaError_t e = cudaMallocAsync(&ptr, want, stream);
        if (e != cudaSuccess) {
            cudaGetLastError();
            t_last_cuda_error = cudaGetErrorString(e);
            return SDPA_ERR_NO_MEMORY;
        }
        if (w.ptr) w.retired.emplace_back(w.ptr, w.bytes);
        w.ptr = ptr;
        w.bytes = want;
    }
    *out = w.ptr;
    return SDPA_OK;
}

int counter_region(int dev, cudaStream_t stream, int64_t ctas, int lo, int extra, size_t n_ints, int** out) {
    std::lock_guard<std::mutex> lk(g_mu);
    Workspace& w = g_ws[{dev, stream}];
    auto& slot = w.counters[std::make_tuple(ctas, lo, extra)];
    if (slot.second < n_ints) {
        int* c = nullptr;
        cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(&c), n_ints * sizeof(int), stream);
        if (e == cudaSuccess) e = cudaMemsetAsync(c, 0, n_ints * sizeof(int), stream);
        if (e != cudaSuccess) {
            cudaGetLastError();
            t_last_cuda_error = cudaGetErrorString(e);
            return SDPA_ERR_NO_MEMORY;
        }
        if (slot.first) w.retired.emplace_back(slot.first, slot.second * sizeof(int));
        slot = {c, n_ints};
    }
    *out = slot.first;
    return SDPA_OK;
}

void log_once(const char* what, const AttnParams& p, int dtype, const LaunchPlan& plan) {
    static std::mutex mu;
    static std::set<std::string> seen;
    char key[512];
    snprintf(key, sizeof key,
             "%s dtype=%d B=%lld Hq=%lld Hkv=%lld Lq=%lld Lk=%lld Dqk=%lld Dv=%lld mask=%d grid=(%u,%u,%u) "
             "block=%u smem=%zu splits=%d",
             what, dtype, (long long)p.B, (long long)p.Hq, (long long)p.Hkv, (long long)p.Lq, (long long)p.Lk,
             (long long)p.Dqk, (long long)p.Dv, p.mask_kind, plan.grid.x, plan.grid.y, plan.grid.z, plan.block.x,
             plan.smem_bytes, plan.splits);
    std::lock_guard<std::mutex> lk(mu);
    if (seen.insert(key).second) fprintf(stderr, "[sdpa] %s\n", key);
}

int check_plan(const LaunchPlan& plan, const DeviceInfo& dev) {
    if (plan.grid.x == 0 || plan.grid.y == 0 || plan.grid.z == 0) return SDPA_ERR_LAUNCH_CONFIG;
    if (plan.grid.y > 65535 || plan.grid.z > 65535) return SDPA_ERR_LAUNCH_CONFIG;
    if (plan.block.x == 0 || plan.block.x > 1024) return SDPA_ERR_LAUNCH_CONFIG;
    if ((int64_t)plan.smem_bytes > dev.max_smem_optin) return SDPA_ERR_LAUNCH_CONFIG;
    return SDPA_OK;
}

int cuda_fail(cudaError_t e) {
    t_last_cuda_error = cudaGetErrorString(e);
    return SDPA_ERR_CUDA;
}

// Zeroes the decode split-barrier counters of this (device, stream)'s
// workspace, on that stream, and waits for it.
int clear_counters(int dev, cudaStream_t stream) {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_ws.find({dev, stream});
    if (it == g_ws.end()) return SDPA_OK;
    cudaError_t e = cudaSuccess;
    for (auto& kv : it->second.counters)
        if (e == cudaSuccess && kv.second.first)
            e = cudaMemsetAsync(kv.second.first, 0, kv.second.second * sizeof(int), stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(e);
    }
    return SDPA_OK;
}

// ---------------------------------------------------------------- opt-in event timing
std::atomic<bool> g_prof_on{false};
std::mutex g_prof_mu;
struct ProfRecord {
    int family;
    cudaEvent_t start, stop;
};
std::vector<ProfRecord> g_prof_records;
std::vector<cudaEvent_t> g_prof_pool;

cudaEvent_t prof_event() {
    if (!g_prof_pool.empty()) {
        cudaEvent_t e = g_prof_pool.back();
        g_prof_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Launches `fn` on `stream`, bracketed by events when timing is enabled.
template <typename F>
cudaError_t timed(int family, cudaStream_t stream, F&& fn) {
    if (!g_prof_on.load(std::memory_order_relaxed)) return fn();
    std::lock_guard<std::mutex> lk(g_prof_mu);
    ProfRecord r{family, prof_event(), prof_event()};
    cudaEventRecord(r.start, stream);
    cudaError_t e = fn();
    cudaEventRecord(r.stop, stream);
    g_prof_records.push_back(r);
    return e;
}

}  // namespace

int record_cuda_error(cudaError_t e) {
    cudaGetLastError();
    return cuda_fail(e);
}

void clear_last_cuda_error() { t_last_cuda_error.clear(); }

}  // namespace sdpa

using namespace sdpa;

extern "C" int sdpa_supported(int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk, int64_t Dqk,
                              int64_t Dv, const int64_t strides[16], int mask_kind,
                              const int64_t mask_strides[4], int dtype, int* path_out) {
    int path = SDPA_PATH_NONE;
    const int st = validate(B, Hq, Hkv, Lq, Lk, Dqk, Dv, strides, mask_kind, mask_strides, dtype, &path);
    if (path_out) *path_out = (st == SDPA_OK) ? path : SDPA_PATH_NONE;
    return st;
}

namespace sdpa {
namespace {

// Both entry points: sdpa_forward (window = 0; the sliding kind is refused,
// since it needs its window) and sdpa_forward_window (mask_kind = SLIDING).
int forward_impl(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t Hq, int64_t Hkv,
                 int64_t Lq, int64_t Lk, int64_t Dqk, int64_t Dv, const int64_t* strides, float scale,
                 int mask_kind, const void* mask, const int64_t* mask_strides, int64_t window, int dtype,
                 void* stream_ptr) {
    c_calls.fetch_add(1, std::memory_order_relaxed);
    t_last_launches = 0;
    t_last_cuda_error.clear();
    auto reject = [](int st) {
        c_rejected.fetch_add(1, std::memory_order_relaxed);
        return st;
    };
    int path = SDPA_PATH_NONE;
    int st = validate(B, Hq, Hkv, Lq, Lk, Dqk, Dv, strides, mask_kind, mask_strides, dtype, &path);
    if (st != SDPA_OK) return reject(st);
    if ((mask_kind == SDPA_MASK_SLIDING) != (window > 0)) return reject(SDPA_ERR_INVALID_ARG);
    if (!std::isfinite(scale)) return reject(SDPA_ERR_INVALID_ARG);
    const bool needs_mask = (mask_kind == SDPA_MASK_ADDITIVE || mask_kind == SDPA_MASK_BOOL);
    if (needs_mask != (mask != nullptr)) return reject(SDPA_ERR_NULL_POINTER);
    if (path == SDPA_PATH_NONE) {
        c_empty.fetch_add(1, std::memory_order_relaxed);
        return SDPA_OK;
    }
    if (!out || (Lk > 0 && (!q || !k || !v))) return reject(SDPA_ERR_NULL_POINTER);
    auto misaligned = [](const void* ptr) { return ptr && (reinterpret_cast<uintptr_t>(ptr) & 15u) != 0; };
    if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(out)) return reject(SDPA_ERR_MISALIGNED);
    if (mask_kind == SDPA_MASK_ADDITIVE && (reinterpret_cast<uintptr_t>(mask) % elem_size(dtype)) != 0)
        return reject(SDPA_ERR_MISALIGNED);

    DeviceInfo dev;
    if ((st = device_info(&dev)) != SDPA_OK) return reject(st);
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_ptr);

    AttnParams p{};
    p.q = q; p.k = k; p.v = v; p.out = out; p.mask = needs_mask ? mask : nullptr;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lq = Lq; p.Lk = Lk; p.Dqk = Dqk; p.Dv = Dv;
    for (int a = 0; a < 4; ++a) {
        p.sq[a] = strides[a]; p.sk[a] = strides[4 + a]; p.sv[a] = strides[8 + a]; p.so[a] = strides[12 + a];
        p.sm[a] = needs_mask ? mask_strides[a] : 0;
    }
    p.scale = scale;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    p.mask_kind = mask_kind;
    p.group = (int)(Hq / Hkv);
    p.splits = 1;
    const int64_t lim = g_dbg_wait_limit_ns.load(std::memory_order_relaxed);
    p.wait_limit_ns = lim > 0 ? (uint64_t)lim : kWaitLimitNs;
    p.barrier_extra = (int)g_dbg_barrier_extra.load(std::memory_order_relaxed);
    p.window = mask_kind == SDPA_MASK_SLIDING ? window : 0;
    p.key_begin = 0;
    if (mask_kind == SDPA_MASK_SLIDING && Lk - Lq - window + 1 > 0) p.key_begin = Lk - Lq - window + 1;

    const bool log = env_flag("SDPA_LOG");
    cudaError_t e;
    if (Lk == 0) {   // no keys: every row is empty -> zeros
        if ((e = timed(SDPA_KERNEL_ZERO_FILL, stream, [&] { return zero_fill_launch(p, dtype, stream); })) !=
            cudaSuccess)
            return cuda_fail(e);
        (path == SDPA_PATH_DECODE ? c_decode : c_prefill).fetch_add(1, std::memory_order_relaxed);
        t_last_launches = 1;
        return SDPA_OK;
    }

    int launches = 0;
    if (path == SDPA_PATH_DECODE) {
        const bool mma = decode_mma_supported(dtype, Dqk, Dv);
        LaunchPlan plan = mma ? decode_mma_plan(p, dtype, dev) : ffma_plan(p, dtype, dev, /*split_keys=*/true);
        if ((st = check_plan(plan, dev)) != SDPA_OK) return reject(st);
        p.splits = plan.splits;
        p.keys_per_split = plan.keys_per_split;
        int* counters = nullptr;
        if (p.splits > 1) {
            const int64_t rows = B * Hq * Lq;
            const size_t o_bytes = (size_t)rows * p.splits * Dv * sizeof(float);
            const size_t l_bytes = (size_t)rows * p.splits * sizeof(float);
            void* ws = nullptr;
            if ((st = workspace(dev.device, stream, o_bytes + l_bytes + 256, &ws)) != SDPA_OK) return reject(st);
            // tensor-core decode: a split barrier; CUDA-core decode: the last split
            // of a tile merges it (both in the one launch)
            const int64_t shape_key = mma ? (int64_t)plan.grid.x : -(int64_t)plan.grid.x * plan.grid.y * plan.grid.z;
            const size_t n_cnt = mma ? decode_mma_counters(p, plan) : ffma_counters(plan);
            if ((st = counter_region(dev.device, stream, shape_key, plan.split_lo, mma ? plan.split_extra : plan.splits,
                                     n_cnt, &counters)) != SDPA_OK)
                return reject(st);
            if (!mma) p.counters = counters;
            p.part_o = reinterpret_cast<float*>(ws);
            p.part_lse = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + ((o_bytes + 255) / 256) * 256);
        }
        if (log) log_once(mma ? "decode_mma" : "decode_ffma", p, dtype, plan);
        e = timed(mma ? SDPA_KERNEL_DECODE_MMA : SDPA_KERNEL_DECODE_FFMA, stream, [&] {
            return mma ? decode_mma_launch(p, dtype, plan, counters, stream) : ffma_launch(p, dtype, plan, stream);
        });
        if (e != cudaSuccess) return cuda_fail(e);
        (mma ? c_dmma : c_dffma).fetch_add(1, std::memory_order_relaxed);
        launches = 1;

        c_decode.fetch_add(1, std::memory_order_relaxed);
    } else {
        // fp16 / bf16 on tcgen05 kind::f16; fp32 on tcgen05 kind::tf32 with the
        // three-term split where its shared memory fits the head dims, else FFMA
        const bool tc = prefill_tc_supported(dtype, Dqk, Dv, p);
        const bool tf = !tc && prefill_tf32_supported(dtype, Dqk, Dv);
        LaunchPlan plan = tc   ? prefill_tc_plan(p, dtype, dev)
                          : tf ? prefill_tf32_plan(p, dev)
                               : ffma_plan(p, dtype, dev, /*split_keys=*/false);
        if ((st = check_plan(plan, dev)) != SDPA_OK) return reject(st);
        p.splits = plan.splits;
        p.keys_per_split = plan.keys_per_split;
        if (log) log_once(tc ? "prefill_tcgen05" : tf ? "prefill_tf32x3" : "prefill_ffma", p, dtype, plan);
        const int fam = tc ? SDPA_KERNEL_PREFILL_TCGEN05 : tf ? SDPA_KERNEL_PREFILL_TF32 : SDPA_KERNEL_PREFILL_FFMA;
        e = timed(fam, stream, [&] {
            return tc ? prefill_tc_launch(p, dtype, plan, stream)
                      : tf ? prefill_tf32_launch(p, plan, stream) : ffma_launch(p, dtype, plan, stream);
        });
        if (e != cudaSuccess) return cuda_fail(e);
        (tc ? c_tc : tf ? c_tf32 : c_pffma).fetch_add(1, std::memory_order_relaxed);
        c_prefill.fetch_add(1, std::memory_order_relaxed);
        launches = 1;
    }
    t_last_launches = launches;
    if (env_flag("SDPA_DEBUG")) {
        if ((e = cudaStreamSynchronize(stream)) != cudaSuccess) return cuda_fail(e);
        int code = 0;
        if (sdpa_check_device_error(stream, &code) != SDPA_OK) return SDPA_ERR_TIMEOUT;
    }
    return SDPA_OK;
}

}  // namespace
}  // namespace sdpa

extern "C" int sdpa_forward(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t Hq,
                            int64_t Hkv, int64_t Lq, int64_t Lk, int64_t Dqk, int64_t Dv,
                            const int64_t strides[16], float scale, int mask_kind, const void* mask,
                            const int64_t mask_strides[4], int dtype, void* stream_ptr) {
    return forward_impl(q, k, v, out, B, Hq, Hkv, Lq, Lk, Dqk, Dv, strides, scale, mask_kind, mask, mask_strides,
                        0, dtype, stream_ptr);
}

extern "C" int sdpa_forward_window(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t Hq,
                                   int64_t Hkv, int64_t Lq, int64_t Lk, int64_t Dqk, int64_t Dv,
                                   const int64_t strides[16], float scale, int64_t window, int dtype,
                                   void* stream_ptr) {
    if (window < 1) {
        c_calls.fetch_add(1, std::memory_order_relaxed);
        c_rejected.fetch_add(1, std::memory_order_relaxed);
        t_last_launches = 0;
        return SDPA_ERR_INVALID_ARG;
    }
    return forward_impl(q, k, v, out, B, Hq, Hkv, Lq, Lk, Dqk, Dv, strides, scale, SDPA_MASK_SLIDING, nullptr,
                        nullptr, window, dtype, stream_ptr);
}

extern "C" const char* sdpa_error_string(int status) {
    switch (status) {
        case SDPA_OK: return "ok";
        case SDPA_ERR_INVALID_ARG: return "invalid argument (size, enum, Hq % Hkv, or scale)";
        case SDPA_ERR_UNSUPPORTED_DIM: return "unsupported head dims (Dqk, Dv)";
        case SDPA_ERR_UNSUPPORTED_STRIDE: return "unsupported stride (d-stride must be 1; others >= 0 and 16-byte multiples)";
        case SDPA_ERR_MISALIGNED: return "misaligned base pointer (16 bytes required)";
        case SDPA_ERR_LAUNCH_CONFIG: return "launch shape exceeds a device limit; nothing launched";
        case SDPA_ERR_CUDA: return "CUDA runtime error";
        case SDPA_ERR_TIMEOUT: return "a bounded in-kernel wait timed out";
        case SDPA_ERR_NO_MEMORY: return "split-K workspace allocation failed";
        case SDPA_ERR_NULL_POINTER: return "null tensor pointer, or mask pointer does not match mask kind";
        case SDPA_ERR_TOO_LARGE: return "a size exceeds the kernels' index range";
        default: return "unknown status";
    }
}

extern "C" const char* sdpa_last_cuda_error(void) { return t_last_cuda_error.c_str(); }

extern "C" void sdpa_get_counters(sdpa_counters* out) {
    if (!out) return;
    out->calls = c_calls.load();
    out->prefill_calls = c_prefill.load();
    out->decode_calls = c_decode.load();
    out->empty_calls = c_empty.load();
    out->rejected_calls = c_rejected.load();
    out->prefill_tcgen05_launches = c_tc.load();
    out->prefill_ffma_launches = c_pffma.load();
    out->decode_mma_launches = c_dmma.load();
    out->decode_ffma_launches = c_dffma.load();
    out->combine_launches = c_combine.load();
    out->prefill_tf32_launches = c_tf32.load();
}

extern "C" void sdpa_reset_counters(void) {
    for (auto* c : {&c_calls, &c_prefill, &c_decode, &c_empty, &c_rejected, &c_tc, &c_pffma, &c_dmma, &c_dffma,
                    &c_combine, &c_tf32})
        c->store(0);
}

extern "C" int sdpa_last_launch_count(void) { return t_last_launches; }

extern "C" int sdpa_check_device_error(void* stream_ptr, int* code_out) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_ptr);
    int code = take_device_error_prefill_tc(stream);
    const int code_d = take_device_error_decode(stream);
    if (code == 0 || code_d < 0) code = code_d;
    const int code_f = take_device_error_tf32(stream);
    if (code == 0 || code_f < 0) code = code_f;
    if (code_out) *code_out = code;
    if (code < 0) return SDPA_ERR_CUDA;
    if (code) {
        // A wait that gave up may have left a split barrier short of its target:
        // start this stream's next decode call from zeroed counters.
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess) clear_counters(dev, stream);
        return SDPA_ERR_TIMEOUT;
    }
    return SDPA_OK;
}

extern "C" int sdpa_debug_set(int knob, int64_t value) {
    switch (knob) {
        case SDPA_DEBUG_WAIT_LIMIT_NS: g_dbg_wait_limit_ns.store(value); return SDPA_OK;
        case SDPA_DEBUG_DECODE_BARRIER_EXTRA:
            if (value < 0 || value > 1024) return SDPA_ERR_INVALID_ARG;
            g_dbg_barrier_extra.store(value);
            return SDPA_OK;
        case SDPA_DEBUG_FAIL_ALLOCS:
            if (value < 0) return SDPA_ERR_INVALID_ARG;
            g_dbg_fail_allocs.store(value);
            return SDPA_OK;
        default: return SDPA_ERR_INVALID_ARG;
    }
}

extern "C" int64_t sdpa_workspace_bytes(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    int64_t total = 0;
    for (auto& kv : g_ws) {
        total += (int64_t)kv.second.bytes;
        for (auto& r : kv.second.retired) total += (int64_t)r.second;
        for (auto& c : kv.second.counters) total += (int64_t)(c.second.second * sizeof(int));
    }
    return total;
}

extern "C" int sdpa_shutdown(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    for (auto& kv : g_ws) {
        int cur = 0;
        cudaGetDevice(&cur);
        cudaSetDevice(kv.first.first);
        // synchronous frees: the owning stream may no longer exist
        if (kv.second.ptr) cudaFree(kv.second.ptr);
        for (auto& r : kv.second.retired) cudaFree(r.first);
        for (auto& c : kv.second.counters)
            if (c.second.first) cudaFree(c.second.first);
        cudaSetDevice(cur);
    }
    g_ws.clear();
    return SDPA_OK;
}

extern "C" int sdpa_abi_version(void) { return 2; }

extern "C" int sdpa_profile_enable(int on) {
    g_prof_on.store(on != 0);
    return SDPA_OK;
}

extern "C" int sdpa_profile_collect(uint64_t launches[SDPA_KERNEL_FAMILIES], double total_ms[SDPA_KERNEL_FAMILIES]) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    int status = SDPA_OK;
    for (auto& r : g_prof_records) {
        float ms = 0.f;
        cudaError_t e = cudaEventSynchronize(r.stop);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.start, r.stop);
        if (e != cudaSuccess) {
            t_last_cuda_error = cudaGetErrorString(e);
            status = SDPA_ERR_CUDA;
        } else if (launches && total_ms && r.family >= 0 && r.family < SDPA_KERNEL_FAMILIES) {
            launches[r.family] += 1;
            total_ms[r.family] += ms;
        }
        g_prof_pool.push_back(r.start);
        g_prof_pool.push_back(r.stop);
    }
    g_prof_records.clear();
    return status;
}
