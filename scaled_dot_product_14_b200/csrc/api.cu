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
std::atomic<uint64_t> c_tc{0}, c_pffma{0}, c_dmma{0}, c_dffma{0}, c_combine{0};

thread_local std::string t_last_cuda_error;
thread_local int t_last_launches = 0;

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
    if (mask_kind < SDPA_MASK_NONE || mask_kind > SDPA_MASK_CAUSAL) return SDPA_ERR_INVALID_ARG;
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
// Per (device, stream): split-K partials (contents do not outlive a call) and
// the decode kernel's per-group counters (zero between calls: zeroed when
// allocated, and every call leaves them zero).
struct Workspace {
    void* ptr = nullptr;
    size_t bytes = 0;
    int* counters = nullptr;
    size_t n_counters = 0;
};
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;

int workspace(int dev, cudaStream_t stream, size_t bytes, size_t n_counters, void** out, int** counters) {
    std::lock_guard<std::mutex> lk(g_mu);
    Workspace& w = g_ws[{dev, stream}];
    if (w.bytes < bytes) {
        if (w.ptr) cudaFreeAsync(w.ptr, stream);
        w.ptr = nullptr;
        w.bytes = 0;
        size_t want = bytes + bytes / 4 + 4096;
        cudaError_t e = cudaMallocAsync(&w.ptr, want, stream);
        if (e != cudaSuccess) {
            cudaGetLastError();
            w.ptr = nullptr;
            t_last_cuda_error = cudaGetErrorString(e);
            return SDPA_ERR_NO_MEMORY;
        }
        w.bytes = want;
    }
    if (w.n_counters < n_counters) {
        if (w.counters) cudaFreeAsync(w.counters, stream);
        w.counters = nullptr;
        w.n_counters = 0;
        const size_t want = n_counters + 1024;
        cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(&w.counters), want * sizeof(int), stream);
        if (e == cudaSuccess) e = cudaMemsetAsync(w.counters, 0, want * sizeof(int), stream);
        if (e != cudaSuccess) {
            cudaGetLastError();
            w.counters = nullptr;
            t_last_cuda_error = cudaGetErrorString(e);
            return SDPA_ERR_NO_MEMORY;
        }
        w.n_counters = want;
    }
    *out = w.ptr;
    *counters = w.counters;
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

extern "C" int sdpa_forward(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t Hq,
                            int64_t Hkv, int64_t Lq, int64_t Lk, int64_t Dqk, int64_t Dv,
                            const int64_t strides[16], float scale, int mask_kind, const void* mask,
                            const int64_t mask_strides[4], int dtype, void* stream_ptr) {
    c_calls.fetch_add(1, std::memory_order_relaxed);
    t_last_launches = 0;
    auto reject = [](int st) {
        c_rejected.fetch_add(1, std::memory_order_relaxed);
        return st;
    };
    int path = SDPA_PATH_NONE;
    int st = validate(B, Hq, Hkv, Lq, Lk, Dqk, Dv, strides, mask_kind, mask_strides, dtype, &path);
    if (st != SDPA_OK) return reject(st);
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
            const size_t n_cnt = mma ? decode_mma_counters(p, plan) : 0;
            void* ws = nullptr;
            if ((st = workspace(dev.device, stream, o_bytes + l_bytes + 256, n_cnt, &ws, &counters)) != SDPA_OK)
                return reject(st);
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
        if (p.splits > 1 && !mma) {   // the mma decode kernel merges its splits itself
            if ((e = timed(SDPA_KERNEL_COMBINE, stream, [&] { return combine_launch(p, dtype, stream); })) !=
                cudaSuccess)
                return cuda_fail(e);
            c_combine.fetch_add(1, std::memory_order_relaxed);
            launches = 2;
        }
        c_decode.fetch_add(1, std::memory_order_relaxed);
    } else {
        const bool tc = prefill_tc_supported(dtype, Dqk, Dv, p);
        LaunchPlan plan = tc ? prefill_tc_plan(p, dtype, dev) : ffma_plan(p, dtype, dev, /*split_keys=*/false);
        if ((st = check_plan(plan, dev)) != SDPA_OK) return reject(st);
        p.splits = plan.splits;
        p.keys_per_split = plan.keys_per_split;
        if (log) log_once(tc ? "prefill_tcgen05" : "prefill_ffma", p, dtype, plan);
        e = timed(tc ? SDPA_KERNEL_PREFILL_TCGEN05 : SDPA_KERNEL_PREFILL_FFMA, stream, [&] {
            return tc ? prefill_tc_launch(p, dtype, plan, stream) : ffma_launch(p, dtype, plan, stream);
        });
        if (e != cudaSuccess) return cuda_fail(e);
        (tc ? c_tc : c_pffma).fetch_add(1, std::memory_order_relaxed);
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
}

extern "C" void sdpa_reset_counters(void) {
    for (auto* c : {&c_calls, &c_prefill, &c_decode, &c_empty, &c_rejected, &c_tc, &c_pffma, &c_dmma, &c_dffma,
                    &c_combine})
        c->store(0);
}

extern "C" int sdpa_last_launch_count(void) { return t_last_launches; }

extern "C" int sdpa_check_device_error(void* stream_ptr, int* code_out) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_ptr);
    int code = take_device_error_prefill_tc(stream);
    const int code_d = take_device_error_decode(stream);
    if (code == 0 || code_d < 0) code = code_d;
    if (code_out) *code_out = code;
    if (code < 0) return SDPA_ERR_CUDA;
    return code ? SDPA_ERR_TIMEOUT : SDPA_OK;
}

extern "C" int sdpa_shutdown(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    for (auto& kv : g_ws) {
        if (kv.second.ptr || kv.second.counters) {
            int cur = 0;
            cudaGetDevice(&cur);
            cudaSetDevice(kv.first.first);
            cudaFree(kv.second.ptr);   // synchronous: the owning stream may no longer exist
            if (kv.second.counters) cudaFree(kv.second.counters);
            cudaSetDevice(cur);
        }
    }
    g_ws.clear();
    return SDPA_OK;
}

extern "C" int sdpa_abi_version(void) { return 1; }

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
