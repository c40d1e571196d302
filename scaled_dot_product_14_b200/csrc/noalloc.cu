// noalloc.cu -- sdpa_forward_noalloc: the fp16/bf16 decode path with its
// split-K scratch in a fixed device array compiled into the library, so a
// call allocates no memory.
//
// Who needs it: callers that cannot call cudaMalloc at the point where they
// run attention.  Examples are a process whose memory manager already
// reserved the whole GPU (a caching allocator or a serving runtime with a
// fixed budget, where a foreign cudaMalloc fails or fragments that budget),
// and latency-critical decode loops that must never pay for cudaMalloc or
// cudaFree (which can synchronise the device).  sdpa_forward allocates its
// split-K workspace on first use per (device, stream); this entry point never
// allocates.
//
// How: the partial outputs and log-sum-exps of the split-K decode kernel live
// in g_noalloc_scratch, a file-scope __device__ array of kNoallocScratchBytes
// that every GPU which loads this library holds until the process exits.  On
// the host that symbol is only a stand-in, not a device address, so the first
// call on each device (with that device current) asks the runtime for the
// array's device address with cudaGetSymbolAddress and caches it; the kernels
// receive that address.  Make that first call before any stream capture.
//
// Every call on a device shares the one array and leaves the last call's
// partials in it.  Its first kCounterBytes hold the decode kernel's per-group
// completion counters, which must be zero when the kernel starts: each call
// clears the ones it uses (cudaMemsetAsync on the call's stream; no
// allocation) before launching.  Partials need no clearing: each split writes
// all of its partials before the last CTA reads them.  Calls that can overlap
// on the GPU (different streams, no ordering between them) race on the array
// and must not be issued.
#include <cuda_runtime.h>
#include <stdint.h>

#include <map>
#include <mutex>

#include "../../include/sdpa.h"
#include "kernels.h"

namespace sdpa {
namespace {

constexpr size_t kNoallocScratchBytes = size_t(4) << 20;   // 4 MiB per device
constexpr size_t kCounterBytes = 64 * 1024;                 // completion counters at the front

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

struct NoallocDevice {
    void* scratch = nullptr;   // device address of g_noalloc_scratch on this device
    int sm_count = 0;
    int max_smem_optin = 0;
};

std::mutex g_na_mu;
std::map<int, NoallocDevice> g_na_devices;

// Set-up, once per device, with that device current.
int noalloc_device(int dev, NoallocDevice* out) {
    std::lock_guard<std::mutex> lk(g_na_mu);
    auto it = g_na_devices.find(dev);
    if (it == g_na_devices.end()) {
        NoallocDevice d;
        cudaError_t e = cudaGetSymbolAddress(&d.scratch, g_noalloc_scratch);
        if (e != cudaSuccess) return record_cuda_error(e);
        if (d.scratch == nullptr) return record_cuda_error(cudaErrorInvalidSymbol);
        if ((e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
                cudaSuccess)
            return record_cuda_error(e);
        it = g_na_devices.emplace(dev, d).first;
    }
    *out = it->second;
    return SDPA_OK;
}

}  // namespace
}  // namespace sdpa

using namespace sdpa;

extern "C" int sdpa_forward_noalloc(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t Hq,
                                    int64_t Hkv, int64_t Lq, int64_t Lk, int64_t Dqk, int64_t Dv,
                                    const int64_t strides[16], float scale, int mask_kind, const void* mask,
                                    const int64_t mask_strides[4], int dtype, void* stream_ptr) {
    clear_last_cuda_error();
    // the same validation as sdpa_forward
    int path = SDPA_PATH_NONE;
    int st = sdpa_supported(B, Hq, Hkv, Lq, Lk, Dqk, Dv, strides, mask_kind, mask_strides, dtype, &path);
    if (st != SDPA_OK) return st;
    if (!(scale == scale) || scale > 3.4e38f || scale < -3.4e38f) return SDPA_ERR_INVALID_ARG;
    const bool needs_mask = (mask_kind == SDPA_MASK_ADDITIVE || mask_kind == SDPA_MASK_BOOL);
    if (needs_mask != (mask != nullptr)) return SDPA_ERR_NULL_POINTER;
    if (mask_kind == SDPA_MASK_SLIDING) return SDPA_ERR_INVALID_ARG;   // needs a window: sdpa_forward_window
    if (path == SDPA_PATH_NONE) return SDPA_OK;
    // this entry point covers the fp16 / bf16 decode path of the tensor-core
    // decode kernel only (not the absorbed-MLA dims, which run on CUDA cores);
    // everything here is checked before the first CUDA call
    if (path != SDPA_PATH_DECODE || (dtype != SDPA_F16 && dtype != SDPA_BF16)) return SDPA_ERR_INVALID_ARG;
    if (!decode_mma_supported(dtype, Dqk, Dv)) return SDPA_ERR_INVALID_ARG;
    if (!out || (Lk > 0 && (!q || !k || !v))) return SDPA_ERR_NULL_POINTER;
    auto misaligned = [](const void* ptr) { return ptr && (reinterpret_cast<uintptr_t>(ptr) & 15u) != 0; };
    if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(out)) return SDPA_ERR_MISALIGNED;
    if (mask_kind == SDPA_MASK_ADDITIVE && (reinterpret_cast<uintptr_t>(mask) & 1u) != 0) return SDPA_ERR_MISALIGNED;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return record_cuda_error(e);
    NoallocDevice nd;
    if ((st = noalloc_device(dev, &nd)) != SDPA_OK) return st;
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
    p.wait_limit_ns = kWaitLimitNs;
    p.barrier_extra = 0;
    p.window = 0;
    p.key_begin = 0;
    if (Lk == 0) {
        if ((e = zero_fill_launch(p, dtype, stream)) != cudaSuccess) return record_cuda_error(e);
        return SDPA_OK;
    }

    DeviceInfo di{};
    di.device = dev;
    di.sm_count = nd.sm_count;
    di.max_smem_optin = nd.max_smem_optin;
    const LaunchPlan plan = decode_mma_plan(p, dtype, di);
    if (plan.grid.x == 0 || plan.grid.y == 0 || plan.grid.z == 0 || plan.grid.y > 65535 || plan.grid.z > 65535 ||
        (int64_t)plan.smem_bytes > nd.max_smem_optin)
        return SDPA_ERR_LAUNCH_CONFIG;
    p.splits = plan.splits;
    p.keys_per_split = plan.keys_per_split;
    int* counters = nullptr;
    if (p.splits > 1) {
        const int64_t rows = B * Hq * Lq;
        const size_t o_bytes = ((size_t)rows * p.splits * Dv * sizeof(float) + 255) / 256 * 256;
        const size_t l_bytes = (size_t)rows * p.splits * sizeof(float);
        const size_t c_bytes = decode_mma_counters(p, plan) * sizeof(int);
        if (c_bytes > kCounterBytes || kCounterBytes + o_bytes + l_bytes > kNoallocScratchBytes)
            return SDPA_ERR_TOO_LARGE;   // the scratch array would overflow
        char* base = reinterpret_cast<char*>(nd.scratch);
        counters = reinterpret_cast<int*>(base);
        p.part_o = reinterpret_cast<float*>(base + kCounterBytes);
        p.part_lse = reinterpret_cast<float*>(base + kCounterBytes + o_bytes);
        if ((e = cudaMemsetAsync(counters, 0, c_bytes, stream)) != cudaSuccess) return record_cuda_error(e);
    }
    if ((e = decode_mma_launch(p, dtype, plan, counters, stream)) != cudaSuccess) return record_cuda_error(e);
    return SDPA_OK;
}
