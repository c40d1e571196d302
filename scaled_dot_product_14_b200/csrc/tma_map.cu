// tma_map.cu -- host-side construction of TMA tensor maps from explicit
// (b, h, l, d) element strides (cuTensorMapEncodeTiled through the runtime's
// driver entry point, so the library links no driver library).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.h"

namespace sdpa {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// Encoded maps are cached by everything that determines them (the kind of
// map, base address, dtype, sizes, strides and box rows), so a call repeated
// on the same tensors does not encode again.  A small table with round-robin
// replacement; encoding is a host-only computation, so a miss costs only time.
struct MapKey {
    int kind, dtype, box_rows;
    const void* base;
    int64_t D, L, H, B, st[3];
    bool operator==(const MapKey& o) const {
        return kind == o.kind && dtype == o.dtype && box_rows == o.box_rows && base == o.base && D == o.D &&
               L == o.L && H == o.H && B == o.B && st[0] == o.st[0] && st[1] == o.st[1] && st[2] == o.st[2];
    }
};
struct MapEntry {
    MapKey key;
    CUtensorMap map;
    MapAxes ax;
    bool used = false;
};
constexpr int kMapCache = 64;
std::mutex g_map_mu;
MapEntry g_maps[kMapCache];
int g_map_next = 0;

MapKey map_key(int kind, const void* base, int dtype, int64_t D, int64_t L, int64_t H, int64_t B,
               const int64_t* st, int box_rows) {
    MapKey k{};
    k.kind = kind;
    k.dtype = dtype;
    k.box_rows = box_rows;
    k.base = base;
    k.D = D;
    k.L = L;
    k.H = H;
    k.B = B;
    k.st[0] = st[0];
    k.st[1] = st[1];
    k.st[2] = st[2];
    return k;
}

bool cache_find(const MapKey& k, CUtensorMap* map, MapAxes* ax) {
    std::lock_guard<std::mutex> lk(g_map_mu);
    for (auto& e : g_maps)
        if (e.used && e.key == k) {
            *map = e.map;
            *ax = e.ax;
            return true;
        }
    return false;
}

void cache_put(const MapKey& k, const CUtensorMap& map, const MapAxes& ax) {
    std::lock_guard<std::mutex> lk(g_map_mu);
    MapEntry& e = g_maps[g_map_next];
    g_map_next = (g_map_next + 1) % kMapCache;
    e.key = k;
    e.map = map;
    e.ax = ax;
    e.used = true;
}

bool encode_tiled(CUtensorMap* map, MapAxes* ax, const void* base, int dtype, int64_t D, int64_t L, int64_t H,
                  int64_t B, const int64_t* st, int box_rows);
bool encode_rows(CUtensorMap* map, MapAxes* ax, const void* base, int dtype, int64_t D, int64_t L, int64_t H,
                 int64_t B, const int64_t* st, int box_rows);

}  // namespace

bool make_tensor_map(CUtensorMap* map, MapAxes* ax, const void* base, int dtype, int64_t D, int64_t L, int64_t H,
                     int64_t B, const int64_t* st, int box_rows) {
    const MapKey k = map_key(0, base, dtype, D, L, H, B, st, box_rows);
    if (cache_find(k, map, ax)) return true;
    if (!encode_tiled(map, ax, base, dtype, D, L, H, B, st, box_rows)) return false;
    cache_put(k, *map, *ax);
    return true;
}

bool make_tensor_map_rows(CUtensorMap* map, MapAxes* ax, const void* base, int dtype, int64_t D, int64_t L,
                          int64_t H, int64_t B, const int64_t* st, int box_rows) {
    const MapKey k = map_key(1, base, dtype, D, L, H, B, st, box_rows);
    if (cache_find(k, map, ax)) return true;
    if (!encode_rows(map, ax, base, dtype, D, L, H, B, st, box_rows)) return false;
    cache_put(k, *map, *ax);
    return true;
}

namespace {

// A 4-D tiled map (d, then the sequence / head / batch axes in increasing
// stride order; an axis of extent 1 or stride 0 is pinned to coordinate 0),
// 128-byte swizzle, box = 128 bytes of d (64 16-bit or 32 fp32 elements) x
// box_rows rows, zero fill out of bounds.
bool encode_tiled(CUtensorMap* map, MapAxes* ax, const void* base, int dtype, int64_t D, int64_t L, int64_t H,
                  int64_t B, const int64_t* st, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    const int64_t esz = dtype == 0 ? 4 : 2;
    struct Axis {
        int which;   // 0 = l, 1 = h, 2 = b
        int64_t ext, stride;
    } axes[3] = {{0, L, st[2] * esz}, {1, H, st[1] * esz}, {2, B, st[0] * esz}};
    // degenerate axes go last with a stride past every other axis
    int64_t span = ((D * esz + 15) / 16) * 16;
    for (auto& a : axes)
        if (a.ext > 1 && a.stride > 0 && a.stride * a.ext > span) span = a.stride * a.ext;
    for (auto& a : axes)
        if (a.ext <= 1 || a.stride == 0) {
            a.ext = 1;
            a.stride = ((span + 15) / 16) * 16;
        }
    // the sequence axis must stay a real dimension for the box rows; sort by (degenerate, stride)
    for (int x = 0; x < 3; ++x)
        for (int y = x + 1; y < 3; ++y) {
            const bool dx = axes[x].ext == 1 && axes[x].which != 0, dy = axes[y].ext == 1 && axes[y].which != 0;
            if (dx > dy || (dx == dy && axes[y].stride < axes[x].stride)) {
                Axis t = axes[x];
                axes[x] = axes[y];
                axes[y] = t;
            }
        }
    cuuint64_t gdim[4] = {(cuuint64_t)D, 0, 0, 0};
    cuuint64_t gstride[3];
    int pos[3] = {0, 0, 0};
    for (int x = 0; x < 3; ++x) {
        gdim[x + 1] = (cuuint64_t)axes[x].ext;
        gstride[x] = (cuuint64_t)axes[x].stride;
        pos[axes[x].which] = (axes[x].ext > 1 || axes[x].which == 0) ? x + 1 : 0;
    }
    cuuint32_t box[4] = {(cuuint32_t)(128 / esz), 1, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    for (int x = 0; x < 3; ++x)
        if (axes[x].which == 0) box[x + 1] = (cuuint32_t)box_rows;
    const CUtensorMapDataType dt = dtype == 0   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : dtype == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUresult r = fn(map, dt, 4, const_cast<void*>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    ax->l_pos = pos[0];
    ax->h_pos = pos[1];
    ax->b_pos = pos[2];
    return r == CUDA_SUCCESS;
}

// A 5-D map whose box covers every 64-element chunk of a row at once (one copy
// instead of D / 64): dim 0 = 64 elements, dim 1 = the sequence axis, dim 2 =
// the D / 64 chunks (stride 128 bytes), dims 3 / 4 = head / batch (an extent-1
// or zero-stride axis is pinned to coordinate 0).  D must be a multiple of 64,
// so every chunk lies inside its row.  Shared memory receives the box chunk by
// chunk: [chunk][row][64 elements], the layout of D / 64 separate boxes.
bool encode_rows(CUtensorMap* map, MapAxes* ax, const void* base, int dtype, int64_t D, int64_t L, int64_t H,
                 int64_t B, const int64_t* st, int box_rows) {
    auto fn = encode_fn();
    if (!fn || dtype == 0 || D % 64 != 0 || D / 64 > 256) return false;   // 16-bit elements only
    const int64_t esz = 2;
    int64_t span = D * esz;
    const int64_t ext[3] = {L, H, B}, str[3] = {st[2] * esz, st[1] * esz, st[0] * esz};
    for (int x = 0; x < 3; ++x)
        if (ext[x] > 1 && str[x] > 0 && str[x] * ext[x] > span) span = str[x] * ext[x];
    span = (span + 15) / 16 * 16;
    cuuint64_t gdim[5] = {64, (cuuint64_t)L, (cuuint64_t)(D / 64), 1, 1};
    cuuint64_t gstride[4] = {(cuuint64_t)(L > 1 && str[0] > 0 ? str[0] : span), 128, (cuuint64_t)span,
                             (cuuint64_t)span};
    ax->l_pos = 1;
    ax->h_pos = 0;
    ax->b_pos = 0;
    if (H > 1 && str[1] > 0) {
        gdim[3] = (cuuint64_t)H;
        gstride[2] = (cuuint64_t)str[1];
        ax->h_pos = 3;
    }
    if (B > 1 && str[2] > 0) {
        gdim[4] = (cuuint64_t)B;
        gstride[3] = (cuuint64_t)str[2];
        ax->b_pos = 4;
    }
    cuuint32_t box[5] = {64, (cuuint32_t)box_rows, (cuuint32_t)(D / 64), 1, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUtensorMapDataType dt =
        dtype == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    return fn(map, dt, 5, const_cast<void*>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace sdpa
