/*
 * sdpa.h -- C ABI of the B200 (sm_100a) fused scaled-dot-product attention
 * forward pass.
 *
 * Operation (per batch b, query head h, query row i):
 *
 *     out[b,h,i,:] = softmax_j( scale * q[b,h,i,:] . k[b,g,j,:] + mask[b,h,i,j] ) . v[b,g,j,:]
 *
 *   - the definition is the fixed composite of MLX issue #3585
 *     ("mx.fast.scaled_dot_product_attention produces incorrect attention
 *     scores (MLX 0.31.2)"), section "Reproduction": scores = q k^T * scale,
 *     softmax along the key axis, times v;
 *   - GQA: g = h / (Hq / Hkv), the contiguous grouping [B, n_kv, n_rep, qL, kL]
 *     of MLX issue #3885 ("Metal SDPA: no fused path for head_dim=512"),
 *     section "Measured impact";
 *   - path split: Lq <= 8 runs the decode ("vector") path, Lq > 8 the prefill
 *     ("full") path, as in that issue's section "Current routing";
 *   - head dims: Dqk in {64, 72, 80, 96, 128, 192, 256, 512} with Dv == Dqk,
 *     plus (Dqk, Dv) = (192, 128) (same section; head dim 72 from MLX PR #4330
 *     "Support head dimension 72 in Metal full attention"), plus (40, 32):
 *     absorbed multi-head latent attention on the small MLA fixture of mlxcel
 *     issue #1065, section "Why this is a precision problem" (keys = 32 latent
 *     + 8 rope columns, values = the 32 latent columns, so v may point at k
 *     with k's strides); these dims run on the CUDA-core kernels;
 *   - masks: none, additive, boolean, causal (MLX PR #4330, "Proposed changes"),
 *     and a causal sliding window (the local-attention layers of Gemma 4's
 *     hybrid layout, MLX issue #3885, "Current routing"; sdpa_forward_window).
 *
 * Layout is never inferred from a tensor's shape: every tensor is passed as a
 * base pointer plus explicit (b, h, l, d) element strides, so [B,L,H,D] and
 * [B,H,L,D] buffers (or any other strided view) are described exactly.  The
 * layout misread of MLX issue #3585, section "Root cause analysis", cannot
 * happen through this interface.
 *
 * Readings where the pages are silent:
 *   - additive mask is added after scaling; -inf entries remove a key;
 *   - boolean mask: nonzero = attend, zero = removed;
 *   - causal with Lq != Lk is aligned bottom-right: key j is visible to query
 *     i iff j <= i + (Lk - Lq);
 *   - sliding window of W keys, with the same alignment: key j is visible to
 *     query i iff i + (Lk - Lq) - W < j <= i + (Lk - Lq);
 *   - a query row with no visible key yields zeros (never NaN).
 *
 * Threading: the functions are thread-safe.  Execution is asynchronous on the
 * caller's stream; validation is synchronous and happens before any launch.
 * The fp16/bf16 decode kernel is launched with programmatic dependent launch
 * allowed: its blocks may start while the previous kernel of the stream is
 * still running, but none touches global memory before that kernel has
 * completed (griddepcontrol.wait), so stream order holds for every input and
 * output.  A later kernel launched the same way may likewise start early and
 * must wait the same way before it reads this call's output.
 * There is no fallback path of any kind: a case the kernels do not cover is
 * rejected with an error status and nothing is launched.
 */
#ifndef SDPA_B200_SDPA_H
#define SDPA_B200_SDPA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element types of q, k, v, out (and of an additive mask). */
typedef enum {
    SDPA_F32 = 0,   /* IEEE binary32; fp32-class accuracy: FFMA, or TF32 tensor cores only with
                       the three-term split hi*hi + hi*lo + lo*hi (never plain TF32 or fp16) */
    SDPA_F16 = 1,   /* IEEE binary16 storage, fp32 accumulation */
    SDPA_BF16 = 2   /* bfloat16 storage, fp32 accumulation */
} sdpa_dtype;

typedef enum {
    SDPA_MASK_NONE = 0,      /* mask must be NULL */
    SDPA_MASK_ADDITIVE = 1,  /* mask: same element type as q, added to scale*q.k */
    SDPA_MASK_BOOL = 2,      /* mask: uint8, nonzero = attend */
    SDPA_MASK_CAUSAL = 3,    /* mask must be NULL; bottom-right aligned */
    SDPA_MASK_SLIDING = 4    /* causal sliding window; only through sdpa_forward_window (which
                                carries the window length); sdpa_supported accepts it */
} sdpa_mask_kind;

typedef enum {
    SDPA_OK = 0,
    SDPA_ERR_INVALID_ARG = 1,         /* negative size, Hq % Hkv != 0, bad enum, non-finite scale */
    SDPA_ERR_UNSUPPORTED_DIM = 2,     /* (Dqk, Dv) not in the supported set */
    SDPA_ERR_UNSUPPORTED_STRIDE = 3,  /* d-stride != 1, negative stride, or a stride that is not a
                                         multiple of 16 bytes */
    SDPA_ERR_MISALIGNED = 4,          /* a base pointer not 16-byte aligned */
    SDPA_ERR_LAUNCH_CONFIG = 5,       /* the launch shape exceeds a device limit (grid size,
                                         shared memory); nothing was launched */
    SDPA_ERR_CUDA = 6,                /* a CUDA runtime call failed (see sdpa_last_cuda_error) */
    SDPA_ERR_TIMEOUT = 7,             /* a bounded in-kernel wait ran out (debug check only) */
    SDPA_ERR_NO_MEMORY = 8,           /* the split-K workspace could not be allocated */
    SDPA_ERR_NULL_POINTER = 9,        /* q, k, v or out is NULL (with a non-empty problem), or the
                                         mask pointer does not match mask_kind */
    SDPA_ERR_TOO_LARGE = 10           /* a size exceeds the kernels' index range */
} sdpa_status;

typedef enum {
    SDPA_PATH_NONE = 0,     /* empty problem: nothing to launch */
    SDPA_PATH_PREFILL = 1,  /* Lq > 8: tiled flash kernel (tcgen05 kind::f16 for fp16/bf16; for fp32
                               tcgen05 kind::tf32 with a three-term hi/lo split at head dims
                               (40,32), 64, 72, 80, 96, FFMA at the others) */
    SDPA_PATH_DECODE = 2    /* Lq <= 8: split-K kernel with the log-sum-exp merge of its
                               splits in the same launch */
} sdpa_path;

/*
 * sdpa_forward -- out = softmax(scale * q k^T + mask) v.
 *
 * q    : device pointer, element (b,h,i,d) at q + b*s[0] + h*s[1] + i*s[2] + d*s[3]   (h < Hq,  i < Lq, d < Dqk)
 * k    : device pointer, element (b,g,j,d) at k + b*s[4] + g*s[5] + j*s[6] + d*s[7]   (g < Hkv, j < Lk, d < Dqk)
 * v    : device pointer, element (b,g,j,e) at v + b*s[8] + g*s[9] + j*s[10] + e*s[11] (g < Hkv, j < Lk, e < Dv)
 * out  : device pointer, element (b,h,i,e) at out + b*s[12] + h*s[13] + i*s[14] + e*s[15]
 *        (the only memory the call writes besides the library's own workspace)
 * strides : 16 element strides (not bytes).  Requirements: every d-stride
 *        (s[3], s[7], s[11], s[15]) is 1; every other stride is >= 0 and, times
 *        the element size, a multiple of 16 bytes (a stride whose dimension has
 *        extent 1 is not checked).
 * scale: multiplies q.k before the mask is added (usually Dqk^-0.5).
 * mask_kind / mask / mask_strides:
 *        ADDITIVE: mask element (b,h,i,j) at mask + b*m[0] + h*m[1] + i*m[2] + j*m[3],
 *                  element type = dtype; strides in elements, 0 broadcasts.
 *        BOOL:     same indexing, uint8 elements.
 *        NONE / CAUSAL: mask and mask_strides must be NULL.
 *        SLIDING: refused here (SDPA_ERR_INVALID_ARG); use sdpa_forward_window.
 * dtype : sdpa_dtype of q, k, v, out.
 * stream: a cudaStream_t (NULL = the legacy default stream).
 *
 * Requirements: Hq % Hkv == 0; (Dqk, Dv) supported; base pointers 16-byte
 * aligned.  out must not overlap q, k, v or mask.
 * Empty problems (B, Hq or Lq == 0) return SDPA_OK without launching; Lk == 0
 * writes zeros to out.
 * Ownership: all pointers are the caller's.  The decode path uses a split-K
 * workspace the library allocates on first use per (device, stream), keeps,
 * and frees in sdpa_shutdown(); two calls on the same stream share it safely
 * because the stream orders them.  A larger problem grows the workspace
 * without freeing the smaller buffer (a CUDA graph captured earlier may still
 * use it), so graphs captured with sdpa_forward calls stay valid until
 * sdpa_shutdown.
 * Returns an sdpa_status.  On any status other than SDPA_OK and SDPA_ERR_CUDA
 * nothing was launched.
 */
int sdpa_forward(const void* q, const void* k, const void* v, void* out,
                 int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk,
                 int64_t Dqk, int64_t Dv, const int64_t strides[16], float scale,
                 int mask_kind, const void* mask, const int64_t mask_strides[4],
                 int dtype, void* stream);

/*
 * sdpa_forward_window -- causal sliding-window (local) attention: with
 * own = i + (Lk - Lq), key j is visible to query i iff own - window < j <= own,
 * the `window` most recent keys up to the query's own bottom-right-aligned
 * position.  Gemma 4's hybrid layout interleaves such layers with global ones
 * (MLX issue #3885, "Current routing"); the pages give no rule for the
 * window, and this is the plainest reading of local causal attention.
 * window >= Lk is plain causal attention; a query whose window holds no key
 * (own < 0) yields zeros.
 *
 * Arguments are those of sdpa_forward without the mask arguments; window >= 1
 * (else SDPA_ERR_INVALID_ARG).  Both paths skip every key tile that lies
 * outside all of a CTA's windows: those keys are never loaded.
 */
int sdpa_forward_window(const void* q, const void* k, const void* v, void* out,
                        int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk,
                        int64_t Dqk, int64_t Dv, const int64_t strides[16], float scale,
                        int64_t window, int dtype, void* stream);

/*
 * sdpa_forward_noalloc -- sdpa_forward for callers that cannot allocate device
 * memory when they call attention: a process whose memory manager already owns
 * the whole GPU (a caching allocator, a serving runtime with a fixed memory
 * budget), or a latency-critical decode loop that must never pay for
 * cudaMalloc / cudaFree, which can synchronise the device.  The pages describe
 * no counterpart of this entry point.
 *
 * Arguments, layout, validation and result are those of sdpa_forward, but it
 * covers only the decode path with fp16 / bf16 (Lq <= 8) on the head dims of
 * the tensor-core decode kernel (every supported pair except the absorbed-MLA
 * (40, 32)); other problems return SDPA_ERR_INVALID_ARG, decided before any
 * CUDA call (an empty problem returns SDPA_OK).  It allocates
 * nothing: the split-K partials and the per-group completion counters go to
 * a 4 MiB array compiled into the library (the counters take its first 64 KiB
 * and are cleared by each call with a memset on `stream`), which every GPU
 * that loads the library holds until the process exits.  A problem whose
 * partials do not fit (query rows x splits x (Dv + 1) fp32 values, with the
 * split count sdpa_forward would use) returns SDPA_ERR_TOO_LARGE and launches
 * nothing.  The first call on each device
 * looks up that array's device address (with the device current); make it
 * before any stream capture.  All calls on a device share the one array, which
 * keeps the last call's contents: calls that may overlap on the GPU (different
 * streams with no ordering between them) race and must not be issued.  The call
 * counters do not count this entry point.
 */
int sdpa_forward_noalloc(const void* q, const void* k, const void* v, void* out,
                         int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk,
                         int64_t Dqk, int64_t Dv, const int64_t strides[16], float scale,
                         int mask_kind, const void* mask, const int64_t mask_strides[4],
                         int dtype, void* stream);

/*
 * sdpa_supported -- the same validation sdpa_forward runs, without pointers
 * and without launching.  Writes the path that would run (sdpa_path) to
 * *path_out when path_out is not NULL.  Returns an sdpa_status; SDPA_OK means
 * sdpa_forward would accept these sizes and strides (given aligned pointers).
 */
int sdpa_supported(int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk,
                   int64_t Dqk, int64_t Dv, const int64_t strides[16], int mask_kind,
                   const int64_t mask_strides[4], int dtype, int* path_out);

/* Static text for a status code. */
const char* sdpa_error_string(int status);

/* Text of the CUDA error (or failed workspace allocation) of this thread's most
 * recent sdpa_forward, sdpa_forward_window or sdpa_forward_noalloc call; ""
 * when that call had none.  Each call clears it on entry. */
const char* sdpa_last_cuda_error(void);

/*
 * Call counters (process-wide).  Invariant:
 *   calls == prefill_calls + decode_calls + empty_calls + rejected_calls.
 * The kernel counters say which kernel family served each call.
 */
typedef struct {
    uint64_t calls;
    uint64_t prefill_calls;
    uint64_t decode_calls;
    uint64_t empty_calls;
    uint64_t rejected_calls;
    uint64_t prefill_tcgen05_launches;  /* fp16/bf16 prefill on tcgen05 tensor cores */
    uint64_t prefill_ffma_launches;     /* fp32 prefill on CUDA cores */
    uint64_t decode_mma_launches;       /* fp16/bf16 split-K decode */
    uint64_t decode_ffma_launches;      /* fp32 split-K decode */
    uint64_t combine_launches;          /* separate combine launches: always 0 (every split kernel
                                           merges its partials in the same launch) */
    uint64_t prefill_tf32_launches;     /* fp32 prefill on tcgen05 kind::tf32, three-term split */
} sdpa_counters;

void sdpa_get_counters(sdpa_counters* out);
void sdpa_reset_counters(void);

/*
 * Kernel launches the most recent successful sdpa_forward on this thread
 * made (1, or 0 for an empty problem).  Lets a caller count launches without
 * a profiler.
 */
int sdpa_last_launch_count(void);

/*
 * Reads and clears the device-side error flag that bounded in-kernel waits
 * set when they give up (0 = none).  Synchronises the stream.  Returns an
 * sdpa_status: SDPA_ERR_TIMEOUT if the flag was set; in that case it also
 * zeroes the decode split-barrier counters of this (device, stream)'s
 * workspace (on the stream, synchronously), so the next decode call on the
 * stream starts from a clean barrier whatever the timed-out call left.
 */
int sdpa_check_device_error(void* stream, int* code_out);

/*
 * Test and diagnostic hooks; none is needed in normal use.  Each is
 * process-wide and applies from the next call.  They exist so that the
 * failure paths (a bounded wait that runs out, a workspace that cannot be
 * allocated) can be exercised without faulting or hanging a GPU.
 *   SDPA_DEBUG_WAIT_LIMIT_NS: every bounded wait of the fp16/bf16 decode
 *       kernel gives up after `value` nanoseconds instead of about 2 s
 *       (value <= 0 restores the default).
 *   SDPA_DEBUG_DECODE_BARRIER_EXTRA: added to the number of split arrivals
 *       the decode kernel's split barrier waits for (0..1024; 0 restores).
 *       A value > 0 makes the target unreachable: every CTA's wait runs out
 *       after the wait limit, the device error flag is set (read it with
 *       sdpa_check_device_error) and the output is left unwritten.
 *   SDPA_DEBUG_FAIL_ALLOCS: the next `value` calls of sdpa_forward that need
 *       split-K workspace fail as if the allocation had failed: they return
 *       SDPA_ERR_NO_MEMORY and launch nothing.
 * Returns SDPA_OK, or SDPA_ERR_INVALID_ARG for an unknown knob or a value out
 * of range.
 */
typedef enum {
    SDPA_DEBUG_WAIT_LIMIT_NS = 0,
    SDPA_DEBUG_DECODE_BARRIER_EXTRA = 1,
    SDPA_DEBUG_FAIL_ALLOCS = 2
} sdpa_debug_knob;

int sdpa_debug_set(int knob, int64_t value);

/* Bytes of split-K workspace sdpa_forward currently holds, over every device
 * and stream (0 before the first decode call that splits keys). */
int64_t sdpa_workspace_bytes(void);

/*
 * Optional per-kernel timing with CUDA events (off by default).  While
 * enabled, sdpa_forward brackets every kernel it launches with two events
 * recorded on the call's stream.  sdpa_profile_collect waits for those events,
 * adds their elapsed times per kernel family into launches[] / total_ms[]
 * (arrays of SDPA_KERNEL_FAMILIES entries, indexed by sdpa_kernel_family),
 * and forgets them.  Nothing else changes: the same kernels run.
 */
typedef enum {
    SDPA_KERNEL_PREFILL_TCGEN05 = 0,
    SDPA_KERNEL_PREFILL_FFMA = 1,
    SDPA_KERNEL_DECODE_MMA = 2,
    SDPA_KERNEL_DECODE_FFMA = 3,
    SDPA_KERNEL_COMBINE = 4,
    SDPA_KERNEL_ZERO_FILL = 5,
    SDPA_KERNEL_PREFILL_TF32 = 6,
    SDPA_KERNEL_FAMILIES = 7
} sdpa_kernel_family;

int sdpa_profile_enable(int on);
int sdpa_profile_collect(uint64_t launches[SDPA_KERNEL_FAMILIES], double total_ms[SDPA_KERNEL_FAMILIES]);

/* Frees every cached workspace.  Call with no sdpa work in flight. */
int sdpa_shutdown(void);

/* ABI version of this header (increases on incompatible change): 2 added the
 * sliding-window entry point, the tf32 counter and kernel family. */
int sdpa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SDPA_B200_SDPA_H */
