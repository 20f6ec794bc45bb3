// nomas_seg_attn_static: segment attention without a caller-provided workspace.
//
// nomas_seg_attn needs device scratch (rotated Q and K, split partials, a
// status word) that the caller allocates and passes in. Some callers cannot
// allocate device memory at the point where they run attention: an operator
// plugin whose host framework hands it only its inputs and outputs, or code
// running where a cudaMalloc would synchronise the device or fail because the
// framework has already reserved all device memory. For them this entry point
// takes its scratch from a fixed array that is part of the library's device
// image: NOMAS_STATIC_SCRATCH_BYTES per GPU, held by every GPU that loads the
// library until the process exits.
//
// Set-up: the first call in each CUDA context (with that context current)
// looks up the array's device address with cudaGetSymbolAddress -- in host
// code the array's name is only a host-side stand-in, never a device address
// -- and clears its status header with an asynchronous memset on the call's
// stream, ahead of the call's kernels. Make that first call before any stream
// capture. The address is cached per context (by the driver's context id,
// which is never reused), so a context created after a device reset sets the
// array up again. Every later call shares the same array: calls that overlap
// on the GPU (different streams, or host threads racing on one device) race
// on it and corrupt each other's results, so such calls must be ordered by
// the caller -- the first call's clear included. The call allocates nothing:
// no cudaMalloc, cudaFree or allocating library routine runs on this path.
// nomas_seg_attn_static_status reads and clears the array's status header
// (bounded device waits that ran out), as nomas_device_status does for a
// caller's workspace.
#include "nomas_internal.h"

#include <mutex>

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[NOMAS_STATIC_SCRATCH_BYTES];

constexpr int kMaxContexts = 64;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct StaticScratch {
    std::mutex mu;
    bool resolved = false;
    CtxGetCurrentFn get_current = nullptr;
    CtxGetIdFn get_id = nullptr;
    unsigned long long ctx_id[kMaxContexts] = {};
    void* ptr[kMaxContexts] = {};
    int used = 0;
};

StaticScratch& scratch_table() {
    static StaticScratch t;
    return t;
}

// Driver entry points for the current context and its id (the library links
// the CUDA runtime statically and reaches the driver through it).
bool resolve_driver(StaticScratch& t) {
    if (!t.resolved) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            t.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            t.get_id = reinterpret_cast<CtxGetIdFn>(p);
        t.resolved = true;
    }
    return t.get_current && t.get_id;
}

// Device address of the static scratch in the current context; the first use
// in a context clears the status header on `stream`.
int static_scratch(void** out, cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NOMAS_ERR_CUDA; // also makes the primary context current
    StaticScratch& t = scratch_table();
    std::lock_guard<std::mutex> lock(t.mu);
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!resolve_driver(t) || t.get_current(&ctx) != CUDA_SUCCESS || !ctx || t.get_id(ctx, &id) != CUDA_SUCCESS)
        return NOMAS_ERR_CUDA;
    for (int i = 0; i < t.used; ++i)
        if (t.ctx_id[i] == id) {
            *out = t.ptr[i];
            return NOMAS_OK;
        }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return NOMAS_ERR_CUDA;
    // the status header starts at zero; the rest is fully written before it is read
    if (cudaMemsetAsync(p, 0, 256, stream) != cudaSuccess) return NOMAS_ERR_CUDA;
    const int slot = t.used < kMaxContexts ? t.used++ : kMaxContexts - 1; // the oldest entries stay
    t.ctx_id[slot] = id;
    t.ptr[slot] = p;
    *out = p;
    return NOMAS_OK;
}

} // namespace

extern "C" int nomas_seg_attn_static(const nomas_cache* c, const void* q, const void* k, const void* v,
                                     int64_t token_stride, int32_t n_video_frames, int32_t n_text, void* out,
                                     float* lse, void* stream) {
    const size_t need = nomas_seg_attn_workspace_min_bytes(c, n_video_frames, n_text);
    if (need == 0) // invalid descriptor or sizes: report the exact reason without touching memory
        return nomas_seg_attn(c, q, k, v, token_stride, n_video_frames, n_text, out, lse, nullptr, 0, stream);
    if (need > static_cast<size_t>(NOMAS_STATIC_SCRATCH_BYTES)) return NOMAS_ERR_WORKSPACE;
    void* ws = nullptr;
    const int rc = static_scratch(&ws, static_cast<cudaStream_t>(stream));
    if (rc != NOMAS_OK) return rc;
    return nomas_seg_attn(c, q, k, v, token_stride, n_video_frames, n_text, out, lse, ws,
                          static_cast<size_t>(NOMAS_STATIC_SCRATCH_BYTES), stream);
}

extern "C" int nomas_seg_attn_static_status(void* stream) {
    void* ws = nullptr;
    const int rc = static_scratch(&ws, static_cast<cudaStream_t>(stream));
    if (rc != NOMAS_OK) return rc;
    return nomas_device_status(ws, stream);
}
