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
// Set-up: the first call on each device (with that device current) looks up
// the array's device address with cudaGetSymbolAddress -- in host code the
// array's name is only a host-side stand-in, never a device address -- and
// clears its status header once. Make that first call before any stream
// capture. Every later call shares the same array: calls that overlap on the
// GPU (different streams, or host threads racing on one device) race on it
// and corrupt each other's results, so such calls must be ordered by the
// caller. The call allocates nothing: no cudaMalloc, cudaFree or allocating
// library routine runs on this path.
#include "nomas_internal.h"

#include <mutex>

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[NOMAS_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

struct StaticScratch {
    std::mutex mu;
    void* ptr[kMaxDevices] = {};
};

StaticScratch& scratch_table() {
    static StaticScratch t;
    return t;
}

// Device address of the static scratch on the current device (set-up on first use).
int static_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NOMAS_ERR_CUDA;
    StaticScratch& t = scratch_table();
    std::lock_guard<std::mutex> lock(t.mu);
    if (!t.ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return NOMAS_ERR_CUDA;
        // the status header starts at zero; the rest is fully written before it is read
        if (cudaMemset(p, 0, 256) != cudaSuccess) return NOMAS_ERR_CUDA;
        t.ptr[dev] = p;
    }
    *out = t.ptr[dev];
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
    const int rc = static_scratch(&ws);
    if (rc != NOMAS_OK) return rc;
    return nomas_seg_attn(c, q, k, v, token_stride, n_video_frames, n_text, out, lse, ws,
                          static_cast<size_t>(NOMAS_STATIC_SCRATCH_BYTES), stream);
}
