// Internal interface between the C-ABI host code (nomas_host.cu) and the
// kernel translation units. Not installed; not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <utility>
#include <cstdint>

#include "nomas.h" // found through -I include

namespace nomas {

constexpr int kD = 128;             // head dimension
constexpr int kPairs = kD / 2;      // RoPE pairs per head
constexpr int kTPairs = 8;          // pairs of the t block (dims [0,16))
constexpr int kHWPairs = 28;        // pairs of the h and w blocks (dims [16,72), [72,128))
constexpr int kMaxFramesPerLaunch = 128;

// RoPE cos/sin rows. The t rows of the latent frames one launch touches travel
// as a launch argument (RopeTab). The spatial rows -- grid rows [0, grid_h)
// followed by grid columns [grid_h, grid_h + grid_w) -- depend only on
// (theta, grid) and are uploaded once per device and configuration into a
// table in the library's device image (rope_hw_device); kernels read them
// through L1. All values are computed on the host, so every launch sees the
// same fp32 bits as the oracle's tables.
template <int kFrames>
struct RopeTabT {
    float2 t[kFrames][kTPairs];
};
using RopeTab = RopeTabT<kMaxFramesPerLaunch>;
struct RopeHW {
    float2 hw[NOMAS_MAX_GRID_HW][kHWPairs];
};
constexpr int kRopeConfigs = 16; // distinct (theta, grid) configurations per device

// Device address of the spatial rows of configuration (theta, grid_h, grid_w)
// on the current device, uploading `host` on the first use of that
// configuration on that device (a blocking copy). cudaErrorMemoryAllocation
// when kRopeConfigs configurations are already in use on the device.
cudaError_t rope_hw_device(const RopeHW& host, float theta, int grid_h, int grid_w, const float2** dev);

// Unsigned division by a runtime constant d for n < 2^31 (Granlund-Montgomery
// round-up method): q = (umulhi(n, m) + n) >> s with s = ceil(log2 d) and
// m = floor(2^32 (2^s - d) / d) + 1.
struct FastDiv {
    uint32_t d, m, s;
};

inline FastDiv make_fastdiv(uint32_t d) {
    uint32_t s = 0;
    while ((uint64_t(1) << s) < d) ++s;
    const uint64_t m = ((uint64_t(1) << 32) * ((uint64_t(1) << s) - d)) / d + 1;
    return FastDiv{d, static_cast<uint32_t>(m), s};
}

#ifdef __CUDACC__
__device__ __forceinline__ uint32_t fast_div(uint32_t n, const FastDiv& f) {
    return (__umulhi(n, f.m) + n) >> f.s;
}
#endif

// Per-layer pointers of one commit launch (layers share every other argument).
struct CommitLayer {
    const uint16_t* k;      // segment K, BF16 bits, token-major
    const uint16_t* v;      // segment V
    void* ck;               // cache K (int8 codes or BF16 bits), head-major
    void* cv;
    float* cks;             // cache K scales (INT8 mode)
    float* cvs;
};
constexpr int kMaxLayersPerLaunch = 128; // RopeTab + CommitArgs + CommitLayers stay under the 32 KB argument limit
template <int kLayers>
struct CommitLayersT {
    CommitLayer l[kLayers];
};
using CommitLayers = CommitLayersT<kMaxLayersPerLaunch>;
// Launches of at most kSmallFrames frames and kSmallLayers layers (the common
// few-frame commit of one layer, the RoPE prep of a short segment) carry
// argument tables of that size: a launch's arguments are copied with it, and
// the full-size tables would be ~14 KB for a few hundred bytes used.
constexpr int kSmallFrames = 8, kSmallLayers = 8;

struct CommitArgs {
    int32_t n_layers;       // layers of this launch (entries of CommitLayers)
    int64_t token_stride;   // elements between tokens
    int64_t cap_tok;        // capacity_frames * tokens_per_frame
    int32_t heads, tpf, grid_h, grid_w;
    int32_t n_frames;       // frames written by this launch
    int32_t in_frame0;      // segment-local index of the first of them
    int64_t abs_frame0;     // absolute frame index of the first of them
    int32_t window;         // ring modulus (0: slot = absolute frame)
    int32_t slot0;          // slot of the first frame of this launch
    int32_t int8_mode;
    FastDiv div_heads, div_tpf, div_gw;
    int32_t head_group;     // heads of one token handled by one warp task (set by launch_commit)
    FastDiv div_groups;     // ceil(heads / head_group)
    FastDiv div_layer_tasks; // warp tasks per layer (set by launch_commit)
    const float2* hw;       // spatial RoPE rows in device memory (rope_hw_device)
};
static_assert(sizeof(RopeTab) + sizeof(CommitArgs) + sizeof(CommitLayers) <= 32764,
              "commit launch arguments exceed the 32,764-byte limit");

struct PrepArgs {
    const uint16_t* q;      // segment Q, BF16 bits, token-major
    const uint16_t* k;
    int64_t token_stride;
    uint16_t* qt;           // rotated Q, head-major [heads][nq][128]
    uint16_t* kt;           // rotated K, head-major
    int32_t heads, tpf, grid_h, grid_w;
    int32_t nq, nv;         // tokens in the segment, video tokens
    int32_t tok0, tok1;     // token range handled by this launch
    int32_t frame0;         // segment-local frame of table row t[0]
    FastDiv div_heads, div_tpf, div_gw;
    unsigned* counters;     // split-KV arrival counters of the attention call, zeroed here
    int32_t n_counters;     // (by the launch with tok0 == 0 only)
    const float2* hw;       // spatial RoPE rows in device memory (rope_hw_device)
    // INT8 caches (FP16 operands, nomas_f16.cuh); null te for a BF16 cache
    float4* te;             // [heads][tiles_c + tiles_q] tile records
    float* qs;              // [heads][nq] 2^a_i of each Q row
    const float* ksc;       // cache K / V scales [heads][cap_tok]
    const float* vsc;
    int64_t cap_tok;
    int32_t nc, tiles_c, tiles_q;
    int32_t te_cache_tasks; // heads * tiles_c on the launch with tok0 == 0, else 0
};

struct AttnArgs {
    int32_t heads;
    int32_t nq;             // current-segment tokens
    int32_t nc;             // visible cache tokens
    int32_t tiles_c;        // ceil(nc / 128)
    int32_t tiles_q;        // ceil(nq / 128)
    int32_t pairs;          // Q-tile pairs per head: ceil(ceil(nq/128) / 2)
    int32_t splits;         // KV splits per (head, pair)
    int32_t tiles_per_split;
    int64_t cap_tok;        // cache row stride between heads (INT8 path)
    const int8_t* kc8;      // INT8 cache codes (INT8 mode)
    const int8_t* vc8;
    const float* ksc;       // INT8 cache scales
    const float* vsc;
    uint16_t* out;          // [nq][heads][128] BF16
    float* lse;             // [heads][nq] or null
    uint4* part_o;          // splits > 1: [splits][units][16][256] O / l * 2^-e in FP16, 8 dims per word
    float4* part_ml;        // splits > 1: [splits][units][256] (reference max in log2 units, sum, 2^e, 0)
    unsigned* counters;     // splits > 1: [units] arrivals; the last CTA of a unit merges the splits
    unsigned* err;          // workspace status word
    float scale_log2;       // log2(e) / sqrt(128)
    const float4* te;       // INT8: [heads][tiles_c + tiles_q] tile records (2^b, 2^-b, c, 2^-c)
    const float* qs;        // INT8: [heads][nq] 2^a_i of each FP16 Q row
};

// Dequantisation of an INT8 cache's visible window into an FP16 copy, once per
// attention call: rows [0, nc) of every head, written head-major
// [heads][nc][128], each 128-key tile as code * RN16(scale * 2^-e) with the
// tile's exponent e (nomas_f16.cuh) -- the values the in-shared-memory
// conversion produces.
struct DequantArgs {
    const int8_t* kc;
    const int8_t* vc;
    const float* ks;
    const float* vs;
    uint16_t* kd;
    uint16_t* vd;
    int64_t cap_tok; // token capacity of one head's slab in the cache
    int32_t nc;      // visible tokens per head
    int32_t heads;
    int32_t tiles_c; // ceil(nc / 128)
};

// Forms of the attention kernel: a BF16 cache; an INT8 cache read through its
// FP16 window copy; an INT8 cache converted to FP16 in shared memory.
enum class AttnForm { kBf16Cache, kInt8Window, kInt8Fused };

// Per-latent-frame camera cross-attention: rows are (video token, head) pairs,
// row = token * heads + head; token i uses camera chunk (i / tpf) / chunk_frames.
struct CamArgs {
    const uint16_t* q;      // video Q, BF16 bits, token-major
    int64_t q_stride;       // elements between tokens
    const uint16_t* k_cam;  // [n_chunks][n_cam][heads][128]
    const uint16_t* v_cam;
    uint16_t* out;          // BF16 bits, token-major
    int64_t out_stride;
    int64_t rows;           // n_video * heads (< 2^31)
    int32_t heads, n_cam;
    FastDiv div_heads, div_tpf, div_chunk;
    float scale_log2;       // log2(e) / sqrt(128)
};

// Launch `kernel` with programmatic stream serialisation: it may begin while
// the previous kernel on `s` finishes and must call grid_dep_wait before it
// reads anything that kernel (or an earlier one) wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Kernel launchers (return cudaError_t of the launch).
cudaError_t launch_commit(const CommitArgs& a, const CommitLayers& layers, const RopeTab& tab, cudaStream_t s);
cudaError_t launch_prep(const PrepArgs& a, const RopeTab& tab, cudaStream_t s);
cudaError_t launch_attn(const AttnArgs& a, AttnForm form, const CUtensorMap& tm_q, const CUtensorMap& tm_kcur,
                        const CUtensorMap& tm_vcur, const CUtensorMap& tm_kc, const CUtensorMap& tm_vc,
                        cudaStream_t s);
cudaError_t launch_dequant_window(const DequantArgs& a, cudaStream_t s);
cudaError_t launch_camera_attn(const CamArgs& a, cudaStream_t s);

} // namespace nomas
