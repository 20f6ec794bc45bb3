// Per-latent-frame camera cross-attention (Hy-Nomas model card, "Text and
// Camera Conditioning"; "Hy-Nomas Explained" blog, "Camera conditioning"):
// after the video MLP of each double-stream block, the video tokens query the
// projected camera features; with per-chunk camera attention and a chunk of
// one latent frame, the tokens of latent frame t see only the camera tokens
// of their own chunk (one token per latent frame in the blog's reading).
//
//   out[i][h] = softmax_j(<q[i][h], k[c][j][h]> / sqrt(128)) . v[c][j][h],
//   c = (i / tokens_per_frame) / chunk_frames,  j < n_cam.
//
// The key set of a row is tiny (n_cam vectors, a few KB per chunk for all
// heads, held in L1), so the work is one read of Q and one write of O: an
// HBM-bound stream, not a contraction. Layout of the work: 8 threads per
// (token, head) row, each owning 16 of the 128 dims as two 16-byte vectors;
// dot products reduce across the row's 8-lane group by shuffles; an online
// softmax runs over the chunk's camera tokens in fp32 (with one token the
// weight is exactly 1 and the output is that token's V). Two rows per group
// are in flight per iteration (all their Q loads issue before any
// arithmetic); the grid is one resident wave with a grid-stride loop.
#include "nomas_internal.h"

#include <cuda_bf16.h>

namespace nomas {
namespace {

// 8 threads per row with two 16-byte vectors each, two rows in flight, 3 blocks
// of 256 threads per SM (80 registers, no spills). Measured on B200 for a
// 72-frame segment with one camera token per frame: 4.6 TB/s, against 3.8 TB/s
// for 16 threads per row (per-row index and softmax work repeated 16 times,
// half the bytes in flight) and 4.0 TB/s for four rows in flight (spills).
constexpr int kThreads = 256;
constexpr int kMinBlocksPerSm = 3;
constexpr int kLanesPerRow = 8;                 // threads per (token, head) row
constexpr int kVecs = 128 / 8 / kLanesPerRow;   // 16-byte vectors per thread per row
constexpr int kGroups = kThreads / kLanesPerRow;
constexpr int kRowsInFlight = 2;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&p);
}

__global__ void __launch_bounds__(kThreads, kMinBlocksPerSm) camera_attn_kernel(const CamArgs a) {
    const int lane = threadIdx.x & 31;
    const int sub = threadIdx.x & (kLanesPerRow - 1); // this thread's vectors: sub + v * kLanesPerRow
    const unsigned mask = (kLanesPerRow == 32 ? 0xFFFFFFFFu : ((1u << kLanesPerRow) - 1u))
                          << (lane & (32 - kLanesPerRow)); // this row's lane group
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kGroups;
    int64_t row0 = static_cast<int64_t>(blockIdx.x) * kGroups + (threadIdx.x / kLanesPerRow);

    for (; row0 < a.rows; row0 += stride * kRowsInFlight) {
        uint4 qv[kRowsInFlight][kVecs];
        int64_t tok[kRowsInFlight];
        int32_t head[kRowsInFlight], chunk[kRowsInFlight];
        bool live[kRowsInFlight];
        // issue every row's Q loads before any arithmetic
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
            const int64_t row = row0 + r * stride;
            live[r] = row < a.rows;
            const uint32_t rr = live[r] ? static_cast<uint32_t>(row) : 0u;
            const uint32_t t = fast_div(rr, a.div_heads);
            tok[r] = t;
            head[r] = static_cast<int32_t>(rr - t * static_cast<uint32_t>(a.heads));
            chunk[r] = static_cast<int32_t>(fast_div(fast_div(t, a.div_tpf), a.div_chunk));
            const uint4* qp = reinterpret_cast<const uint4*>(a.q + tok[r] * a.q_stride + head[r] * kD) + sub;
#pragma unroll
            for (int v = 0; v < kVecs; ++v) qv[r][v] = live[r] ? __ldg(qp + v * kLanesPerRow) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
            if (!live[r]) continue; // uniform across the row's lane group
            float acc[kVecs][8];
#pragma unroll
            for (int v = 0; v < kVecs; ++v)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[v][e] = 0.0f;
            float m = -INFINITY, l = 0.0f;
            const int64_t base = (static_cast<int64_t>(chunk[r]) * a.n_cam * a.heads + head[r]) * kD;
            for (int j = 0; j < a.n_cam; ++j) {
                const int64_t off = base + static_cast<int64_t>(j) * a.heads * kD;
                const uint4* kp = reinterpret_cast<const uint4*>(a.k_cam + off) + sub;
                float d = 0.0f;
#pragma unroll
                for (int v = 0; v < kVecs; ++v) {
                    float q[8], k[8];
                    bf16x8_to_f32(qv[r][v], q);
                    bf16x8_to_f32(__ldg(kp + v * kLanesPerRow), k);
#pragma unroll
                    for (int e = 0; e < 8; ++e) d = fmaf(q[e], k[e], d);
                }
#pragma unroll
                for (int o = kLanesPerRow / 2; o > 0; o >>= 1) d += __shfl_xor_sync(mask, d, o);
                const float s = d * a.scale_log2;
                const float m_new = fmaxf(m, s);
                const float corr = exp2f(m - m_new);
                const float p = exp2f(s - m_new);
                l = fmaf(l, corr, p);
                const uint4* vp = reinterpret_cast<const uint4*>(a.v_cam + off) + sub;
#pragma unroll
                for (int v = 0; v < kVecs; ++v) {
                    float vv[8];
                    bf16x8_to_f32(__ldg(vp + v * kLanesPerRow), vv);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[v][e] = fmaf(acc[v][e], corr, p * vv[e]);
                }
                m = m_new;
            }
            const float inv = 1.0f / l;
            uint4* op = reinterpret_cast<uint4*>(a.out + tok[r] * a.out_stride + head[r] * kD) + sub;
#pragma unroll
            for (int v = 0; v < kVecs; ++v) {
                uint4 o;
                o.x = pack_bf16x2(acc[v][0] * inv, acc[v][1] * inv);
                o.y = pack_bf16x2(acc[v][2] * inv, acc[v][3] * inv);
                o.z = pack_bf16x2(acc[v][4] * inv, acc[v][5] * inv);
                o.w = pack_bf16x2(acc[v][6] * inv, acc[v][7] * inv);
                op[v * kLanesPerRow] = o;
            }
        }
    }
}

} // namespace

cudaError_t launch_camera_attn(const CamArgs& a, cudaStream_t s) {
    // one wave of resident blocks (SM count x blocks per SM the registers allow)
    static const int64_t wave = [] {
        int dev = 0, sms = 148, per_sm = 4;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, camera_attn_kernel, kThreads, 0) != cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
        return static_cast<int64_t>(sms) * per_sm;
    }();
    const int64_t need = (a.rows + kGroups - 1) / kGroups;
    const int grid = static_cast<int>(need < wave ? need : wave);
    camera_attn_kernel<<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

} // namespace nomas
