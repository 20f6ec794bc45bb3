// HBM-bound kernels of the cache path:
//  * commit_kernel: RoPE(K) -> per-(token, head) INT8 quantisation (or BF16
//    rounding) -> write into the ring-buffer cache; V is quantised unrotated.
//    (Hy-Nomas model card, "Single-GPU Low-Memory Inference": INT8 KV storage
//    and an 18-latent-frame history budget; "Segment-Autoregressive Diffusion
//    Transformer": cached keys/values of earlier segments, 3D RoPE.)
//  * prep_kernel: RoPE of the current segment's Q and K, BF16 out, relayout
//    token-major -> head-major for the attention kernel's TMA loads.
//
// Work split: a half-warp owns one (token, head) row of 128 elements at a
// time; each lane moves 16 bytes (8 BF16 = 4 RoPE pairs) with one 128-bit load
// per tensor, marked evict-first (each input byte is read once; kept out of
// L1, it leaves room there for the RoPE rows every task reads). The 16 lanes of a row fall into exactly one RoPE axis block each
// (lanes 0-1: t, 2-8: h, 9-15: w). In the commit a warp walks the heads of one
// token (or of a group of its heads), so position, RoPE coefficients and ring
// slot are set up once per token; every row write is one full 128-byte
// (codes) or 256-byte (BF16) run. The RoPE tables arrive as launch arguments
// and are staged once per block into shared memory; the grid is persistent
// (two blocks per SM) so the staging is paid a few hundred times, not per row.
//
// Commit arithmetic is fixed bit for bit: products and fused multiply-adds
// use the _rn intrinsics (no contraction freedom), the scale is an IEEE
// division absmax / 127, codes are round-half-even of an IEEE division.
#include "nomas_div127.cuh"
#include "nomas_f16.cuh"
#include "nomas_internal.h"
#include "nomas_ptx.cuh"

#include <cuda_bf16.h>

#include <mutex>

namespace nomas {

namespace {

constexpr int kThreads = 512;

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t rne_bf16x2(float lo, float hi) {
    // round-half-even to BF16 of two finite fp32 values, packed (lo in bits 0-15)
    uint32_t a = __float_as_uint(lo), b = __float_as_uint(hi);
    a = (a + 0x7FFFu + ((a >> 16) & 1u)) >> 16;
    b = (b + 0x7FFFu + ((b >> 16) & 1u)) >> 16;
    return a | (b << 16);
}

// Spatial RoPE rows of up to kRopeConfigs configurations per device, uploaded
// once each by rope_hw_device (host code below).
__device__ __align__(16) float2 g_rope_hw[kRopeConfigs][NOMAS_MAX_GRID_HW][kHWPairs];

// cos/sin of the 4 pairs a lane owns (pairs 4*l .. 4*l+3 of the head): 32
// contiguous bytes of one table row -- the frame's t row (a launch argument)
// for lanes 0-1, the h row for lanes 2-8, the w row for lanes 9-15 (device
// memory, through L1: the rows of a half-warp are contiguous). Spatial rows
// are 224 B and the in-row offsets multiples of 32 B, so both loads are
// aligned 16-byte loads; lanes 0-1 load a valid spatial address too and keep
// the t row, so the half-warp does not diverge around the loads.
template <class Tab>
__device__ __forceinline__ void lane_coeffs(int l, int frame, int hh, int ww, int grid_h, const Tab& tab,
                                            const float2* hw, float2 (&cs)[4]) {
    const float2* src = hw + (l < 9 ? hh * kHWPairs + (l < 2 ? 0 : 4 * l - kTPairs)
                                    : (grid_h + ww) * kHWPairs + (4 * l - kTPairs - kHWPairs));
    float4 a = __ldg(reinterpret_cast<const float4*>(src));
    float4 b = __ldg(reinterpret_cast<const float4*>(src) + 1);
    if (l < 2) {
        const float2* t = &tab.t[frame][4 * l];
        a = make_float4(t[0].x, t[0].y, t[1].x, t[1].y);
        b = make_float4(t[2].x, t[2].y, t[3].x, t[3].y);
    }
    cs[0] = make_float2(a.x, a.y);
    cs[1] = make_float2(a.z, a.w);
    cs[2] = make_float2(b.x, b.y);
    cs[3] = make_float2(b.z, b.w);
}

// y0 = fma(x0, c, -rn(x1*s)), y1 = fma(x0, s, rn(x1*c)) on 4 pairs.
__device__ __forceinline__ void rotate8(const uint4 x, const float2 (&cs)[4], float (&y)[8]) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float x0 = bf16lo(w[i]), x1 = bf16hi(w[i]);
        const float c = cs[i].x, s = cs[i].y;
        y[2 * i] = __fmaf_rn(x0, c, -__fmul_rn(x1, s));
        y[2 * i + 1] = __fmaf_rn(x0, s, __fmul_rn(x1, c));
    }
}

__device__ __forceinline__ void unpack8(const uint4 x, float (&y)[8]) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        y[2 * i] = bf16lo(w[i]);
        y[2 * i + 1] = bf16hi(w[i]);
    }
}

// INT8 code of x for the row scale `scale`: the byte of
// round-half-even(rn(x / scale)), the IEEE quotient's rounding. `inv` is the
// hardware reciprocal approximation of scale (rcp.approx, at most 1 ulp off):
// x * inv lies within 1.5 * 2^-23 relative, i.e. 1.5 * 2^-16 absolute
// (|x / scale| < 128), of the exact quotient, and the IEEE quotient within
// 2^-17; the two can round to different integers only when a half-integer
// lies between them. Away from half-integers (farther than 2^-14) the cheap
// product decides; next to one -- or when the product is not finite, as for a
// subnormal scale whose reciprocal overflows -- the exact division does.
// Rounding to an integer uses the sum with 1.5 * 2^23: in [2^23, 2^24) the
// fp32 grid is the integers, so the add rounds half to even, and the low byte
// of the sum's bit pattern is the code in two's complement.
// |x / scale| <= 127 (1 + 3 * 2^-24) < 127.5, so the code never needs clamping
// to [-127, 127].
__device__ __forceinline__ uint32_t quant_word(float x, float scale, float inv) {
    constexpr float kMagic = 12582912.0f; // 1.5 * 2^23
    const float q = __fmul_rn(x, inv);
    float t = __fadd_rn(q, kMagic);
    const float f = __fsub_rn(q, __fsub_rn(t, kMagic)); // q - rint(q), exact; NaN if q is not finite
    if (!(fabsf(f) <= 0.5f - 6.103515625e-05f)) t = __fadd_rn(__fdiv_rn(x, scale), kMagic);
    return __float_as_uint(t);
}

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Half-warp INT8 quantisation of one row: returns 8 packed codes of this lane
// and the row scale. Both half-warps of a warp must call it together. The
// fast path of quant_word runs on packed pairs for all 8 values; one test of
// the largest distance to the nearest integer (and of the reciprocal being
// finite, which makes every product finite) sends the lane to the exact
// per-value path when any value needs it. Packed fp32 operations round each
// half exactly as the scalar ones do.
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ uint2 quantize8(const float (&y)[8], float& scale_out) {
    float amax = max3f(max3f(fabsf(y[0]), fabsf(y[1]), fabsf(y[2])), max3f(fabsf(y[3]), fabsf(y[4]), fabsf(y[5])),
                       fmaxf(fabsf(y[6]), fabsf(y[7])));
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off, 16));
    if (amax == 0.0f) {
        scale_out = 0.0f;
        return make_uint2(0u, 0u);
    }
    const float scale = div127_rn(amax);
    const float inv = rcp_approx(scale);
    scale_out = scale;
    constexpr float kMagic = 12582912.0f; // 1.5 * 2^23
    constexpr float kNear = 0.5f - 6.103515625e-05f;
    uint32_t w[8];
    float fmax_abs = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 q = __fmul2_rn(make_float2(y[2 * i], y[2 * i + 1]), make_float2(inv, inv));
        const float2 t = __fadd2_rn(q, make_float2(kMagic, kMagic));
        const float2 r = __fadd2_rn(t, make_float2(-kMagic, -kMagic));
        const float2 f = __ffma2_rn(r, make_float2(-1.0f, -1.0f), q); // q - rint(q), exact
        fmax_abs = max3f(fmax_abs, fabsf(f.x), fabsf(f.y));
        w[2 * i] = __float_as_uint(t.x);
        w[2 * i + 1] = __float_as_uint(t.y);
    }
    if (!(fmax_abs <= kNear && inv <= 3.4028234663852886e38f)) {
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = quant_word(y[i], scale, inv);
    }
    // low bytes of w[0..7], in order
    uint2 r;
    r.x = __byte_perm(__byte_perm(w[0], w[1], 0x0040u), __byte_perm(w[2], w[3], 0x0040u), 0x5410u);
    r.y = __byte_perm(__byte_perm(w[4], w[5], 0x0040u), __byte_perm(w[6], w[7], 0x0040u), 0x5410u);
    return r;
}

// At most 64 registers a thread, so that the persistent grid (two blocks per
// SM) is resident in one wave.
template <bool kGrouped, bool kInt8, int kF, int kL>
__global__ void __launch_bounds__(kThreads, 2) commit_kernel(const __grid_constant__ CommitArgs a,
                                                          const __grid_constant__ CommitLayersT<kL> L,
                                                          const __grid_constant__ RopeTabT<kF> tab) {
    // A warp task is one layer's token and a group of `head_group` of its heads; the
    // two half-warps walk the group's heads h = g0 + half, g0 + half + 2, ...
    // (one (token, head) row per half-warp per step). Position, RoPE
    // coefficients and ring slot depend only on the token, so they are set up
    // once per task. The next row's K and V are loaded while the current one
    // is processed, across task boundaries too. Large commits use all heads
    // per task; a commit with too few tokens to fill the GPU splits them.
    // All index math is 32-bit (rows of one launch < 2^31).
    const int lane = threadIdx.x & 31;
    const int half = lane >> 4;
    const int l = lane & 15;
    const uint32_t groups = kGrouped ? a.div_groups.d : 1u;
    const uint32_t layer_tasks = static_cast<uint32_t>(a.n_frames) * a.tpf * groups;
    const uint32_t tasks = layer_tasks * static_cast<uint32_t>(a.n_layers);
    const uint32_t warps = gridDim.x * (kThreads / 32);
    const int steps = ((kGrouped ? a.head_group : a.heads) + 1) >> 1; // rows per half-warp per task
    const int64_t tok0 = static_cast<int64_t>(a.in_frame0) * a.tpf;
    auto row_ptr = [&](const uint16_t* base, uint32_t tok, int h) {
        return reinterpret_cast<const uint4*>(base + (tok0 + tok) * a.token_stride + h * kD + l * 8);
    };
    // layer and token of a task, and the first head of its group
    auto task_token = [&](uint32_t t, uint32_t& ly, uint32_t& tk) {
        ly = a.n_layers > 1 ? fast_div(t, a.div_layer_tasks) : 0u;
        t -= ly * layer_tasks;
        if (!kGrouped) {
            tk = t;
            return 0;
        }
        tk = fast_div(t, a.div_groups);
        return static_cast<int>(t - tk * groups) * a.head_group;
    };
    uint32_t task = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    uint4 kx = make_uint4(0, 0, 0, 0), vx = kx;
    if (task < tasks) {
        uint32_t ly, tk;
        const int h0 = min(task_token(task, ly, tk) + half, a.heads - 1); // out-of-range heads load a valid row, not stored
        kx = __ldcs(row_ptr(L.l[ly].k, tk, h0));
        vx = __ldcs(row_ptr(L.l[ly].v, tk, h0));
    }
    for (; task < tasks; task += warps) {
        uint32_t layer, tok;
        const int g0 = task_token(task, layer, tok);
        const CommitLayer& P = L.l[layer];
        const int g1 = kGrouped ? min(g0 + a.head_group, a.heads) : a.heads; // heads [g0, g1) in this task
        const uint32_t fi = fast_div(tok, a.div_tpf);
        const uint32_t rif = tok - fi * a.tpf;
        const uint32_t hh = fast_div(rif, a.div_gw);
        const uint32_t ww = rif - hh * a.grid_w;
        float2 cs[4];
        lane_coeffs(l, fi, hh, ww, a.grid_h, tab, a.hw, cs);
        // slot of frame fi: ring slots advance with the frame (fi < window within a launch)
        int64_t slot;
        if (a.window > 0) {
            const int32_t s0 = a.slot0 + static_cast<int32_t>(fi);
            slot = s0 >= a.window ? s0 - a.window : s0;
        } else {
            slot = a.abs_frame0 + fi;
        }
        const int64_t row0 = slot * a.tpf + rif; // row of head 0; head h adds h * cap_tok
        const uint32_t task_next = task + warps;
        // pointers of this half-warp's first head; each step moves two heads on
        const int hf = g0 + half;
        const int64_t in_off = (tok0 + tok) * a.token_stride + static_cast<int64_t>(hf) * kD + l * 8;
        const uint4* kp = reinterpret_cast<const uint4*>(P.k + in_off);
        const uint4* vp = reinterpret_cast<const uint4*>(P.v + in_off);
        const int64_t row_f = static_cast<int64_t>(hf) * a.cap_tok + row0;
        const int64_t out_step = 2 * a.cap_tok; // rows between a half-warp's steps
        for (int j = 0; j < steps; ++j) {
            const int h = hf + 2 * j;
            const bool valid = h < g1;
            // next row of this half-warp: the following head, or the first of the next task
            uint4 kn = kx, vn = vx;
            if (j + 1 < steps) {
                if (h + 2 < a.heads) {
                    kn = __ldcs(kp + (j + 1) * (2 * kD / 8));
                    vn = __ldcs(vp + (j + 1) * (2 * kD / 8));
                }
            } else if (task_next < tasks) {
                uint32_t ln, tn;
                const int hn = min(task_token(task_next, ln, tn) + half, a.heads - 1);
                kn = __ldcs(row_ptr(L.l[ln].k, tn, hn));
                vn = __ldcs(row_ptr(L.l[ln].v, tn, hn));
            }
            float ky[8], vy[8];
            rotate8(kx, cs, ky);
            unpack8(vx, vy);
            const int64_t row = row_f + j * out_step;
            if (kInt8) {
                float ks, vs;
                const uint2 kc = quantize8(ky, ks);
                const uint2 vc = quantize8(vy, vs);
                if (valid) {
                    *reinterpret_cast<uint2*>(static_cast<int8_t*>(P.ck) + row * kD + l * 8) = kc;
                    *reinterpret_cast<uint2*>(static_cast<int8_t*>(P.cv) + row * kD + l * 8) = vc;
                    if (l == 0) {
                        P.cks[row] = ks;
                        P.cvs[row] = vs;
                    }
                }
            } else if (valid) {
                uint4 ko;
                ko.x = rne_bf16x2(ky[0], ky[1]);
                ko.y = rne_bf16x2(ky[2], ky[3]);
                ko.z = rne_bf16x2(ky[4], ky[5]);
                ko.w = rne_bf16x2(ky[6], ky[7]);
                *reinterpret_cast<uint4*>(static_cast<uint16_t*>(P.ck) + row * kD + l * 8) = ko;
                *reinterpret_cast<uint4*>(static_cast<uint16_t*>(P.cv) + row * kD + l * 8) = vx;
            }
            kx = kn;
            vx = vn;
        }
    }
}

template <int kF>
__global__ void __launch_bounds__(kThreads) prep_kernel(const __grid_constant__ PrepArgs a,
                                                        const __grid_constant__ RopeTabT<kF> tab) {
    // the attention kernel of the call (which waits for this one before it
    // reads anything) may start launching right away
    grid_dep_launch();
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < a.n_counters; i += blockDim.x) a.counters[i] = 0u;

    const int lane = threadIdx.x & 31;
    const int l = lane & 15;
    const uint32_t rows = static_cast<uint32_t>(a.tok1 - a.tok0) * a.heads;
    const uint32_t halves = gridDim.x * (kThreads / 16);
    for (uint32_t r = blockIdx.x * (kThreads / 16) + (threadIdx.x >> 4); r < rows; r += halves) {
        const uint32_t tq = fast_div(r, a.div_heads);
        const int tok = a.tok0 + static_cast<int>(tq);
        const int h = static_cast<int>(r - tq * a.heads);
        const int64_t in_off = static_cast<int64_t>(tok) * a.token_stride + h * kD + l * 8;
        const uint4 qx = __ldcs(reinterpret_cast<const uint4*>(a.q + in_off));
        const uint4 kx = __ldcs(reinterpret_cast<const uint4*>(a.k + in_off));
        uint4 qo = qx, ko = kx;
        if (tok < a.nv) {
            const uint32_t fa = fast_div(static_cast<uint32_t>(tok), a.div_tpf);
            const int fi = static_cast<int>(fa) - a.frame0;
            const uint32_t rif = static_cast<uint32_t>(tok) - fa * a.tpf;
            const uint32_t hh = fast_div(rif, a.div_gw);
            float2 cs[4];
            lane_coeffs(l, fi, hh, rif - hh * a.grid_w, a.grid_h, tab, a.hw, cs);
            float qy[8], ky[8];
            rotate8(qx, cs, qy);
            rotate8(kx, cs, ky);
            qo.x = rne_bf16x2(qy[0], qy[1]);
            qo.y = rne_bf16x2(qy[2], qy[3]);
            qo.z = rne_bf16x2(qy[4], qy[5]);
            qo.w = rne_bf16x2(qy[6], qy[7]);
            ko.x = rne_bf16x2(ky[0], ky[1]);
            ko.y = rne_bf16x2(ky[2], ky[3]);
            ko.z = rne_bf16x2(ky[4], ky[5]);
            ko.w = rne_bf16x2(ky[6], ky[7]);
        }
        const int64_t out_off = (static_cast<int64_t>(h) * a.nq + tok) * kD + l * 8;
        *reinterpret_cast<uint4*>(a.qt + out_off) = qo;
        *reinterpret_cast<uint4*>(a.kt + out_off) = ko;
    }
}

// INT8 caches: RoPE of Q and K in fp32 to FP16 operands with power-of-two
// exponents (nomas_f16.cuh), and every tile record of the attention call.
// A block of 256 threads takes one (128-token tile, head) task; half-warp g of
// the block owns rows g, g + 16, ..., g + 112 of the tile. Each Q row gets its
// own exponent (a half-warp reduction) and is written at once. K takes two
// passes: the first finds the tile's maximum (a block reduction), the second
// loads the rows again (from L1) and writes them with the tile's exponent; the
// RoPE products are recomputed, bit for bit the same. Launch chunks start at
// multiples of 128 frames, so a tile never spans two launches. The launch
// with tok0 == 0 also writes the records of the cache tiles (a warp per tile:
// the maxima of its 128 K and V scales).
constexpr int kPrep16Threads = 256;
constexpr int kPrep16Rows = 128 / (kPrep16Threads / 16); // rows per half-warp

template <int kF>
__global__ void __launch_bounds__(kPrep16Threads, 3) prep16_kernel(const __grid_constant__ PrepArgs a,
                                                                const __grid_constant__ RopeTabT<kF> tab) {
    grid_dep_launch();
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < a.n_counters; i += blockDim.x) a.counters[i] = 0u;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int ttot = a.tiles_c + a.tiles_q;

    // ---- cache tile records
    const int nwarps = gridDim.x * (kPrep16Threads / 32);
    for (int task = blockIdx.x * (kPrep16Threads / 32) + warp; task < a.te_cache_tasks; task += nwarps) {
        const int h = task / a.tiles_c;
        const int T = task - h * a.tiles_c;
        float mk = 0.0f, mv = 0.0f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int key = T * 128 + q * 32 + lane;
            if (key < a.nc) {
                const int64_t g = static_cast<int64_t>(h) * a.cap_tok + key;
                mk = fmaxf(mk, __ldg(a.ksc + g));
                mv = fmaxf(mv, __ldg(a.vsc + g));
            }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            mk = fmaxf(mk, __shfl_xor_sync(0xFFFFFFFFu, mk, off));
            mv = fmaxf(mv, __shfl_xor_sync(0xFFFFFFFFu, mv, off));
        }
        if (lane == 0)
            a.te[static_cast<int64_t>(h) * ttot + T] =
                tile_record(pow2_exponent(mk, kTopCode), pow2_exponent(mv, kTopCode));
    }

    // ---- current tiles
    __shared__ float red[kPrep16Threads / 32];
    const int l = lane & 15;
    const int g = threadIdx.x >> 4;
    const int T0 = a.tok0 / 128;
    const int T1 = (a.tok1 + 127) / 128;
    const int tasks = (T1 - T0) * a.heads;
    // RoPE of one row's 8 elements owned by this lane (video rows), or the
    // elements themselves (text rows)
    auto rope8 = [&](int tok, uint4 x, float (&y)[8]) {
        if (tok < a.nv) {
            const uint32_t fa = fast_div(static_cast<uint32_t>(tok), a.div_tpf);
            const int fi = static_cast<int>(fa) - a.frame0;
            const uint32_t rif = static_cast<uint32_t>(tok) - fa * a.tpf;
            const uint32_t hh = fast_div(rif, a.div_gw);
            float2 cs[4];
            lane_coeffs(l, fi, hh, rif - hh * a.grid_w, a.grid_h, tab, a.hw, cs);
            rotate8(x, cs, y);
        } else {
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                y[2 * i] = bf16lo(w[i]);
                y[2 * i + 1] = bf16hi(w[i]);
            }
        }
    };
    for (int task = blockIdx.x; task < tasks; task += gridDim.x) {
        const int T = T0 + task / a.heads;
        const int h = task - (task / a.heads) * a.heads;
        const int tok0 = T * 128 + g;
        float kmax = 0.0f;
        // pass 1 in two batches of rows (their loads in flight together)
#pragma unroll
        for (int b0 = 0; b0 < kPrep16Rows; b0 += kPrep16Rows / 2) {
            uint4 qx[kPrep16Rows / 2], kx[kPrep16Rows / 2];
#pragma unroll
            for (int rr = 0; rr < kPrep16Rows / 2; ++rr) {
                const int tok = tok0 + 16 * (b0 + rr);
                qx[rr] = kx[rr] = make_uint4(0u, 0u, 0u, 0u);
                if (tok < a.tok1) {
                    const int64_t in_off = static_cast<int64_t>(tok) * a.token_stride + h * kD + l * 8;
                    qx[rr] = __ldcs(reinterpret_cast<const uint4*>(a.q + in_off));
                    kx[rr] = __ldg(reinterpret_cast<const uint4*>(a.k + in_off));
                }
            }
#pragma unroll
            for (int rr = 0; rr < kPrep16Rows / 2; ++rr) {
                const int tok = tok0 + 16 * (b0 + rr);
                if (tok < a.tok1) {
                    float qy[8], ky[8];
                    rope8(tok, qx[rr], qy);
                    rope8(tok, kx[rr], ky);
                    float qm = 0.0f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        qm = fmaxf(qm, fabsf(qy[i]));
                        kmax = fmaxf(kmax, fabsf(ky[i]));
                    }
                    // rows of a half-warp are valid together: the shuffles stay in it
#pragma unroll
                    for (int off = 8; off >= 1; off >>= 1)
                        qm = fmaxf(qm, __shfl_xor_sync(0xFFFFu << (lane & 16), qm, off));
                    const int ea = pow2_exponent(qm, kTopFloat);
                    const float f = exp2_int(-ea);
                    const int64_t out_off = (static_cast<int64_t>(h) * a.nq + tok) * kD + l * 8;
                    *reinterpret_cast<uint4*>(a.qt + out_off) =
                        make_uint4(pack_f16x2(qy[0] * f, qy[1] * f), pack_f16x2(qy[2] * f, qy[3] * f),
                                   pack_f16x2(qy[4] * f, qy[5] * f), pack_f16x2(qy[6] * f, qy[7] * f));
                    if (l == 0) a.qs[static_cast<int64_t>(h) * a.nq + tok] = exp2_int(ea);
                }
            }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) kmax = fmaxf(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, off));
        if (lane == 0) red[warp] = kmax;
        __syncthreads();
        float tmax = red[0];
#pragma unroll
        for (int i = 1; i < kPrep16Threads / 32; ++i) tmax = fmaxf(tmax, red[i]);
        const int eb = pow2_exponent(tmax, kTopFloat);
        const float f = exp2_int(-eb);
#pragma unroll
        for (int rr = 0; rr < kPrep16Rows; ++rr) {
            const int tok = tok0 + 16 * rr;
            if (tok < a.tok1) {
                const int64_t in_off = static_cast<int64_t>(tok) * a.token_stride + h * kD + l * 8;
                float ky[8];
                rope8(tok, __ldcs(reinterpret_cast<const uint4*>(a.k + in_off)), ky);
                const int64_t out_off = (static_cast<int64_t>(h) * a.nq + tok) * kD + l * 8;
                *reinterpret_cast<uint4*>(a.kt + out_off) =
                    make_uint4(pack_f16x2(ky[0] * f, ky[1] * f), pack_f16x2(ky[2] * f, ky[3] * f),
                               pack_f16x2(ky[4] * f, ky[5] * f), pack_f16x2(ky[6] * f, ky[7] * f));
            }
        }
        if (threadIdx.x == 0) a.te[static_cast<int64_t>(h) * ttot + a.tiles_c + T] = tile_record(eb, 0);
        __syncthreads(); // red[] is reused by the next task
    }
}

int grid_for(int64_t work_items, int items_per_block) {
    // SM count of the first device that launches (every device of this library is a B200);
    // a function-local static is initialised once, thread-safely
    static const int sms = [] {
        int dev = 0, n = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        return n;
    }();
    // a persistent grid: two blocks of 512 threads per SM, grid-stride loops
    int64_t want = (work_items + items_per_block - 1) / items_per_block;
    const int64_t cap = static_cast<int64_t>(sms) * 2;
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    return static_cast<int>(want);
}

} // namespace

// One table per (device, configuration): the host keeps which configuration
// each slot of g_rope_hw holds on each device; a slot is written once (a
// blocking copy, before its first kernel) and never changes afterwards.
cudaError_t rope_hw_device(const RopeHW& host, float theta, int grid_h, int grid_w, const float2** dev) {
    struct Key {
        float theta;
        int gh, gw;
    };
    struct Table {
        std::mutex mu;
        Key keys[64][kRopeConfigs];
        int used[64] = {};
        const float2* base[64] = {};
    };
    static Table t;
    int d = 0;
    cudaError_t e = cudaGetDevice(&d);
    if (e != cudaSuccess) return e;
    if (d < 0 || d >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(t.mu);
    if (!t.base[d]) {
        void* p = nullptr;
        if ((e = cudaGetSymbolAddress(&p, g_rope_hw)) != cudaSuccess) return e;
        t.base[d] = static_cast<const float2*>(p);
    }
    const size_t slot_elems = static_cast<size_t>(NOMAS_MAX_GRID_HW) * kHWPairs;
    for (int i = 0; i < t.used[d]; ++i) {
        const Key& k = t.keys[d][i];
        if (k.theta == theta && k.gh == grid_h && k.gw == grid_w) {
            *dev = t.base[d] + i * slot_elems;
            return cudaSuccess;
        }
    }
    if (t.used[d] == kRopeConfigs) return cudaErrorMemoryAllocation;
    const int i = t.used[d];
    const size_t bytes = sizeof(float2) * kHWPairs * static_cast<size_t>(grid_h + grid_w);
    if ((e = cudaMemcpyToSymbol(g_rope_hw, host.hw, bytes, i * slot_elems * sizeof(float2))) != cudaSuccess) return e;
    t.keys[d][i] = Key{theta, grid_h, grid_w};
    t.used[d] = i + 1;
    *dev = t.base[d] + i * slot_elems;
    return cudaSuccess;
}

template <int kF, int kL>
void commit_variant(const CommitArgs& a, int grid, const CommitLayersT<kL>& L, const RopeTabT<kF>& tab,
                    cudaStream_t s) {
    if (a.head_group < a.heads) {
        if (a.int8_mode) commit_kernel<true, true, kF, kL><<<grid, kThreads, 0, s>>>(a, L, tab);
        else commit_kernel<true, false, kF, kL><<<grid, kThreads, 0, s>>>(a, L, tab);
    } else {
        if (a.int8_mode) commit_kernel<false, true, kF, kL><<<grid, kThreads, 0, s>>>(a, L, tab);
        else commit_kernel<false, false, kF, kL><<<grid, kThreads, 0, s>>>(a, L, tab);
    }
}

cudaError_t launch_commit(const CommitArgs& a_in, const CommitLayers& layers, const RopeTab& tab, cudaStream_t s) {
    // heads per warp task: all of a token's heads when there are enough tokens
    // to give every resident warp (two 512-thread blocks per SM) two tasks, else
    // halves of that, down to 2, so that small commits still spread over the
    // GPU (a 3-frame commit of 16 heads: 4 heads per task)
    CommitArgs a = a_in;
    const int64_t tokens = static_cast<int64_t>(a.n_frames) * a.tpf * a.n_layers;
    const int64_t want = 2ll * 148 * 2 * (kThreads / 32);
    int hg = a.heads;
    while (hg > 2 && tokens * ((a.heads + hg - 1) / hg) < want) hg = (hg + 1) / 2;
    a.head_group = hg;
    a.div_groups = make_fastdiv(static_cast<uint32_t>((a.heads + hg - 1) / hg));
    const int64_t layer_tasks = static_cast<int64_t>(a.n_frames) * a.tpf * a.div_groups.d;
    a.div_layer_tasks = make_fastdiv(static_cast<uint32_t>(layer_tasks));
    const int grid = grid_for(layer_tasks * a.n_layers, kThreads / 32);
    if (a.n_frames <= kSmallFrames && a.n_layers <= kSmallLayers) {
        RopeTabT<kSmallFrames> t{};
        CommitLayersT<kSmallLayers> L{};
        for (int f = 0; f < a.n_frames; ++f)
            for (int j = 0; j < kTPairs; ++j) t.t[f][j] = tab.t[f][j];
        for (int i = 0; i < a.n_layers; ++i) L.l[i] = layers.l[i];
        commit_variant(a, grid, L, t, s);
    } else {
        commit_variant(a, grid, layers, tab, s);
    }
    return cudaGetLastError();
}

cudaError_t launch_prep(const PrepArgs& a, const RopeTab& tab, cudaStream_t s) {
    const int64_t rows = static_cast<int64_t>(a.tok1 - a.tok0) * a.heads;
    const bool f16 = a.te != nullptr;
    // FP16 form: one block per (tile, head) task, and enough blocks to give the
    // cache tile records a warp each (at most 16 blocks per SM: all resident)
    const int64_t tasks = static_cast<int64_t>((a.tok1 + 127) / 128 - a.tok0 / 128) * a.heads;
    int64_t want16 = tasks;
    const int64_t te_blocks = (a.te_cache_tasks + kPrep16Threads / 32 - 1) / (kPrep16Threads / 32);
    if (te_blocks > want16) want16 = te_blocks;
    if (want16 > 148 * 16) want16 = 148 * 16;
    if (want16 < 1) want16 = 1;
    const int grid = f16 ? static_cast<int>(want16) : grid_for(rows, kThreads / 16);
    const int block = f16 ? kPrep16Threads : kThreads;
    const int nv_frames = a.tok0 < a.nv ? (min(a.tok1, a.nv) - 1) / a.tpf - a.frame0 + 1 : 0;
    if (nv_frames <= kSmallFrames) {
        RopeTabT<kSmallFrames> t{};
        for (int f = 0; f < nv_frames; ++f)
            for (int j = 0; j < kTPairs; ++j) t.t[f][j] = tab.t[f][j];
        if (f16) prep16_kernel<kSmallFrames><<<grid, block, 0, s>>>(a, t);
        else prep_kernel<kSmallFrames><<<grid, kThreads, 0, s>>>(a, t);
    } else {
        if (f16) prep16_kernel<kMaxFramesPerLaunch><<<grid, block, 0, s>>>(a, tab);
        else prep_kernel<kMaxFramesPerLaunch><<<grid, kThreads, 0, s>>>(a, tab);
    }
    return cudaGetLastError();
}

} // namespace nomas
