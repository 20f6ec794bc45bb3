// Segment-causal joint attention on sm_100a tensor cores.
//
// What it computes (Hy-Nomas model card, "Segment-Autoregressive Diffusion
// Transformer"; blog "Segment-wise causal joint attention"): for each head
// and each query token of the current segment, softmax attention over the
// visible cached tokens of earlier segments followed by every token of the
// current segment (no mask inside a segment; causality across segments is
// structural: later segments are never in the cache). An INT8 cache is
// attended to in BF16 (model card, "Single-GPU Low-Memory Inference": INT8 KV
// storage, BF16 attention computation): K as its integer codes, which BF16
// holds exactly, with the per-key K scale applied to the scores in the
// softmax; V as code * scale rounded to BF16.
//
// Three forms (template parameter kMode):
//   kBf16   BF16 cache; every K/V tile arrives by TMA.
//   kWindow INT8 cache whose visible window dequant_window_kernel has written
//           to a BF16 copy once per call (K codes, V code * scale); tiles by
//           TMA, the K scales of each cache tile go into a coefficient ring.
//   kFused  INT8 cache converted in shared memory tile by tile by a filler
//           warpgroup (no copy: for workspaces too small to hold one).
//
// Structure of one CTA (one "unit" = two 128-row Q tiles of one head, and a
// contiguous range of 128-key KV tiles: cache tiles first, then the current
// segment's tiles):
//   warp 0      TMA producer: Q tiles once, then (kBf16, kWindow) every K/V
//               tile into a 2-stage ring; kWindow: the K coefficients
//   warp 1      TMEM allocator + tcgen05.mma issuer
//   warps 4-7   softmax warpgroup for Q tile 0 (one thread per query row)
//   warps 8-11  softmax warpgroup for Q tile 1
//   warps 12-15 kFused only: the one filler of the K/V ring. Cache tiles are
//               converted from codes and scales; current-segment tiles are
//               loaded by TMA. One filler in tile order keeps every parity
//               wait on the ring exact.
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each; the BF16
// probabilities P overwrite the first 64 columns of their S block and feed
// the P.V product straight from TMEM (A operand in tensor memory).
// MMA order per KV tile j: PV0(j-1) S0(j) | PV1(j-1) S1(j) -- while one
// softmax warpgroup exponentiates, the tensor core works for the other. The
// issuer waits for V(j-1) before PV0(j-1) and for K(j) only before S0(j).
// Online softmax in base 2 with lazy rescaling: the running reference max is
// raised only when a tile's max may exceed it by more than 8 (so P <= 256),
// and only then is O rescaled in TMEM.
// Split-KV: with splits > 1 each CTA leaves (O unnormalised, max, sum) in the
// workspace and counts itself in per unit; the last CTA of a unit to arrive
// merges the splits and writes the output (the partials are still in L2).
#include "nomas_internal.h"
#include "nomas_ptx.cuh"

#include <atomic>

namespace nomas {

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kStages = 2;
constexpr int kCoefSlots = 4;                 // ring of per-tile K coefficients (INT8 caches)
constexpr uint32_t kTileBytes = BM * kD * 2;  // one BF16 128x128 tile
constexpr uint32_t kHalfBytes = kTileBytes / 2;
constexpr float kRescaleThreshold = 8.0f;     // P <= 2^8 between rescales

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;                                // 2 tiles
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;           // kStages tiles
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;     // kStages tiles
constexpr uint32_t kOffCoef = kOffV + kStages * kTileBytes;  // kCoefSlots x 128 fp32
constexpr uint32_t kOffBound = kOffCoef + kCoefSlots * BN * 4; // kCoefSlots x 4 warps x (max, min)
constexpr uint32_t kOffBar = kOffBound + kCoefSlots * 4 * 8; // barriers
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;        // + alignment slack

// barrier slots (8 bytes each)
enum {
    B_QFULL = 0,
    B_KFULL = 1,                // + stage
    B_VFULL = B_KFULL + kStages,
    B_KEMPTY = B_VFULL + kStages,  // K and V stages are released separately: K as soon
    B_VEMPTY = B_KEMPTY + kStages, // as the S MMAs that read it are done, V after P.V
    B_SFULL = B_VEMPTY + kStages,  // + softmax warpgroup
    B_PFULL = B_SFULL + 2,
    B_OFULL = B_PFULL + 2,
    B_DRAIN = B_OFULL + 2,
    B_CFULL = B_DRAIN + 1,          // + coefficient slot: the filler wrote a tile's K coefficients
    B_CEMPTY = B_CFULL + kCoefSlots, // + coefficient slot: every softmax warp is done with them
    B_COUNT = B_CEMPTY + kCoefSlots
};
constexpr uint32_t kOffTmemSlot = B_COUNT * 8;
constexpr uint32_t kOffAbort = kOffTmemSlot + 8;
constexpr uint32_t kOffDqGo = kOffAbort + 4;
constexpr uint32_t kOffLast = kOffDqGo + 4;
static_assert(kOffLast + 4 <= 256, "barrier area overflow");
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

enum { kBf16 = 0, kWindow = 1, kFused = 2 };

// mbar_wait run by every lane of a converged warp; lane 0's outcome is
// broadcast so the warp leaves the wait converged.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, const WaitCtl& ctl) {
    const bool ok = mbar_wait(bar, parity, ctl);
    return __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
}

// How the MMA issuer issues: kWarp = the whole warp runs the loop and one
// elected lane issues each instruction; otherwise lane 0 alone runs it.
template <bool kWarp>
struct Issuer {
    static __device__ __forceinline__ void ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
        if (kWarp) mma_ss_warp(d, a, b, idesc, acc);
        else mma_ss(d, a, b, idesc, acc);
    }
    static __device__ __forceinline__ void ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
        if (kWarp) mma_ts_warp(d, a, b, idesc, acc);
        else mma_ts(d, a, b, idesc, acc);
    }
    static __device__ __forceinline__ void commit(uint32_t bar) {
        if (kWarp) mma_commit_warp(bar);
        else mma_commit(bar);
    }
    static __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, const WaitCtl& ctl) {
        return kWarp ? mbar_wait_warp(bar, parity, ctl) : mbar_wait(bar, parity, ctl);
    }
};

__device__ __forceinline__ int tile_valid(const AttnArgs& a, int t) {
    const int rem = (t < a.tiles_c) ? a.nc - t * BN : a.nq - (t - a.tiles_c) * BN;
    return rem < BN ? rem : BN;
}

// K-major SW128 descriptor of k-step kk (16 dims) of a 128x128 BF16 tile.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int kk) {
    return smem_desc(tile + (kk >> 2) * kHalfBytes + (kk & 3) * 32, 16, 1024, kSwizzle128B);
}
// MN-major SW128 descriptor of k-step kk (16 keys) of a 128-key V tile.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile, int kk) {
    return smem_desc(tile + kk * 2048, kHalfBytes, 1024, kSwizzle128B);
}
// The start address sits in the low 14 bits of a descriptor in 16-byte units;
// shared addresses stay below 256 KB, so a k-step's descriptor is the tile's
// k-step-0 descriptor plus the step's byte offset / 16 (no carry out of the
// field). The issuer builds the k-step-0 descriptors once and adds these.
__host__ __device__ constexpr uint64_t kstep_kmajor(int kk) {
    return static_cast<uint64_t>(((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
}
__host__ __device__ constexpr uint64_t kstep_mnmajor(int kk) { return static_cast<uint64_t>((kk * 2048) >> 4); }

// 8 INT8 codes -> 8 BF16 values. A code c is read exactly as the float
// 2^23 + (c + 128) (the byte of c ^ 0x80 placed under the exponent of 2^23),
// minus 2^23 + 128. kScale: times the row scale in fp32, then rounded once to
// BF16; otherwise the integer itself, which BF16 holds exactly (at most 7
// significant bits), so its fp32 pattern's upper half is the BF16 pattern.
template <bool kScale>
__device__ __forceinline__ uint4 codes_to_bf16(uint2 w, float scale) {
    const uint32_t w0 = w.x ^ 0x80808080u, w1 = w.y ^ 0x80808080u;
    const float2 bias = make_float2(-8388736.0f, -8388736.0f);
    uint32_t out[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t src = q < 2 ? w0 : w1;
        const uint32_t b = (q & 1) * 2;
        float2 f = make_float2(__uint_as_float(__byte_perm(src, 0x4B000000u, 0x7540u + b)),
                               __uint_as_float(__byte_perm(src, 0x4B000000u, 0x7541u + b)));
        f = __fadd2_rn(f, bias);
        if (kScale) {
            f = __fmul2_rn(f, make_float2(scale, scale));
            out[q] = pack_bf16x2(f.x, f.y);
        } else {
            out[q] = __byte_perm(__float_as_uint(f.x), __float_as_uint(f.y), 0x7632u);
        }
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// 16 columns of 32-bit values from registers into TMEM (one row per thread).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]) : "memory");
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Maximum of one 128-key S row over its valid columns (kMask: columns >= vc
// ignored), raw scores. Eight independent accumulators keep the reduction off
// a single dependency chain.
template <bool kMask>
__device__ __forceinline__ float row_max(uint32_t t_s, int vc) {
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        uint32_t s[64];
        tmem_ld64(t_s + c * 64, s);
        float m[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) m[k] = mx;
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
            float x0 = __uint_as_float(s[e]), x1 = __uint_as_float(s[e + 1]);
            if (kMask) {
                x0 = (c * 64 + e < vc) ? x0 : -INFINITY;
                x1 = (c * 64 + e + 1 < vc) ? x1 : -INFINITY;
            }
            m[(e >> 1) & 7] = max3(m[(e >> 1) & 7], x0, x1);
        }
        mx = max3(max3(m[0], m[1], m[2]), max3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
        // keep this chunk's reduction ahead of the next TMEM load, so its 64
        // registers are dead before the next 64 arrive
        asm volatile("" : "+f"(mx));
    }
    return mx;
}

// row_max in 32-column pieces (fewer registers live: the kWindow softmax holds
// its tile's 128 coefficients in registers meanwhile).
__device__ __forceinline__ float row_max32(uint32_t t_s) {
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t s[32];
        tmem_ld32(t_s + c * 32, s);
        float m[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) m[k] = mx;
#pragma unroll
        for (int e = 0; e < 32; e += 2)
            m[(e >> 1) & 3] = max3(m[(e >> 1) & 3], __uint_as_float(s[e]), __uint_as_float(s[e + 1]));
        mx = fmaxf(max3(m[0], m[1], m[2]), m[3]);
        asm volatile("" : "+f"(mx));
    }
    return mx;
}

// Exact maximum of s_j * c_j over the valid columns of a row (used when the
// cheap bound of a tile is too loose to serve as the reference: keys of very
// different scales). Cold: run by a whole warp only when one of its rows needs it.
__device__ __noinline__ float row_max_scaled(uint32_t t_s, const float4* coef, int vc) {
    float mx = -INFINITY;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        uint32_t s[32];
        tmem_ld32(t_s + c * 32, s);
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
            const float4 k = coef[(c * 32 + e) >> 2];
            const float v[4] = {__uint_as_float(s[e]) * k.x, __uint_as_float(s[e + 1]) * k.y,
                                __uint_as_float(s[e + 2]) * k.z, __uint_as_float(s[e + 3]) * k.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) mx = (c * 32 + e + q < vc) ? fmaxf(mx, v[q]) : mx;
        }
    }
    return mx;
}

// 2^x of two values on the FMA pipe, so that part of a row's exponentials
// leave the MUFU unit (which alone would take as long as the tensor core needs
// for the row's two products). Range reduction x = n + f with n = rint(x)
// (the 1.5 * 2^23 shift puts n in the low mantissa bits of t) and f in
// [-1/2, 1/2]; 2^f by a cubic whose coefficients minimise the maximum relative
// error on that interval (7.5e-5, well under the 2^-9 of the BF16 rounding of P
// that follows; fitted by tests/tools/exp2_poly_fit.py); 2^n by adding n to
// the exponent field (the shift by 23 keeps exactly the low 9 bits of t, i.e.
// n modulo 2^9). x is clamped below at -125 so the result stays normal
// (2^-125 in place of a smaller P, far under the BF16 resolution of the row).
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932608485221863f;
constexpr float kExp2C2 = 0.24261115491390228f;
constexpr float kExp2C3 = 0.05517221987247467f;
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
    x.x = fmaxf(x.x, -125.0f);
    x.y = fmaxf(x.y, -125.0f);
    const float2 t = __fadd2_rn(x, make_float2(12582912.0f, 12582912.0f));
    const float2 nf = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
    const float2 f = __ffma2_rn(nf, make_float2(-1.0f, -1.0f), x);
    float2 q = __ffma2_rn(f, make_float2(kExp2C3, kExp2C3), make_float2(kExp2C2, kExp2C2));
    q = __ffma2_rn(q, f, make_float2(kExp2C1, kExp2C1));
    q = __ffma2_rn(q, f, make_float2(kExp2C0, kExp2C0));
    return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

// Of every 8 column pairs of a full tile, kPoly take exp2_fma2 and the rest
// the MUFU ex2. In the kFused form the converting warps share the FMA pipe
// and issue slots of every SM sub-partition, so there all go to the MUFU.
constexpr int kExp2PolyPairs = 3;
constexpr int kExp2PolyPairsFused = 0;


// One 32-column chunk of an unmasked S row -> 16 packed BF16 P columns;
// x = s * c - m with c the scalar scale_log2, or with kCoef the tile's
// per-column coefficients (scale_log2 times the key's K scale), read from
// shared memory four at a time.
template <int kPoly, bool kCoef>
__device__ __forceinline__ void exp_chunk(const uint32_t (&s)[32], const float4* coef, float2 sl2x2, float2 negm,
                                          float2 (&acc)[4], uint32_t (&p)[16]) {
    float4 c4 = make_float4(sl2x2.x, sl2x2.x, sl2x2.x, sl2x2.x);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        if (kCoef && (e & 1) == 0) c4 = coef[e >> 1];
        const float2 cc = kCoef ? ((e & 1) ? make_float2(c4.z, c4.w) : make_float2(c4.x, c4.y)) : sl2x2;
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1])), cc, negm);
        float2 y;
        if ((e & 7) < kPoly)
            y = exp2_fma2(x);
        else
            y = make_float2(ex2_approx(x.x), ex2_approx(x.y));
        acc[e & 3] = __fadd2_rn(acc[e & 3], y);
        p[e] = pack_bf16x2(y.x, y.y);
    }
}

// P = 2^(s * c - m) of one full 128-key S row, written as packed BF16 pairs
// over the first 64 columns of the row's S block; returns the fp32 row sum
// (four independent packed accumulators). The TMEM loads are software
// pipelined: chunk c + 1 is in flight while chunk c is exponentiated. P chunk c
// lands on columns [16c, 16c + 16), all of which were read with chunks <= c.
template <int kPoly, bool kCoef>
__device__ __forceinline__ float row_exp_store_full(uint32_t t_s, const float4* coef, float sl2, float m) {
    const float2 sl2x2 = make_float2(sl2, sl2);
    const float2 negm = make_float2(-m, -m);
    float2 acc[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.0f, 0.0f);
    uint32_t sa[32], sb[32], p[16];
    tmem_ld32_issue(t_s, sa);
    tmem_ld32_wait(sa);
    tmem_ld32_issue(t_s + 32, sb);
    exp_chunk<kPoly, kCoef>(sa, coef, sl2x2, negm, acc, p);
    tmem_st16(t_s, p);
    tmem_ld32_wait(sb);
    tmem_ld32_issue(t_s + 64, sa);
    exp_chunk<kPoly, kCoef>(sb, coef + 8, sl2x2, negm, acc, p);
    tmem_st16(t_s + 16, p);
    tmem_ld32_wait(sa);
    tmem_ld32_issue(t_s + 96, sb);
    exp_chunk<kPoly, kCoef>(sa, coef + 16, sl2x2, negm, acc, p);
    tmem_st16(t_s + 32, p);
    tmem_ld32_wait(sb);
    exp_chunk<kPoly, kCoef>(sb, coef + 24, sl2x2, negm, acc, p);
    tmem_st16(t_s + 48, p);
    const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
    return t.x + t.y;
}

// Full-tile exp pass with per-column coefficients read from shared memory, in
// 16-column chunks (chunk q + 1 of S loads from TMEM while chunk q is
// exponentiated): fewer registers live than the 32-column form, which with
// its coefficients would not fit the softmax warps' registers.
template <int kPoly>
__device__ __forceinline__ void exp_chunk16(const uint32_t (&s)[16], const float4 (&c)[4], float2 negm,
                                            float2 (&acc)[4], uint32_t (&p)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float4 c4 = c[e >> 1];
        const float2 cc = (e & 1) ? make_float2(c4.z, c4.w) : make_float2(c4.x, c4.y);
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1])), cc, negm);
        float2 y;
        if ((e & 7) < kPoly)
            y = exp2_fma2(x);
        else
            y = make_float2(ex2_approx(x.x), ex2_approx(x.y));
        acc[e & 3] = __fadd2_rn(acc[e & 3], y);
        p[e] = pack_bf16x2(y.x, y.y);
    }
}
// The coefficients of chunk q + 1 are read together with its TMEM load, one
// chunk ahead of their use: the TMEM waits order every memory access around
// them, so a read issued after a wait would expose its full latency.
template <int kPoly>
__device__ __forceinline__ float row_exp_store_coef16(uint32_t t_s, const float4* coef, float m) {
    const float2 negm = make_float2(-m, -m);
    float2 acc[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.0f, 0.0f);
    uint32_t sa[16], sb[16], p[8];
    float4 ca[4], cb[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) ca[k] = coef[k];
    tmem_ld16_issue(t_s, sa);
#pragma unroll
    for (int q = 0; q < 8; q += 2) {
        tmem_ld16_wait(sa);
        tmem_ld16_issue(t_s + 16 * (q + 1), sb);
#pragma unroll
        for (int k = 0; k < 4; ++k) cb[k] = coef[4 * (q + 1) + k];
        exp_chunk16<kPoly>(sa, ca, negm, acc, p);
        tmem_st8(t_s + 8 * q, p);
        tmem_ld16_wait(sb);
        if (q + 2 < 8) {
            tmem_ld16_issue(t_s + 16 * (q + 2), sa);
#pragma unroll
            for (int k = 0; k < 4; ++k) ca[k] = coef[4 * (q + 2) + k];
        }
        exp_chunk16<kPoly>(sb, cb, negm, acc, p);
        tmem_st8(t_s + 8 * (q + 1), p);
    }
    const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
    return t.x + t.y;
}

// Masked form for a ragged last tile (columns >= vc get P = 0): MUFU only,
// one 32-column chunk at a time; coef may be null (scalar scale_log2).
__device__ __forceinline__ float row_exp_store_masked_impl(uint32_t t_s, const float4* coef, float sl2, float m,
                                                           int vc) {
    const float2 negm = make_float2(-m, -m);
    float2 acc[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.0f, 0.0f);
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        uint32_t s[32];
        tmem_ld32(t_s + c * 32, s);
        uint32_t p[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            float2 cc = make_float2(sl2, sl2);
            if (coef) {
                const float4 c4 = coef[c * 8 + (e >> 1)];
                cc = (e & 1) ? make_float2(c4.z, c4.w) : make_float2(c4.x, c4.y);
            }
            float2 x = __ffma2_rn(make_float2(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1])), cc, negm);
            const int col = c * 32 + 2 * e;
            x.x = col < vc ? x.x : -INFINITY;
            x.y = col + 1 < vc ? x.y : -INFINITY;
            const float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
            acc[e & 3] = __fadd2_rn(acc[e & 3], make_float2(p0, p1));
            p[e] = pack_bf16x2(p0, p1);
        }
        tmem_st16(t_s + c * 16, p);
    }
    const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
    return t.x + t.y;
}

// Cold paths kept out of line, so they do not add to the register pressure of
// the per-tile loop: tail tiles (masked), O rescaling, the epilogues.
__device__ __noinline__ float row_max_masked(uint32_t t_s, int vc) { return row_max<true>(t_s, vc); }
__device__ __noinline__ float row_exp_store_masked(uint32_t t_s, const float4* coef, float sl2, float m, int vc) {
    return row_exp_store_masked_impl(t_s, coef, sl2, m, vc);
}

// O *= alpha for one row (one thread), in TMEM.
__device__ __noinline__ void rescale_o(uint32_t t_o, float alpha) {
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + c * 32, o);
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
        tmem_st32(t_o + c * 32, o);
        tmem_st_wait();
    }
}

// Final output row: O / l -> BF16 (all lanes load from TMEM; only valid rows store).
__device__ __noinline__ void store_out_row(uint32_t t_o, float inv_l, uint16_t* dst, bool row_ok) {
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + c * 32, o);
        uint32_t b[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
            b[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
        if (row_ok) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
            d4[0] = make_uint4(b[0], b[1], b[2], b[3]);
            d4[1] = make_uint4(b[4], b[5], b[6], b[7]);
            d4[2] = make_uint4(b[8], b[9], b[10], b[11]);
            d4[3] = make_uint4(b[12], b[13], b[14], b[15]);
        }
    }
}

// Partial row of one split: unnormalised fp32 O, 4 dims per float4, laid out
// [32 chunks][256 rows] so that consecutive rows (threads) touch consecutive
// 16-byte words.
__device__ __noinline__ void store_partial_row(uint32_t t_o, float4* dst) {
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + c * 32, o);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            dst[(c * 8 + e) * 256] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                                 __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
    }
}

// Merge of the splits of one row (run by the last CTA of a unit to arrive):
// O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s with M = max_s m_s. Eight
// 16-byte loads per split are in flight at a time.
__device__ __noinline__ void merge_row(const AttnArgs& a, int unit, int row, uint16_t* dst, float* lse_dst) {
    const int units = a.heads * a.pairs;
    float mmax = -INFINITY;
    for (int s = 0; s < a.splits; ++s)
        mmax = fmaxf(mmax, __ldcg(&a.part_ml[(static_cast<int64_t>(s) * units + unit) * 256 + row]).x);
    float L = 0.0f;
    for (int s = 0; s < a.splits; ++s) {
        const float2 ml = __ldcg(&a.part_ml[(static_cast<int64_t>(s) * units + unit) * 256 + row]);
        L += ml.y * exp2f(ml.x - mmax);
    }
    const float inv = 1.0f / L;
#pragma unroll 1
    for (int c0 = 0; c0 < 32; c0 += 8) {
        float4 acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
        for (int s = 0; s < a.splits; ++s) {
            const int64_t pu = static_cast<int64_t>(s) * units + unit;
            const float g = exp2f(__ldcg(&a.part_ml[pu * 256 + row]).x - mmax);
            const float4* base = a.part_o + pu * 32 * 256 + row;
            float4 o[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) o[k] = __ldcg(base + (c0 + k) * 256);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                acc[k].x += o[k].x * g;
                acc[k].y += o[k].y * g;
                acc[k].z += o[k].z * g;
                acc[k].w += o[k].w * g;
            }
        }
#pragma unroll
        for (int k = 0; k < 8; k += 2)
            reinterpret_cast<uint4*>(dst)[(c0 + k) >> 1] =
                make_uint4(pack_bf16x2(acc[k].x * inv, acc[k].y * inv), pack_bf16x2(acc[k].z * inv, acc[k].w * inv),
                           pack_bf16x2(acc[k + 1].x * inv, acc[k + 1].y * inv),
                           pack_bf16x2(acc[k + 1].z * inv, acc[k + 1].w * inv));
    }
    if (lse_dst) *lse_dst = (mmax + log2f(L)) * 0.69314718055994531f;
}

// Arm a K (or V) stage for tile t and issue its two TMA boxes.
__device__ __forceinline__ void load_k_tile(const AttnArgs& a, int t, int head, uint32_t kdst, uint32_t kbar,
                                            const CUtensorMap* tm_kc, const CUtensorMap* tm_kcur) {
    mbar_arrive_expect_tx(kbar, kTileBytes);
    if (t < a.tiles_c) {
        tma_load_3d(kdst, tm_kc, 0, t * BN, head, kbar);
        tma_load_3d(kdst + kHalfBytes, tm_kc, 64, t * BN, head, kbar);
    } else {
        const int row = (t - a.tiles_c) * BN;
        tma_load_3d(kdst, tm_kcur, 0, row, head, kbar);
        tma_load_3d(kdst + kHalfBytes, tm_kcur, 64, row, head, kbar);
    }
}

__device__ __forceinline__ void load_v_tile(const AttnArgs& a, int t, int head, uint32_t vdst, uint32_t vbar,
                                            const CUtensorMap* tm_vc, const CUtensorMap* tm_vcur) {
    mbar_arrive_expect_tx(vbar, kTileBytes);
    if (t < a.tiles_c) {
        tma_load_3d(vdst, tm_vc, 0, t * BN, head, vbar);
        tma_load_3d(vdst + kHalfBytes, tm_vc, 64, t * BN, head, vbar);
    } else {
        const int row = (t - a.tiles_c) * BN;
        tma_load_3d(vdst, tm_vcur, 0, head, row, vbar);
        tma_load_3d(vdst + kHalfBytes, tm_vcur, 64, head, row, vbar);
    }
}

// Bounded wait for the last armed phase of each K and V stage: no copy may
// still be in flight when the CTA exits (matters only after an abort).
__device__ __forceinline__ void drain_armed(const int (&k_armed)[kStages], const int (&v_armed)[kStages],
                                            uint32_t kfull0, uint32_t vfull0) {
    for (int st = 0; st < kStages; ++st) {
        const uint64_t t0 = global_timer_ns();
        while ((k_armed[st] >= 0 && !mbar_try_wait(kfull0 + 8u * st, k_armed[st])) ||
               (v_armed[st] >= 0 && !mbar_try_wait(vfull0 + 8u * st, v_armed[st]))) {
            if (global_timer_ns() - t0 > NOMAS_WAIT_NS) break;
        }
    }
}

template <int kMode>
__global__ void __launch_bounds__(kMode == kFused ? 512 : 384, 1)
    attn_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap tm_q,
                const __grid_constant__ CUtensorMap tm_kcur, const __grid_constant__ CUtensorMap tm_vcur,
                const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc) {
    constexpr bool kInt8 = kMode != kBf16;   // cache tiles carry per-key K coefficients
    constexpr bool kFill = kMode == kFused;  // cache tiles converted by the filler warpgroup
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + kOffBar;
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kOffBar + kOffTmemSlot);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffBar + kOffAbort);
    volatile int* dq_go = reinterpret_cast<volatile int*>(smem + kOffBar + kOffDqGo);
    volatile int* last_flag = reinterpret_cast<volatile int*>(smem + kOffBar + kOffLast);
    const WaitCtl ctl{abort_flag, a.err};

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work unit
    const int unit = blockIdx.x / a.splits;
    const int split = blockIdx.x % a.splits;
    const int head = unit / a.pairs;
    const int pair = unit % a.pairs;
    const int qt0 = 2 * pair;
    const bool has_q1 = (qt0 + 1) < a.tiles_q;
    const int nq_tiles = has_q1 ? 2 : 1;
    const int t_total = a.tiles_c + a.tiles_q;
    const int t_begin = split * a.tiles_per_split;
    int t_end = t_begin + a.tiles_per_split;
    if (t_end > t_total) t_end = t_total;
    const int n = t_end - t_begin; // >= 1 by construction of the split count
    // cache tiles of this CTA come first: i < nci (INT8 caches: K coefficients per tile)
    const int nci = kInt8 ? max(0, min(t_end, a.tiles_c) - t_begin) : 0;

    // ---- setup
    if (threadIdx.x == 0) {
        mbar_init(bar(B_QFULL), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(B_KFULL + s), 1);
            mbar_init(bar(B_VFULL + s), 1);
            mbar_init(bar(B_KEMPTY + s), 1);
            mbar_init(bar(B_VEMPTY + s), 1);
        }
        for (int w = 0; w < 2; ++w) {
            mbar_init(bar(B_SFULL + w), 1);
            mbar_init(bar(B_PFULL + w), 4);
            mbar_init(bar(B_OFULL + w), 1);
        }
        mbar_init(bar(B_DRAIN), 1);
        for (int c = 0; c < kCoefSlots; ++c) {
            mbar_init(bar(B_CFULL + c), 1);
            mbar_init(bar(B_CEMPTY + c), 4 * nq_tiles); // one arrival per active softmax warp
        }
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(sbase + kOffBar + kOffTmemSlot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // launched dependent on the previous kernel of the call: barriers and TMEM
    // are set up while it finishes; nothing it wrote is read before this point
    grid_dep_wait();

    // the K coefficients of cache tile t into coefficient slot `slot`: scale_log2
    // times the key's K scale (keys past the end get scale_log2, so that a masked
    // score -inf stays -inf), and per writer warp the range over valid keys
    auto put_coef = [&](int t, float ks, bool key_ok, int key_local, uint32_t slot, int bound_idx) {
        const float c = key_ok ? a.scale_log2 * ks : a.scale_log2;
        float cmax = key_ok ? c : -INFINITY, cmin = key_ok ? c : INFINITY;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            cmax = fmaxf(cmax, __shfl_xor_sync(0xFFFFFFFFu, cmax, off));
            cmin = fminf(cmin, __shfl_xor_sync(0xFFFFFFFFu, cmin, off));
        }
        reinterpret_cast<float*>(smem + kOffCoef + slot * (BN * 4))[key_local] = c;
        if (lane == 0) reinterpret_cast<float2*>(smem + kOffBound + slot * 32)[bound_idx] = make_float2(cmax, cmin);
        (void)t;
    };

    if (warp < 4) {
      if (warp == 0) {
        // ================================================================ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_kcur);
            tma_prefetch_desc(&tm_vcur);
            if (!kFill) {
                tma_prefetch_desc(&tm_kc);
                tma_prefetch_desc(&tm_vc);
            }
            mbar_arrive_expect_tx(bar(B_QFULL), static_cast<uint32_t>(nq_tiles) * kTileBytes);
            for (int w = 0; w < nq_tiles; ++w) {
                const uint32_t dst = sbase + kOffQ + w * kTileBytes;
                tma_load_3d(dst, &tm_q, 0, (qt0 + w) * BM, head, bar(B_QFULL));
                tma_load_3d(dst + kHalfBytes, &tm_q, 64, (qt0 + w) * BM, head, bar(B_QFULL));
            }
            // kFused: one filler for every stage, the converting warpgroup (codes for
            // cache tiles, TMA for current-segment tiles): with a single filler in
            // tile order every parity wait on the stage ring is exact.
            if (!kFill) {
                int k_armed[kStages] = {-1, -1}, v_armed[kStages] = {-1, -1};
                for (int i = 0; i < n; ++i) {
                    const int st = i % kStages;
                    const uint32_t free_ph = ((i / kStages) & 1) ^ 1;
                    if (i >= kStages && !mbar_wait(bar(B_KEMPTY + st), free_ph, ctl)) break;
                    load_k_tile(a, t_begin + i, head, sbase + kOffK + st * kTileBytes, bar(B_KFULL + st), &tm_kc,
                                &tm_kcur);
                    k_armed[st] = (i / kStages) & 1;
                    if (i >= kStages && !mbar_wait(bar(B_VEMPTY + st), free_ph, ctl)) break;
                    load_v_tile(a, t_begin + i, head, sbase + kOffV + st * kTileBytes, bar(B_VFULL + st), &tm_vc,
                                &tm_vcur);
                    v_armed[st] = (i / kStages) & 1;
                }
                drain_armed(k_armed, v_armed, bar(B_KFULL), bar(B_VFULL));
            }
        }
      } else if (warp == 2) {
        // ================================================================ K coefficients
        // kWindow: the K scales of every cache tile (4 keys per lane) into the
        // coefficient ring, off the TMA producer's path (their global loads
        // would hold up the stage ring).
        if (kMode == kWindow) {
            for (int i = 0; i < nci; ++i) {
                const uint32_t slot = static_cast<uint32_t>(i % kCoefSlots);
                const int t = t_begin + i;
                float ks[4];
                bool ko[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int key = t * BN + q * 32 + lane;
                    ko[q] = key < a.nc;
                    ks[q] = ko[q] ? __ldg(a.ksc + static_cast<int64_t>(head) * a.cap_tok + key) : 0.0f;
                }
                if (i >= kCoefSlots && !mbar_wait_warp(bar(B_CEMPTY + slot), ((i / kCoefSlots) & 1) ^ 1, ctl)) break;
#pragma unroll
                for (int q = 0; q < 4; ++q) put_coef(t, ks[q], ko[q], q * 32 + lane, slot, q);
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_CFULL + slot));
            }
        }
      } else if (warp == 1) {
        // ================================================================ MMA issuer
        // The whole warp runs the loop (warp-uniform waits and conditions) and
        // one elected lane issues each MMA and commit; MMAs issued by a single
        // lane in a divergent branch run at little more than half the
        // tensor-core rate whenever a branch separates two groups of them.
        using I = Issuer<true>;
        constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, kD, false, true);
        // TMEM columns: S of Q tile w at 128 w, O of Q tile w at 256 + 128 w
        auto tm_s = [&](int w) { return tmem + 128u * static_cast<uint32_t>(w); };
        auto tm_o = [&](int w) { return tmem + 256u + 128u * static_cast<uint32_t>(w); };
        bool ok = I::wait(bar(B_QFULL), 0, ctl);
        tc_fence_after();
        // k-step-0 descriptors of the Q tiles and of the K and V stages (scalars:
        // selected, not indexed, so they stay in registers)
        static_assert(kStages == 2, "the stage descriptors below assume two stages");
        const uint64_t q_desc0 = desc_kmajor(sbase + kOffQ, 0), q_desc1 = desc_kmajor(sbase + kOffQ + kTileBytes, 0);
        const uint64_t k_desc0 = desc_kmajor(sbase + kOffK, 0), k_desc1 = desc_kmajor(sbase + kOffK + kTileBytes, 0);
        const uint64_t v_desc0 = desc_mnmajor(sbase + kOffV, 0);
        const uint64_t v_desc1 = desc_mnmajor(sbase + kOffV + kTileBytes, 0);
        auto issue_s = [&](int w, int st) {
            const uint64_t qd = w ? q_desc1 : q_desc0, kd = st ? k_desc1 : k_desc0;
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk)
                I::ss(tm_s(w), qd + kstep_kmajor(kk), kd + kstep_kmajor(kk), idesc_qk, kk > 0 ? 1u : 0u);
        };
        auto issue_pv = [&](int w, int st, bool first_tile) {
            const uint64_t vd = st ? v_desc1 : v_desc0;
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
                I::ts(tm_o(w), tm_s(w) + kk * 8, vd + kstep_mnmajor(kk), idesc_pv, (first_tile && kk == 0) ? 0u : 1u);
        };
        if (ok) ok = I::wait(bar(B_KFULL + 0), 0, ctl);
        if (ok) {
            tc_fence_after();
            for (int w = 0; w < nq_tiles; ++w) {
                issue_s(w, 0);
                I::commit(bar(B_SFULL + w));
            }
            // K of tile 0 is free once these S MMAs finish (a fill of tile 2 waits for it)
            if (kStages < n) I::commit(bar(B_KEMPTY + 0));
        }
        for (int i = 0; ok && i < n; ++i) {
            const int st = i % kStages;
            const uint32_t ph = (i / kStages) & 1;
            const int st1 = (i + 1) % kStages;
            const uint32_t ph1 = ((i + 1) / kStages) & 1;
            const bool last = (i + 1 == n);
            if (!(ok = I::wait(bar(B_VFULL + st), ph, ctl))) break;
            for (int w = 0; w < nq_tiles; ++w) {
                if (!(ok = I::wait(bar(B_PFULL + w), i & 1, ctl))) break;
                tc_fence_after();
                issue_pv(w, st, i == 0);
                // each release is committed only when a later fill waits for it,
                // so no arrival is left pending at exit
                if (w == nq_tiles - 1 && i + kStages < n) I::commit(bar(B_VEMPTY + st));
                if (!last) {
                    // K of tile i + 1 is needed from here on only: P.V of Q tile 0
                    // never waits for it
                    if (w == 0) {
                        if (!(ok = I::wait(bar(B_KFULL + st1), ph1, ctl))) break;
                        tc_fence_after();
                    }
                    issue_s(w, st1);
                    I::commit(bar(B_SFULL + w));
                    if (w == nq_tiles - 1 && i + 1 + kStages < n) I::commit(bar(B_KEMPTY + st1));
                } else {
                    I::commit(bar(B_OFULL + w));
                }
            }
        }
        // drain: every MMA issued above has completed before teardown
        I::commit(bar(B_DRAIN));
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bar(B_DRAIN), 0)) {
            if (global_timer_ns() - t0 > NOMAS_WAIT_NS) break;
        }
      }
    } else if (warp < 12) {
        // ================================================================ softmax
        const int w = (warp - 4) >> 2;
        const int quad = warp & 3;
        const int r = quad * 32 + lane; // row inside the Q tile
        const bool active = (w == 0 || has_q1);
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t t_s = tmem + lane_off + w * 128;
        const uint32_t t_o = tmem + lane_off + 256 + w * 128;
        float m_ref = -INFINITY; // reference max, log2 units
        float l = 0.0f;
        bool ok = true;
        // kWindow: the coefficient range of the next cache tile, read (after its
        // CFULL wait) at the end of the previous tile
        float chi_next = 0.0f, clo_next = 0.0f;
        auto load_coefs = [&](int i) -> bool {
            const uint32_t slot = static_cast<uint32_t>(i % kCoefSlots);
            if (!mbar_wait(bar(B_CFULL + slot), (i / kCoefSlots) & 1, ctl)) return false;
            const uint32_t bd = sbase + kOffBound + slot * 32;
            const float4 b0 = lds128_ordered(bd), b1 = lds128_ordered(bd + 16);
            chi_next = fmaxf(fmaxf(b0.x, b0.z), fmaxf(b1.x, b1.z));
            clo_next = fminf(fminf(b0.y, b0.w), fminf(b1.y, b1.w));
            return true;
        };
        if (active) {
            const float sl2 = a.scale_log2;
            if (kMode == kWindow && nci > 0) ok = load_coefs(0);
            for (int i = 0; ok && i < n; ++i) {
                const int t = t_begin + i;
                const bool coef = kInt8 && i < nci; // warp-uniform
                const uint32_t slot = static_cast<uint32_t>(i % kCoefSlots);
                if (!(ok = mbar_wait(bar(B_SFULL + w), i & 1, ctl))) break;
                tc_fence_after();
                const int vc = tile_valid(a, t);
                const bool full = (vc == BN);
                float chi = sl2, clo = sl2;
                const float4* cf = nullptr;
                if (coef) {
                    cf = reinterpret_cast<const float4*>(smem + kOffCoef + slot * (BN * 4));
                    if (kMode == kWindow) {
                        // loaded (after their CFULL wait) at the end of the previous tile
                        chi = chi_next;
                        clo = clo_next;
                    } else {
                        if (!(ok = mbar_wait(bar(B_CFULL + slot), (i / kCoefSlots) & 1, ctl))) break;
                        const uint32_t bd = sbase + kOffBound + slot * 32;
                        const float4 b0 = lds128_ordered(bd), b1 = lds128_ordered(bd + 16);
                        chi = fmaxf(fmaxf(b0.x, b0.z), fmaxf(b1.x, b1.z));
                        clo = fminf(fminf(b0.y, b0.w), fminf(b1.y, b1.w));
                    }
                }
                // pass 1: the tile's raw maximum; x_j = s_j * c_j with every c_j in
                // [clo, chi], so the scaled maximum lies in [lo, hi] below
                const float mx = !full ? row_max_masked(t_s, vc)
                                 : (kMode == kWindow && coef) ? row_max32(t_s)
                                                               : row_max<false>(t_s, vc);
                const float hi = mx >= 0.0f ? mx * chi : mx * clo;
                const float lo = mx >= 0.0f ? mx * clo : mx * chi;
                // the reference moves only when the tile may exceed it by more than the
                // threshold: to the upper bound when that is within the threshold of
                // the true maximum (always so without coefficients), else to the
                // exact scaled maximum
                const bool up = hi > m_ref + kRescaleThreshold;
                const bool exact = up && hi - lo > kRescaleThreshold;
                float m_new = up ? hi : m_ref;
                if (coef && __any_sync(0xFFFFFFFFu, exact)) {
                    const float me = row_max_scaled(t_s, cf, vc);
                    if (exact) m_new = me;
                }
                const float alpha = up ? ex2_approx(m_ref - m_new) : 1.0f; // 0 on the first tile
                if (i > 0 && __any_sync(0xFFFFFFFFu, up)) rescale_o(t_o, alpha);
                l *= alpha;
                m_ref = m_new;
                // pass 2: P into TMEM, row sum in fp32
                if (coef) {
                    if constexpr (kMode == kWindow)
                        l += full ? row_exp_store_coef16<kExp2PolyPairs>(t_s, cf, m_ref)
                                  : row_exp_store_masked(t_s, cf, sl2, m_ref, vc);
                    else
                        l += full ? row_exp_store_full<kExp2PolyPairsFused, true>(t_s, cf, sl2, m_ref)
                                  : row_exp_store_masked(t_s, cf, sl2, m_ref, vc);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(B_CEMPTY + slot));
                } else {
                    l += full ? row_exp_store_full<kFill ? kExp2PolyPairsFused : kExp2PolyPairs, false>(t_s, nullptr,
                                                                                                       sl2, m_ref)
                              : row_exp_store_masked(t_s, nullptr, sl2, m_ref, vc);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_PFULL + w));
                // kWindow: the next cache tile's coefficients, loaded now so that their
                // shared-memory loads (which queue behind the tensor core's operand
                // reads) complete while this warp waits for the next S
                if (kMode == kWindow && i + 1 < nci && !(ok = load_coefs(i + 1))) break;
            }
            // ---- epilogue
            if (ok) ok = mbar_wait(bar(B_OFULL + w), 0, ctl);
        }
        const int qrow = (qt0 + w) * BM + r;
        const bool row_ok = active && ok && qrow < a.nq;
        if (a.splits == 1) {
            if (active && ok) {
                tc_fence_after();
                store_out_row(t_o, 1.0f / l, a.out + (static_cast<int64_t>(qrow) * a.heads + head) * kD, row_ok);
                if (row_ok && a.lse)
                    a.lse[static_cast<int64_t>(head) * a.nq + qrow] = (m_ref + log2f(l)) * 0.69314718055994531f;
            }
        } else {
            // partial of this split, then the unit's arrival count; the last CTA to
            // arrive merges every split's partial of its rows
            const int units = a.heads * a.pairs;
            const int64_t pu = static_cast<int64_t>(split) * units + unit;
            const int prow = w * BM + r;
            if (active && ok) {
                tc_fence_after();
                store_partial_row(t_o, a.part_o + pu * 32 * 256 + prow);
                a.part_ml[pu * 256 + prow] = make_float2(m_ref, l);
            }
            __threadfence();
            named_bar_sync(2, 256);
            if (threadIdx.x == 128) {
                const unsigned old = atomicAdd(&a.counters[unit], 1u);
                const bool is_last = old == static_cast<unsigned>(a.splits - 1);
                if (is_last) a.counters[unit] = 0u; // every split has arrived: ready for the next call
                *last_flag = is_last ? 1 : 0;
            }
            named_bar_sync(2, 256);
            if (*last_flag) {
                __threadfence();
                if (row_ok)
                    merge_row(a, unit, prow, a.out + (static_cast<int64_t>(qrow) * a.heads + head) * kD,
                              a.lse ? a.lse + static_cast<int64_t>(head) * a.nq + qrow : nullptr);
            }
        }
    } else if (kFill && warp >= 12) {
        // ================================================================ INT8 filler
        // Warp wq converts rows [32 wq, 32 wq + 32) of a cache tile; in step j a
        // warp covers rows 2j and 2j+1, 16 lanes per row, 8 codes per lane, so a
        // lane writes exactly one 16-byte BF16 chunk and each quarter-warp hits 8
        // distinct chunk slots of the swizzled row (no bank conflicts). Filler
        // thread f (0..127) also loads the K and V scales of key f of the tile.
        // The next cache tile's codes are loaded into registers as soon as the
        // current tile has been converted, so global latency overlaps the MMAs.
        const int f = threadIdx.x - 384;
        const int wq = warp - 12;
        const int half = lane >> 4;
        const int l16 = lane & 15;
        const bool elected = (f == 0);
        const uint32_t chunk_off = (l16 >> 3) * kHalfBytes;
        uint2 kb[16], vb[16];
        float ks_own = 0.0f, vs_own = 0.0f; // scales of key f of the tile whose codes are in kb / vb
        bool key_ok = false;
        // row (32 wq + 2j + half) of a tile: (row & 7) = (2j & 7) ^ half, so the swizzled
        // chunk slot is slot0 ^ (2j & 7) and the byte offset is a constant per j
        const uint32_t slot0 = static_cast<uint32_t>((l16 & 7) ^ half);
        const uint32_t row_off0 = chunk_off + static_cast<uint32_t>(wq * 32 + half) * 128u;
        auto load_codes = [&](const int8_t* base, int t, uint2 (&buf)[16]) {
            const int key0 = t * BN + wq * 32 + half;
            const int64_t grow0 = static_cast<int64_t>(head) * a.cap_tok + key0;
            const uint2* p = reinterpret_cast<const uint2*>(base + grow0 * kD) + l16;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const bool in = key0 + 2 * j < a.nc;
                buf[j] = in ? __ldg(p + j * 32) : make_uint2(0u, 0u); // 2 rows = 256 B = 32 uint2
            }
        };
        auto load_scales = [&](int t) {
            const int key = t * BN + f;
            key_ok = key < a.nc;
            const int64_t g = static_cast<int64_t>(head) * a.cap_tok + key;
            ks_own = key_ok ? __ldg(a.ksc + g) : 0.0f;
            vs_own = key_ok ? __ldg(a.vsc + g) : 0.0f;
        };
        auto convert_k = [&](uint32_t tile) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint32_t off = row_off0 + j * 256u + ((slot0 ^ static_cast<uint32_t>((2 * j) & 7)) << 4);
                st_shared_v4(tile + off, codes_to_bf16<false>(kb[j], 0.0f));
            }
        };
        auto convert_v = [&](uint32_t tile) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float sc = __shfl_sync(0xFFFFFFFFu, vs_own, 2 * j + half);
                const uint32_t off = row_off0 + j * 256u + ((slot0 ^ static_cast<uint32_t>((2 * j) & 7)) << 4);
                st_shared_v4(tile + off, codes_to_bf16<true>(vb[j], sc));
            }
        };
        // one elected thread waits; the group learns the outcome after a named
        // barrier, so all 128 threads take the same branch
        auto group_wait = [&](uint32_t barrier, uint32_t parity) -> bool {
            if (elected) *dq_go = mbar_wait(barrier, parity, ctl) ? 1 : 0;
            named_bar_sync(1, 128);
            return *dq_go != 0;
        };
        int k_armed[kStages] = {-1, -1}, v_armed[kStages] = {-1, -1};
        if (nci > 0) {
            load_codes(a.kc8, t_begin, kb);
            load_codes(a.vc8, t_begin, vb);
            load_scales(t_begin);
        }
        for (int i = 0; i < n; ++i) {
            const int t = t_begin + i;
            const int st = i % kStages;
            const uint32_t free_ph = ((i / kStages) & 1) ^ 1;
            const uint32_t ktile = sbase + kOffK + st * kTileBytes;
            const uint32_t vtile = sbase + kOffV + st * kTileBytes;
            const bool cached = i < nci;
            const bool next_cached = i + 1 < nci;
            // ---- K (freed early: right after the S MMAs of tile i - 2)
            if (i >= kStages && !group_wait(bar(B_KEMPTY + st), free_ph)) break;
            if (!cached) {
                if (elected) {
                    load_k_tile(a, t, head, ktile, bar(B_KFULL + st), &tm_kc, &tm_kcur);
                    k_armed[st] = (i / kStages) & 1;
                }
            } else {
                const uint32_t slot = static_cast<uint32_t>(i % kCoefSlots);
                convert_k(ktile);
                if (next_cached) load_codes(a.kc8, t + 1, kb);
                // the tile's K coefficients into the coefficient ring
                if (i >= kCoefSlots && !group_wait(bar(B_CEMPTY + slot), ((i / kCoefSlots) & 1) ^ 1)) break;
                put_coef(t, ks_own, key_ok, f, slot, wq);
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (elected) {
                    mbar_arrive(bar(B_KFULL + st));
                    mbar_arrive(bar(B_CFULL + slot));
                }
            }
            // ---- V (freed after the P.V MMAs of tile i - 2)
            if (i >= kStages && !group_wait(bar(B_VEMPTY + st), free_ph)) break;
            if (!cached) {
                if (elected) {
                    load_v_tile(a, t, head, vtile, bar(B_VFULL + st), &tm_vc, &tm_vcur);
                    v_armed[st] = (i / kStages) & 1;
                }
            } else {
                convert_v(vtile);
                if (next_cached) {
                    load_codes(a.vc8, t + 1, vb);
                    load_scales(t + 1);
                }
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (elected) mbar_arrive(bar(B_VFULL + st));
            }
        }
        if (elected) drain_armed(k_armed, v_armed, bar(B_KFULL), bar(B_VFULL));
    }

    // ---- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// One work item = 16 codes (16 bytes) of one row of K or V; 8 items per row,
// consecutive threads on consecutive items, so loads (128 B per row) and
// stores (256 B per row) are fully coalesced. Grid-stride over both tensors.
// K rows are written as their codes (exact in BF16; the K scale reaches the
// scores through the attention kernel's coefficients), V rows as code * scale.
__global__ void __launch_bounds__(512) dequant_window_kernel(const __grid_constant__ DequantArgs a) {
    // Launched dependent on the RoPE prep kernel and overlapping it: it reads
    // only the cache, which was complete before prep started. It lets the
    // attention kernel launch early, and before it exits it waits for prep, so
    // the attention kernel's wait on it covers prep too.
    grid_dep_launch();
    const uint32_t rows = static_cast<uint32_t>(a.heads) * static_cast<uint32_t>(a.nc); // per tensor, < 2^31
    const uint32_t items = 2u * rows * 8u;                                              // < 2^32 by the host check
    for (uint32_t it = blockIdx.x * blockDim.x + threadIdx.x; it < items; it += gridDim.x * blockDim.x) {
        const uint32_t trow = it >> 3;
        const uint32_t part = it & 7u;
        const bool is_v = trow >= rows;
        const uint32_t r = is_v ? trow - rows : trow;
        const uint32_t head = fast_div(r, a.div_nc);
        const uint32_t tok = r - head * static_cast<uint32_t>(a.nc);
        const int64_t src_row = static_cast<int64_t>(head) * a.cap_tok + tok;
        const uint4 w = __ldg(reinterpret_cast<const uint4*>((is_v ? a.vc : a.kc) + src_row * kD) + part);
        uint4* dst = reinterpret_cast<uint4*>((is_v ? a.vd : a.kd) + static_cast<int64_t>(r) * kD) + 2 * part;
        if (is_v) {
            const float sc = __ldg(a.vs + src_row);
            dst[0] = codes_to_bf16<true>(make_uint2(w.x, w.y), sc);
            dst[1] = codes_to_bf16<true>(make_uint2(w.z, w.w), sc);
        } else {
            dst[0] = codes_to_bf16<false>(make_uint2(w.x, w.y), 0.0f);
            dst[1] = codes_to_bf16<false>(make_uint2(w.z, w.w), 0.0f);
        }
    }
    grid_dep_wait();
}

// The dynamic shared-memory limit of a kernel is an attribute of the kernel in
// one device's context: it is raised once per device (and per kernel), the
// first time that device launches it. Concurrent first launches may both set
// it, which is harmless.
template <int kMode>
cudaError_t ensure_smem_attr() {
    constexpr int kMaxDev = 64;
    static std::atomic<bool> done[kMaxDev];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDev && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    e = cudaFuncSetAttribute(attn_kernel<kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e == cudaSuccess && dev >= 0 && dev < kMaxDev) done[dev].store(true, std::memory_order_release);
    return e;
}

template <int kMode>
cudaError_t launch_mode(const AttnArgs& a, const CUtensorMap& tm_q, const CUtensorMap& tm_kcur,
                        const CUtensorMap& tm_vcur, const CUtensorMap& tm_kc, const CUtensorMap& tm_vc,
                        cudaStream_t s) {
    cudaError_t e = ensure_smem_attr<kMode>();
    if (e != cudaSuccess) return e;
    return launch_dependent(attn_kernel<kMode>, dim3(a.heads * a.pairs * a.splits), dim3(kMode == kFused ? 512 : 384),
                            kSmemBytes, s, a, tm_q, tm_kcur, tm_vcur, tm_kc, tm_vc);
}

} // namespace

cudaError_t launch_dequant_window(const DequantArgs& a, cudaStream_t s) {
    const uint64_t items = 2ull * static_cast<uint64_t>(a.heads) * static_cast<uint64_t>(a.nc) * 8ull;
    if (items == 0) return cudaSuccess;
    uint64_t blocks = (items + 511) / 512;
    const uint64_t cap = 148ull * 4ull; // persistent: 4 blocks of 512 threads per SM
    if (blocks > cap) blocks = cap;
    return launch_dependent(dequant_window_kernel, dim3(static_cast<unsigned>(blocks)), dim3(512), 0, s, a);
}

cudaError_t launch_attn(const AttnArgs& a, AttnForm form, const CUtensorMap& tm_q, const CUtensorMap& tm_kcur,
                        const CUtensorMap& tm_vcur, const CUtensorMap& tm_kc, const CUtensorMap& tm_vc,
                        cudaStream_t s) {
    switch (form) {
    case AttnForm::kBf16Cache: return launch_mode<kBf16>(a, tm_q, tm_kcur, tm_vcur, tm_kc, tm_vc, s);
    case AttnForm::kInt8Window: return launch_mode<kWindow>(a, tm_q, tm_kcur, tm_vcur, tm_kc, tm_vc, s);
    default: return launch_mode<kFused>(a, tm_q, tm_kcur, tm_vcur, tm_kc, tm_vc, s);
    }
}

} // namespace nomas
