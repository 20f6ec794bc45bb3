// Segment-causal joint attention on sm_100a tensor cores.
//
// What it computes (Hy-Nomas model card, "Segment-Autoregressive Diffusion
// Transformer"; blog "Segment-wise causal joint attention"): for each head
// and each query token of the current segment, softmax attention over the
// visible cached tokens of earlier segments followed by every token of the
// current segment (no mask inside a segment; causality across segments is
// structural: later segments are never in the cache). An INT8 cache is
// attended to in 16-bit floating point (model card, "Single-GPU Low-Memory
// Inference": INT8 KV storage, 16-bit attention computation), here FP16 with
// power-of-two exponents per Q row and per 128-key tile (nomas_f16.cuh): the
// scores of a tile are s = Q^.K^ * 2^(a_i + b_T), its V values V^ * 2^c_T.
//
// Three forms (template parameter kMode):
//   kBf16   BF16 cache; every K/V tile arrives by TMA; BF16 Q, K, P.
//   kWindow INT8 cache whose visible window dequant_window_kernel has written
//           to an FP16 copy once per call; tiles by TMA.
//   kFused  INT8 cache converted to FP16 in shared memory tile by tile by a
//           filler warpgroup (no copy: for workspaces too small to hold one).
// In both INT8 forms Q and K are FP16 for every tile; P.V is FP16 for cache
// tiles and BF16 for the current segment's tiles (V is the caller's BF16).
//
// Structure of one CTA (one "unit" = two 128-row Q tiles of one head, and a
// contiguous range of 128-key KV tiles: cache tiles first, then the current
// segment's tiles):
//   warp 0      TMA producer: Q tiles once, then (kBf16, kWindow) every K
//               tile into a 2-stage ring
//   warp 2      (kBf16, kWindow) TMA producer of every V tile, 3-stage ring
//   warp 1      TMEM allocator + tcgen05.mma issuer
//   warps 4-7   softmax warpgroup for Q tile 0 (one thread per query row)
//   warps 8-11  softmax warpgroup for Q tile 1
//   warps 12-15 kFused only: the one filler of the K/V ring. Cache tiles are
//               converted from codes and scales; current-segment tiles are
//               loaded by TMA. One filler in tile order keeps every parity
//               wait on the ring exact.
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each; the 16-bit
// probabilities P overwrite the first 64 columns of their S block and feed
// the P.V product straight from TMEM (A operand in tensor memory).
// MMA order per KV tile j: PV0(j-1) S0(j) | PV1(j-1) S1(j) -- while one
// softmax warpgroup exponentiates, the tensor core works for the other. The
// issuer waits for the loads of later tiles only right after it has issued a
// group of MMAs, so between groups it waits only for P.
// Online softmax in base 2 with lazy rescaling: the running reference max is
// raised only when a tile's max may exceed it by more than 8 (so P <= 256,
// inside FP16's range), and only then is O rescaled in TMEM. With INT8 caches
// the reference follows x + c_T (x the log2-scaled score, c_T the V exponent
// of its tile): P' = 2^(x + c_T - m) times V^ is 2^(x - m) times V, and the
// row sum adds P' * 2^-c_T.
// Split-KV: with splits > 1 each CTA leaves O/l in FP16 (times a per-row 2^-e)
// and (max, sum, 2^e) in the workspace and counts itself in per unit; the last
// CTA of a unit merges the splits and writes the output (partials still in L2).
#include "nomas_f16.cuh"
#include "nomas_internal.h"
#include "nomas_ptx.cuh"

#include <atomic>

namespace nomas {

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kKStages = 2;                   // K ring (a K stage is free again after the S MMAs)
constexpr int kVStages = 3;                   // V ring (free only after the P.V MMAs: one more stage)
constexpr uint32_t kTileBytes = BM * kD * 2;  // one 16-bit 128x128 tile
constexpr uint32_t kHalfBytes = kTileBytes / 2;
constexpr float kRescaleThreshold = 8.0f;     // P <= 2^8 between rescales

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;                                // 2 tiles
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;           // kKStages tiles
constexpr uint32_t kOffV = kOffK + kKStages * kTileBytes;    // kVStages tiles
constexpr uint32_t kOffBar = kOffV + kVStages * kTileBytes;  // barriers
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;        // + alignment slack

// barrier slots (8 bytes each)
enum {
    B_QFULL = 0,
    B_KFULL = 1,                // + stage
    B_VFULL = B_KFULL + kKStages,
    B_KEMPTY = B_VFULL + kVStages,  // K and V stages are released separately: K as soon
    B_VEMPTY = B_KEMPTY + kKStages, // as the S MMAs that read it are done, V after P.V
    B_SFULL = B_VEMPTY + kVStages,  // + softmax warpgroup
    B_PFULL = B_SFULL + 2,
    B_OFULL = B_PFULL + 2,
    B_DRAIN = B_OFULL + 2,
    B_COUNT = B_DRAIN + 1
};
constexpr uint32_t kOffTmemSlot = B_COUNT * 8;
constexpr uint32_t kOffAbort = kOffTmemSlot + 8;
constexpr uint32_t kOffDqGo = kOffAbort + 4;
constexpr uint32_t kOffLast = kOffDqGo + 4;
static_assert(kOffLast + 4 <= 256, "barrier area overflow");
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

enum { kBf16 = 0, kWindow = 1, kFused = 2 };

// kFused runs 512 threads, launched at 128 registers each (the whole register
// file of one SM). Per-warpgroup budgets move registers from the producer/MMA
// warpgroup and the filler to the two softmax warpgroups; they add up to the
// launch's 4 x 128. The host checks the compiled register count before the
// first launch (a smaller one would leave an inc waiting).
constexpr uint32_t kFusedRegsLaunch = 128;
constexpr uint32_t kFusedRegsCtl = 64;
constexpr uint32_t kFusedRegsSoftmax = 168;
constexpr uint32_t kFusedRegsFill = 112;
static_assert(kFusedRegsCtl + 2 * kFusedRegsSoftmax + kFusedRegsFill == 4 * kFusedRegsLaunch,
              "register budgets of the fused form");

// mbar_wait run by every lane of a converged warp; lane 0's outcome is
// broadcast so the warp leaves the wait converged.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, const WaitCtl& ctl) {
    const bool ok = mbar_wait(bar, parity, ctl);
    return __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
}

// The MMA issuer: the whole warp runs the loop (warp-uniform waits and
// conditions) and an elected lane issues each instruction inside the asm.
struct Issuer {
    static __device__ __forceinline__ void ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
        mma_ss_warp(d, a, b, idesc, acc);
    }
    static __device__ __forceinline__ void ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
        mma_ts_warp(d, a, b, idesc, acc);
    }
    static __device__ __forceinline__ void commit(uint32_t bar) { mma_commit_warp(bar); }
    static __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, const WaitCtl& ctl) {
        return mbar_wait_warp(bar, parity, ctl);
    }
};

__device__ __forceinline__ int tile_valid(const AttnArgs& a, int t) {
    const int rem = (t < a.tiles_c) ? a.nc - t * BN : a.nq - (t - a.tiles_c) * BN;
    return rem < BN ? rem : BN;
}

// K-major SW128 descriptor of k-step kk (16 dims) of a 128x128 16-bit tile.
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
constexpr int kExp2PolyPairs = 2;
constexpr int kExp2PolyPairsFused = 0;


// One 32-column chunk of an unmasked S row -> 16 packed 16-bit P columns
// (kF16: FP16, else BF16), P = 2^(s * c + b) with the tile's scalars c (the
// log2-scaled score coefficient) and b (the V exponent minus the reference).
template <int kPoly, bool kF16>
__device__ __forceinline__ void exp_chunk(const uint32_t (&s)[32], float2 cc, float2 bb, float2 (&acc)[4],
                                          uint32_t (&p)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1])), cc, bb);
        float2 y;
        if ((e & 7) < kPoly)
            y = exp2_fma2(x);
        else
            y = make_float2(ex2_approx(x.x), ex2_approx(x.y));
        acc[e & 3] = __fadd2_rn(acc[e & 3], y);
        p[e] = kF16 ? pack_f16x2(y.x, y.y) : pack_bf16x2(y.x, y.y);
    }
}

// P = 2^(s * c + b) of one full 128-key S row, written as packed 16-bit pairs
// over the first 64 columns of the row's S block; returns the fp32 row sum
// (four independent packed accumulators). The TMEM loads are software
// pipelined: chunk c + 1 is in flight while chunk c is exponentiated. P chunk c
// lands on columns [16c, 16c + 16), all of which were read with chunks <= c.
template <int kPoly, bool kF16>
__device__ __forceinline__ float row_exp_store_full(uint32_t t_s, float c, float b) {
    const float2 cc = make_float2(c, c);
    const float2 bb = make_float2(b, b);
    float2 acc[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.0f, 0.0f);
    uint32_t sa[32], sb[32], p[16];
    tmem_ld32_issue(t_s, sa);
    tmem_ld32_wait(sa);
    tmem_ld32_issue(t_s + 32, sb);
    exp_chunk<kPoly, kF16>(sa, cc, bb, acc, p);
    tmem_st16(t_s, p);
    tmem_ld32_wait(sb);
    tmem_ld32_issue(t_s + 64, sa);
    exp_chunk<kPoly, kF16>(sb, cc, bb, acc, p);
    tmem_st16(t_s + 16, p);
    tmem_ld32_wait(sa);
    tmem_ld32_issue(t_s + 96, sb);
    exp_chunk<kPoly, kF16>(sa, cc, bb, acc, p);
    tmem_st16(t_s + 32, p);
    tmem_ld32_wait(sb);
    exp_chunk<kPoly, kF16>(sb, cc, bb, acc, p);
    tmem_st16(t_s + 48, p);
    const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
    return t.x + t.y;
}

// Masked form for a ragged last tile (columns >= vc get P = 0): MUFU only,
// one 32-column chunk at a time.
__device__ __forceinline__ float row_exp_store_masked_impl(uint32_t t_s, float c, float b, int vc, bool f16) {
    const float2 cc = make_float2(c, c), bb = make_float2(b, b);
    float2 acc[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.0f, 0.0f);
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
        uint32_t s[32];
        tmem_ld32(t_s + ch * 32, s);
        uint32_t p[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            float2 x = __ffma2_rn(make_float2(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1])), cc, bb);
            const int col = ch * 32 + 2 * e;
            x.x = col < vc ? x.x : -INFINITY;
            x.y = col + 1 < vc ? x.y : -INFINITY;
            const float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
            acc[e & 3] = __fadd2_rn(acc[e & 3], make_float2(p0, p1));
            p[e] = f16 ? pack_f16x2(p0, p1) : pack_bf16x2(p0, p1);
        }
        tmem_st16(t_s + ch * 16, p);
    }
    const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
    return t.x + t.y;
}

// Cold paths kept out of line, so they do not add to the register pressure of
// the per-tile loop: tail tiles (masked), O rescaling, the epilogues.
__device__ __noinline__ float row_max_masked(uint32_t t_s, int vc) { return row_max<true>(t_s, vc); }
__device__ __noinline__ float row_exp_store_masked(uint32_t t_s, float c, float b, int vc, bool f16) {
    return row_exp_store_masked_impl(t_s, c, b, vc, f16);
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

// Partial row of one split: O / l times 2^-e in FP16, with e from the row's
// largest |O / l| (nomas_f16.cuh: that element lies in [2^14, 2^15), so no value
// leaves FP16's range whatever the magnitude of V), 8 dims per 16-byte word,
// laid out [16 chunks][256 rows] so that consecutive rows (threads) touch
// consecutive words. Returns 2^e, which the merge multiplies back.
__device__ __noinline__ float store_partial_row(uint32_t t_o, float inv_l, uint4* dst) {
    float mx = 0.0f;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + c * 32, o);
#pragma unroll
        for (int e = 0; e < 32; e += 2) mx = max3(mx, fabsf(__uint_as_float(o[e])), fabsf(__uint_as_float(o[e + 1])));
    }
    const int ex = pow2_exponent(mx * inv_l, kTopFloat);
    const float f = inv_l * exp2_int(-ex);
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + c * 32, o);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint32_t* q = o + 8 * e;
            dst[(c * 4 + e) * 256] =
                make_uint4(pack_f16x2(__uint_as_float(q[0]) * f, __uint_as_float(q[1]) * f),
                           pack_f16x2(__uint_as_float(q[2]) * f, __uint_as_float(q[3]) * f),
                           pack_f16x2(__uint_as_float(q[4]) * f, __uint_as_float(q[5]) * f),
                           pack_f16x2(__uint_as_float(q[6]) * f, __uint_as_float(q[7]) * f));
        }
    }
    return exp2_int(ex);
}

__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t w) {
    float lo, hi;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(w));
    return make_float2(lo, hi);
}

// Merge of the splits of one row (run by the last CTA of a unit to arrive):
// O = sum_s 2^(m_s - M) l_s O^_s 2^e_s / sum_s 2^(m_s - M) l_s with M = max_s m_s
// and O^_s the stored FP16 row of split s. Splits are taken four at a time,
// with all their loads issued before any is used: a pass over four chunks
// (32 dims) of up to four splits has 20 loads in flight, so a row costs about
// six L2 round trips instead of one per split and chunk group. Absent splits
// of a group load nothing and weigh 0.
__device__ __noinline__ void merge_row(const AttnArgs& a, int unit, int row, uint16_t* dst, float* lse_dst) {
    const int64_t stride = static_cast<int64_t>(a.heads) * a.pairs * 256; // records between splits
    const float4* ml = a.part_ml + static_cast<int64_t>(unit) * 256 + row;
    const uint4* po = a.part_o + static_cast<int64_t>(unit) * 16 * 256 + row;
    auto load_ml = [&](int s) { return s < a.splits ? __ldcg(ml + s * stride) : make_float4(-INFINITY, 0.f, 0.f, 0.f); };
    float mmax = -INFINITY;
    for (int s0 = 0; s0 < a.splits; s0 += 4) {
        float4 r[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) r[k] = load_ml(s0 + k);
#pragma unroll
        for (int k = 0; k < 4; ++k) mmax = fmaxf(mmax, r[k].x);
    }
    float L = 0.0f;
    for (int s0 = 0; s0 < a.splits; s0 += 4) {
        float4 r[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) r[k] = load_ml(s0 + k);
#pragma unroll
        for (int k = 0; k < 4; ++k) L += r[k].y * exp2f(r[k].x - mmax);
    }
    const float inv = 1.0f / L;
#pragma unroll 1
    for (int c0 = 0; c0 < 16; c0 += 4) {
        float2 acc[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][e] = make_float2(0.0f, 0.0f);
#pragma unroll 1
        for (int s0 = 0; s0 < a.splits; s0 += 4) {
            float4 r[4];
            uint4 o[4][4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const bool on = s0 + k < a.splits;
                r[k] = load_ml(s0 + k);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    o[k][j] = on ? __ldcg(po + (s0 + k) * stride * 16 + (c0 + j) * 256) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float g = exp2f(r[k].x - mmax) * r[k].y * r[k].z;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t w[4] = {o[k][j].x, o[k][j].y, o[k][j].z, o[k][j].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x = f16x2_to_f32x2(w[e]);
                        acc[j][e].x = fmaf(x.x, g, acc[j][e].x);
                        acc[j][e].y = fmaf(x.y, g, acc[j][e].y);
                    }
                }
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
            reinterpret_cast<uint4*>(dst)[c0 + j] =
                make_uint4(pack_bf16x2(acc[j][0].x * inv, acc[j][0].y * inv),
                           pack_bf16x2(acc[j][1].x * inv, acc[j][1].y * inv),
                           pack_bf16x2(acc[j][2].x * inv, acc[j][2].y * inv),
                           pack_bf16x2(acc[j][3].x * inv, acc[j][3].y * inv));
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
__device__ __forceinline__ void drain_armed(const int (&k_armed)[kKStages], const int (&v_armed)[kVStages],
                                            uint32_t kfull0, uint32_t vfull0) {
    for (int st = 0; st < (kKStages > kVStages ? kKStages : kVStages); ++st) {
        const uint64_t t0 = global_timer_ns();
        while ((st < kKStages && k_armed[st] >= 0 && !mbar_try_wait(kfull0 + 8u * st, k_armed[st])) ||
               (st < kVStages && v_armed[st] >= 0 && !mbar_try_wait(vfull0 + 8u * st, v_armed[st]))) {
            if (global_timer_ns() - t0 > NOMAS_WAIT_NS) break;
        }
    }
}

template <int kMode>
__global__ void __launch_bounds__(kMode == kFused ? 512 : 384, 1)
    attn_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap tm_q,
                const __grid_constant__ CUtensorMap tm_kcur, const __grid_constant__ CUtensorMap tm_vcur,
                const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc) {
    constexpr bool kInt8 = kMode != kBf16;   // FP16 Q/K, per-row and per-tile exponents
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
    // cache tiles of this CTA come first: i < nci
    const int nci = max(0, min(t_end, a.tiles_c) - t_begin);

    // ---- setup
    if (threadIdx.x == 0) {
        mbar_init(bar(B_QFULL), 1);
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(bar(B_KFULL + s), 1);
            mbar_init(bar(B_KEMPTY + s), 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(bar(B_VFULL + s), 1);
            mbar_init(bar(B_VEMPTY + s), 1);
        }
        for (int w = 0; w < 2; ++w) {
            mbar_init(bar(B_SFULL + w), 1);
            mbar_init(bar(B_PFULL + w), 4);
            mbar_init(bar(B_OFULL + w), 1);
        }
        mbar_init(bar(B_DRAIN), 1);
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

    if (warp < 4) {
      if constexpr (kFill) regs_dec<kFusedRegsCtl>();
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
            // tile order every parity wait on the stage ring is exact. Otherwise
            // this thread fills the K ring and warp 2 the V ring, so that a K load
            // never queues behind a V stage that is still in use.
            if (!kFill) {
                int k_armed[kKStages], v_armed[kVStages];
                for (int st = 0; st < kKStages; ++st) k_armed[st] = -1;
                for (int st = 0; st < kVStages; ++st) v_armed[st] = -1;
                for (int i = 0; i < n; ++i) {
                    const int ks = i % kKStages;
                    if (i >= kKStages && !mbar_wait(bar(B_KEMPTY + ks), ((i / kKStages) & 1) ^ 1, ctl)) break;
                    load_k_tile(a, t_begin + i, head, sbase + kOffK + ks * kTileBytes, bar(B_KFULL + ks), &tm_kc,
                                &tm_kcur);
                    k_armed[ks] = (i / kKStages) & 1;
                }
                drain_armed(k_armed, v_armed, bar(B_KFULL), bar(B_VFULL));
            }
        }
      } else if (warp == 2) {
        // ================================================================ V producer
        if (!kFill && lane == 0) {
            int k_armed[kKStages], v_armed[kVStages];
            for (int st = 0; st < kKStages; ++st) k_armed[st] = -1;
            for (int st = 0; st < kVStages; ++st) v_armed[st] = -1;
            for (int i = 0; i < n; ++i) {
                const int vs = i % kVStages;
                if (i >= kVStages && !mbar_wait(bar(B_VEMPTY + vs), ((i / kVStages) & 1) ^ 1, ctl)) break;
                load_v_tile(a, t_begin + i, head, sbase + kOffV + vs * kTileBytes, bar(B_VFULL + vs), &tm_vc,
                            &tm_vcur);
                v_armed[vs] = (i / kVStages) & 1;
            }
            drain_armed(k_armed, v_armed, bar(B_KFULL), bar(B_VFULL));
        }
      } else if (warp == 1) {
        // ================================================================ MMA issuer
        // The whole warp runs the loop (warp-uniform waits and conditions) and
        // one elected lane issues each MMA and commit; MMAs issued by a single
        // lane in a divergent branch run at little more than half the
        // tensor-core rate whenever a branch separates two groups of them.
        using I = Issuer;
        constexpr uint32_t idesc_qk = idesc_f32(BM, BN, false, false, kInt8);
        constexpr uint32_t idesc_pv_c = idesc_f32(BM, kD, false, true, kInt8); // cache tiles
        constexpr uint32_t idesc_pv_q = idesc_f32(BM, kD, false, true, false); // current tiles: BF16 V
        // TMEM columns: S of Q tile w at 128 w, O of Q tile w at 256 + 128 w
        auto tm_s = [&](int w) { return tmem + 128u * static_cast<uint32_t>(w); };
        auto tm_o = [&](int w) { return tmem + 256u + 128u * static_cast<uint32_t>(w); };
        bool ok = I::wait(bar(B_QFULL), 0, ctl);
        tc_fence_after();
        // k-step-0 descriptors of the Q tiles and of the K and V stages (scalars:
        // selected, not indexed, so they stay in registers)
        // a K or V stage's descriptor is stage 0's plus the stage offset in the
        // 16-byte address field (shared addresses < 256 KB: no carry)
        const uint64_t q_desc0 = desc_kmajor(sbase + kOffQ, 0), q_desc1 = desc_kmajor(sbase + kOffQ + kTileBytes, 0);
        const uint64_t k_desc0 = desc_kmajor(sbase + kOffK, 0);
        const uint64_t v_desc0 = desc_mnmajor(sbase + kOffV, 0);
        auto issue_s = [&](int w, int st) {
            const uint64_t qd = w ? q_desc1 : q_desc0;
            const uint64_t kd = k_desc0 + static_cast<uint64_t>(st) * (kTileBytes >> 4);
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk)
                I::ss(tm_s(w), qd + kstep_kmajor(kk), kd + kstep_kmajor(kk), idesc_qk, kk > 0 ? 1u : 0u);
        };
        auto issue_pv = [&](int w, int st, bool first_tile, uint32_t idesc_pv) {
            const uint64_t vd = v_desc0 + static_cast<uint64_t>(st) * (kTileBytes >> 4);
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
            // K of tile 0 is free once these S MMAs finish (a later fill waits for it)
            if (kKStages < n) I::commit(bar(B_KEMPTY + 0));
        }
        // Loads are awaited right after a group of MMAs has been issued (the tensor
        // core has queued work meanwhile), never between two groups: V of the next
        // tile and K of the tile after it at the end of each tile, so within a tile
        // only the two P waits separate the groups.
        if (ok) ok = I::wait(bar(B_VFULL + 0), 0, ctl);
        if (ok && n > 1) ok = I::wait(bar(B_KFULL + 1 % kKStages), (1 / kKStages) & 1, ctl);
        tc_fence_after();
        for (int i = 0; ok && i < n; ++i) {
            const int st = i % kVStages;            // V stage of tile i
            const int st1 = (i + 1) % kKStages;     // K stage of tile i + 1
            const bool last = (i + 1 == n);
            const uint32_t idesc_pv = i < nci ? idesc_pv_c : idesc_pv_q;
            for (int w = 0; w < nq_tiles; ++w) {
                if (!(ok = I::wait(bar(B_PFULL + w), i & 1, ctl))) break;
                tc_fence_after();
                issue_pv(w, st, i == 0, idesc_pv);
                // each release is committed only when a later fill waits for it,
                // so no arrival is left pending at exit
                if (w == nq_tiles - 1 && i + kVStages < n) I::commit(bar(B_VEMPTY + st));
                if (!last) {
                    issue_s(w, st1);
                    I::commit(bar(B_SFULL + w));
                    if (w == nq_tiles - 1 && i + 1 + kKStages < n) I::commit(bar(B_KEMPTY + st1));
                } else {
                    I::commit(bar(B_OFULL + w));
                }
            }
            if (!ok) break;
            if (i + 1 < n && !(ok = I::wait(bar(B_VFULL + (i + 1) % kVStages), ((i + 1) / kVStages) & 1, ctl)))
                break;
            if (i + 2 < n && !(ok = I::wait(bar(B_KFULL + (i + 2) % kKStages), ((i + 2) / kKStages) & 1, ctl)))
                break;
            tc_fence_after();
        }
        // drain: every MMA issued above has completed before teardown
        I::commit(bar(B_DRAIN));
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bar(B_DRAIN), 0)) {
            if (global_timer_ns() - t0 > NOMAS_WAIT_NS) break;
        }
      }
    } else if (warp < 12) {
        if constexpr (kFill) regs_inc<kFusedRegsSoftmax>();
        // ================================================================ softmax
        const int w = (warp - 4) >> 2;
        const int quad = warp & 3;
        const int r = quad * 32 + lane; // row inside the Q tile
        const bool active = (w == 0 || has_q1);
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t t_s = tmem + lane_off + w * 128;
        const uint32_t t_o = tmem + lane_off + 256 + w * 128;
        const int qrow = (qt0 + w) * BM + r;
        float m_ref = -INFINITY; // reference max, log2 units (INT8: of x + c_T)
        float l = 0.0f;
        bool ok = true;
        if (active) {
            // per-row score coefficient: log2(e)/sqrt(128), times 2^a_i for FP16 Q
            float qc = a.scale_log2;
            if (kInt8 && qrow < a.nq) qc *= __ldg(a.qs + static_cast<int64_t>(head) * a.nq + qrow);
            const float4* te = kInt8 ? a.te + static_cast<int64_t>(head) * t_total : nullptr;
            // INT8: the record of the next tile, read one tile ahead (its load
            // completes while this warp waits for the tile's scores)
            float4 rec_next = kInt8 ? __ldg(te + t_begin) : make_float4(1.0f, 1.0f, 0.0f, 1.0f);
            for (int i = 0; ok && i < n; ++i) {
                const int t = t_begin + i;
                const float4 rec = rec_next;
                if (kInt8 && i + 1 < n) rec_next = __ldg(te + t + 1);
                const bool f16 = kInt8 && i < nci; // P in FP16 for cache tiles (warp-uniform)
                if (!(ok = mbar_wait(bar(B_SFULL + w), i & 1, ctl))) break;
                tc_fence_after();
                const int vc = tile_valid(a, t);
                const bool full = (vc == BN);
                // x = s * c (c > 0), u = x + c_T: the tile's max of u is exact
                const float c = qc * rec.x;
                const float mx = full ? row_max<false>(t_s, vc) : row_max_masked(t_s, vc);
                const float hi = mx * c + rec.z;
                const bool up = hi > m_ref + kRescaleThreshold;
                const float m_new = up ? hi : m_ref;
                const float alpha = up ? ex2_approx(m_ref - m_new) : 1.0f; // 0 on the first tile
                if (i > 0 && __any_sync(0xFFFFFFFFu, up)) rescale_o(t_o, alpha);
                l *= alpha;
                m_ref = m_new;
                // pass 2: P into TMEM, row sum in fp32 (scaled back by 2^-c_T)
                const float b = rec.z - m_ref;
                float ps;
                if (f16)
                    ps = full ? row_exp_store_full<kFill ? kExp2PolyPairsFused : kExp2PolyPairs, true>(t_s, c, b)
                              : row_exp_store_masked(t_s, c, b, vc, true);
                else
                    ps = full ? row_exp_store_full<kFill ? kExp2PolyPairsFused : kExp2PolyPairs, false>(t_s, c, b)
                              : row_exp_store_masked(t_s, c, b, vc, false);
                l += kInt8 ? ps * rec.w : ps;
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_PFULL + w));
            }
            // ---- epilogue
            if (ok) ok = mbar_wait(bar(B_OFULL + w), 0, ctl);
        }
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
                const float sc = store_partial_row(t_o, 1.0f / l, a.part_o + pu * 16 * 256 + prow);
                a.part_ml[pu * 256 + prow] = make_float4(m_ref, l, sc, 0.0f);
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
        if constexpr (kFill) regs_dec<kFusedRegsFill>();
        // ================================================================ INT8 filler
        // Warp wq converts rows [32 wq, 32 wq + 32) of a cache tile; in step j a
        // warp covers rows 2j and 2j+1, 16 lanes per row, 8 codes per lane, so a
        // lane writes exactly one 16-byte FP16 chunk and each quarter-warp hits 8
        // distinct chunk slots of the swizzled row (no bank conflicts). Filler
        // thread f (0..127) also loads the K and V scales of key f of the tile
        // and forms its FP16 factors r = RN16(scale * 2^-e) with the tile's
        // exponents. The next cache tile's codes are loaded into registers as
        // soon as the current tile has been converted, so global latency
        // overlaps the MMAs.
        const int f = threadIdx.x - 384;
        const int wq = warp - 12;
        const int half = lane >> 4;
        const int l16 = lane & 15;
        const bool elected = (f == 0);
        const uint32_t chunk_off = (l16 >> 3) * kHalfBytes;
        const float4* te = a.te + static_cast<int64_t>(head) * t_total;
        uint2 kb[16], vb[16];
        float ks_own = 0.0f, vs_own = 0.0f; // scales of key f of the tile whose codes are in kb / vb
        float4 rec = make_float4(1.0f, 1.0f, 0.0f, 1.0f);
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
            const int64_t g = static_cast<int64_t>(head) * a.cap_tok + key;
            const bool key_ok = key < a.nc;
            ks_own = key_ok ? __ldg(a.ksc + g) : 0.0f;
            vs_own = key_ok ? __ldg(a.vsc + g) : 0.0f;
            rec = __ldg(te + t);
        };
        // codes of the rows of step j times the factor of that row (held by lane 2j + half)
        auto convert = [&](uint32_t tile, const uint2 (&buf)[16], float r_own) {
            const uint32_t rbits = f16x2_splat(r_own);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint32_t r2 = __shfl_sync(0xFFFFFFFFu, rbits, 2 * j + half);
                const uint32_t off = row_off0 + j * 256u + ((slot0 ^ static_cast<uint32_t>((2 * j) & 7)) << 4);
                st_shared_v4(tile + off, codes_to_f16(buf[j], r2));
            }
        };
        // one elected thread waits; the group learns the outcome after a named
        // barrier, so all 128 threads take the same branch
        auto group_wait = [&](uint32_t barrier, uint32_t parity) -> bool {
            if (elected) *dq_go = mbar_wait(barrier, parity, ctl) ? 1 : 0;
            named_bar_sync(1, 128);
            return *dq_go != 0;
        };
        int k_armed[kKStages], v_armed[kVStages];
        for (int st = 0; st < kKStages; ++st) k_armed[st] = -1;
        for (int st = 0; st < kVStages; ++st) v_armed[st] = -1;
        if (nci > 0) {
            load_codes(a.kc8, t_begin, kb);
            load_codes(a.vc8, t_begin, vb);
            load_scales(t_begin);
        }
        for (int i = 0; i < n; ++i) {
            const int t = t_begin + i;
            const int ks = i % kKStages, vs = i % kVStages;
            const uint32_t ktile = sbase + kOffK + ks * kTileBytes;
            const uint32_t vtile = sbase + kOffV + vs * kTileBytes;
            const bool cached = i < nci;
            const bool next_cached = i + 1 < nci;
            // ---- K (freed early: right after the S MMAs of tile i - kKStages)
            if (i >= kKStages && !group_wait(bar(B_KEMPTY + ks), ((i / kKStages) & 1) ^ 1)) break;
            if (!cached) {
                if (elected) {
                    load_k_tile(a, t, head, ktile, bar(B_KFULL + ks), &tm_kc, &tm_kcur);
                    k_armed[ks] = (i / kKStages) & 1;
                }
            } else {
                convert(ktile, kb, ks_own * rec.y);
                if (next_cached) load_codes(a.kc8, t + 1, kb);
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (elected) mbar_arrive(bar(B_KFULL + ks));
            }
            // ---- V (freed after the P.V MMAs of tile i - kVStages)
            if (i >= kVStages && !group_wait(bar(B_VEMPTY + vs), ((i / kVStages) & 1) ^ 1)) break;
            if (!cached) {
                if (elected) {
                    load_v_tile(a, t, head, vtile, bar(B_VFULL + vs), &tm_vc, &tm_vcur);
                    v_armed[vs] = (i / kVStages) & 1;
                }
            } else {
                convert(vtile, vb, vs_own * rec.w);
                if (next_cached) {
                    load_codes(a.vc8, t + 1, vb);
                    load_scales(t + 1);
                }
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (elected) mbar_arrive(bar(B_VFULL + vs));
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

// One warp per (tensor, head, 128-key tile): the tile's exponent from the
// maximum of its 128 scales (4 per lane, a shuffle reduction), then 32 steps of
// 4 rows: lane l moves the 16 codes [16 (l & 7), 16 (l & 7) + 16) of row
// 4 step + l / 8 (512 contiguous bytes of codes in, 1 KB of FP16 out per
// step). Each row's factor RN16(scale * 2^-e) comes from the lane that loaded
// its scale. Every key of the visible window is written; the tile record the
// attention kernel reads is written by the RoPE prep kernel from the same
// scales with the same exponent function.
__global__ void __launch_bounds__(256, 1) dequant_window_kernel(const __grid_constant__ DequantArgs a) {
    // Launched dependent on the RoPE prep kernel and overlapping it: it reads
    // only the cache, which was complete before prep started. It lets the
    // attention kernel launch early, and before it exits it waits for prep, so
    // the attention kernel's wait on it covers prep too.
    grid_dep_launch();
    const int lane = threadIdx.x & 31;
    const int tasks = 2 * a.heads * a.tiles_c;
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    for (int task = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < tasks; task += nwarps) {
        const bool is_v = task >= a.heads * a.tiles_c;
        const int tv = is_v ? task - a.heads * a.tiles_c : task;
        const int head = tv / a.tiles_c;
        const int T = tv - head * a.tiles_c;
        const float* sc = (is_v ? a.vs : a.ks) + static_cast<int64_t>(head) * a.cap_tok + T * 128;
        const int keys = min(128, a.nc - T * 128);
        float own[4];
        float mx = 0.0f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            own[q] = (q * 32 + lane < keys) ? __ldg(sc + q * 32 + lane) : 0.0f;
            mx = fmaxf(mx, own[q]);
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
        const float inv = exp2_int(-pow2_exponent(mx, kTopCode));
        const int8_t* src = (is_v ? a.vc : a.kc) + (static_cast<int64_t>(head) * a.cap_tok + T * 128) * kD;
        uint16_t* dst = (is_v ? a.vd : a.kd) + (static_cast<int64_t>(head) * a.nc + T * 128) * kD;
        const int part = lane & 7;
        // rows 32 q .. 32 q + 31 have their scales in register own[q]
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll 4
            for (int k = 0; k < 8; ++k) {
                const int row = 32 * q + 4 * k + (lane >> 3);
                const float s_row = __shfl_sync(0xFFFFFFFFu, own[q], row & 31);
                if (row < keys) {
                    const uint4 w = __ldg(reinterpret_cast<const uint4*>(src + row * kD) + part);
                    const uint32_t r2 = f16x2_splat(s_row * inv);
                    uint4* d = reinterpret_cast<uint4*>(dst + row * kD) + 2 * part;
                    d[0] = codes_to_f16(make_uint2(w.x, w.y), r2);
                    d[1] = codes_to_f16(make_uint2(w.z, w.w), r2);
                }
            }
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
    if (kMode == kFused) {
        // the register budgets assume the kernel launches at kFusedRegsLaunch
        // registers per thread
        cudaFuncAttributes fa{};
        if ((e = cudaFuncGetAttributes(&fa, attn_kernel<kMode>)) != cudaSuccess) return e;
        if (fa.numRegs != static_cast<int>(kFusedRegsLaunch)) return cudaErrorInvalidConfiguration;
    }
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
    const uint64_t tasks = 2ull * static_cast<uint64_t>(a.heads) * static_cast<uint64_t>(a.tiles_c);
    if (tasks == 0) return cudaSuccess;
    uint64_t blocks = (tasks + 7) / 8;
    const uint64_t cap = 148ull * 8ull; // persistent: 8 blocks of 256 threads per SM
    if (blocks > cap) blocks = cap;
    return launch_dependent(dequant_window_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, a);
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
