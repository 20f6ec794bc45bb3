// Segment-causal joint attention on sm_100a tensor cores.
//
// What it computes (Hy-Nomas model card, "Segment-Autoregressive Diffusion
// Transformer"; blog "Segment-wise causal joint attention"): for each head
// and each query token of the current segment, softmax attention over the
// visible cached tokens of earlier segments followed by every token of the
// current segment (no mask inside a segment; causality across segments is
// structural: later segments are never in the cache). INT8 caches are
// dequantised to BF16 in shared memory (model card, "Single-GPU Low-Memory
// Inference": INT8 KV storage, BF16 attention computation).
//
// Structure of one CTA (one "unit" = two 128-row Q tiles of one head, and a
// contiguous range of 128-key KV tiles: cache tiles first, then the current
// segment's tiles):
//   warp 0      TMA producer: Q tiles once, then (BF16 caches) every K/V tile
//               into a 2-stage ring
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//   warps 4-7   softmax warpgroup for Q tile 0 (one thread per query row)
//   warps 8-11  softmax warpgroup for Q tile 1
//   warps 12-15 INT8 caches only: the one filler of the K/V ring -- cache
//               tiles are dequantised (codes + scales from global memory ->
//               BF16 in the 128B-swizzled stage layout), current-segment tiles
//               are loaded by TMA. One filler in tile order keeps every parity
//               wait on the ring exact.
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each; the BF16
// probabilities P overwrite the first 64 columns of their S block and feed
// the P.V product straight from TMEM (A operand in tensor memory).
// MMA order per KV tile j: PV0(j-1) S0(j) | PV1(j-1) S1(j) -- while one
// softmax warpgroup exponentiates, the tensor core works for the other.
// Online softmax in base 2 with lazy rescaling: the running reference max is
// raised only when a tile's max exceeds it by more than 8 (so P <= 256), and
// only then is O rescaled in TMEM.
// Split-KV: with splits > 1 each CTA leaves (O unnormalised, max, sum) in the
// workspace and combine_kernel merges them.
#include "nomas_internal.h"
#include "nomas_ptx.cuh"

namespace nomas {

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kStages = 2;
constexpr uint32_t kTileBytes = BM * kD * 2; // one BF16 128x128 tile
constexpr uint32_t kHalfBytes = kTileBytes / 2;
constexpr float kRescaleThreshold = 8.0f;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;                                // 2 tiles
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;           // kStages tiles
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;     // kStages tiles
constexpr uint32_t kOffBar = kOffV + kStages * kTileBytes;   // barriers
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;        // + alignment slack

// barrier slots (8 bytes each)
enum {
    B_QFULL = 0,
    B_KFULL = 1,                // + stage
    B_VFULL = B_KFULL + kStages,
    B_KVEMPTY = B_VFULL + kStages,
    B_SFULL = B_KVEMPTY + kStages, // + softmax warpgroup
    B_PFULL = B_SFULL + 2,
    B_OFULL = B_PFULL + 2,
    B_DRAIN = B_OFULL + 2,
    B_COUNT
};
constexpr uint32_t kOffTmemSlot = B_COUNT * 8;
constexpr uint32_t kOffAbort = kOffTmemSlot + 8;
constexpr uint32_t kOffDqGo = kOffAbort + 4;
static_assert(kOffDqGo + 4 <= 256, "barrier area overflow");

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

__device__ __forceinline__ float dq(uint32_t biased_word, int byte, float scale) {
    // byte of an offset-binary word -> exact float code -> times scale
    const float f = __uint_as_float(__byte_perm(biased_word, 0x4B000000u, 0x7540u + byte)) - 8388736.0f;
    return f * scale;
}

// Arm stage `st` for tile t and issue its K and V loads (4 TMA boxes).
__device__ __forceinline__ void load_kv_tile(const AttnArgs& a, int t, int head, uint32_t kdst, uint32_t vdst,
                                             uint32_t kbar, uint32_t vbar, const CUtensorMap* tm_kc,
                                             const CUtensorMap* tm_vc, const CUtensorMap* tm_kcur,
                                             const CUtensorMap* tm_vcur) {
    mbar_arrive_expect_tx(kbar, kTileBytes);
    mbar_arrive_expect_tx(vbar, kTileBytes);
    if (t < a.tiles_c) {
        tma_load_3d(kdst, tm_kc, 0, t * BN, head, kbar);
        tma_load_3d(kdst + kHalfBytes, tm_kc, 64, t * BN, head, kbar);
        tma_load_3d(vdst, tm_vc, 0, t * BN, head, vbar);
        tma_load_3d(vdst + kHalfBytes, tm_vc, 64, t * BN, head, vbar);
    } else {
        const int row = (t - a.tiles_c) * BN;
        tma_load_3d(kdst, tm_kcur, 0, row, head, kbar);
        tma_load_3d(kdst + kHalfBytes, tm_kcur, 64, row, head, kbar);
        tma_load_3d(vdst, tm_vcur, 0, head, row, vbar);
        tma_load_3d(vdst + kHalfBytes, tm_vcur, 64, head, row, vbar);
    }
}

// Bounded wait for the last armed phase of each stage: no copy may still be
// in flight when the CTA exits (matters only after an abort).
__device__ __forceinline__ void drain_armed(const int (&armed_phase)[kStages], uint32_t kfull0, uint32_t vfull0) {
    for (int st = 0; st < kStages; ++st) {
        if (armed_phase[st] < 0) continue;
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(kfull0 + 8u * st, armed_phase[st]) || !mbar_try_wait(vfull0 + 8u * st, armed_phase[st])) {
            if (global_timer_ns() - t0 > NOMAS_WAIT_NS) break;
        }
    }
}

template <bool kInt8>
__global__ void __launch_bounds__(kInt8 ? 512 : 384, 1)
    attn_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap tm_q,
                const __grid_constant__ CUtensorMap tm_kcur, const __grid_constant__ CUtensorMap tm_vcur,
                const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + kOffBar;
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kOffBar + kOffTmemSlot);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffBar + kOffAbort);
    volatile int* dq_go = reinterpret_cast<volatile int*>(smem + kOffBar + kOffDqGo);
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
    const int t_total = a.tiles_c + a.tiles_q;
    const int t_begin = split * a.tiles_per_split;
    int t_end = t_begin + a.tiles_per_split;
    if (t_end > t_total) t_end = t_total;
    const int n = t_end - t_begin; // >= 1 by construction of the split count

    // ---- setup
    if (threadIdx.x == 0) {
        mbar_init(bar(B_QFULL), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(B_KFULL + s), 1);
            mbar_init(bar(B_VFULL + s), 1);
            mbar_init(bar(B_KVEMPTY + s), 1);
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

    if (warp == 0) {
        // ================================================================ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_kcur);
            tma_prefetch_desc(&tm_vcur);
            if (!kInt8) {
                tma_prefetch_desc(&tm_kc);
                tma_prefetch_desc(&tm_vc);
            }
            mbar_arrive_expect_tx(bar(B_QFULL), (has_q1 ? 2u : 1u) * kTileBytes);
            for (int w = 0; w < (has_q1 ? 2 : 1); ++w) {
                const uint32_t dst = sbase + kOffQ + w * kTileBytes;
                tma_load_3d(dst, &tm_q, 0, (qt0 + w) * BM, head, bar(B_QFULL));
                tma_load_3d(dst + kHalfBytes, &tm_q, 64, (qt0 + w) * BM, head, bar(B_QFULL));
            }
            // An INT8 cache has one filler for every stage, the dequantiser warpgroup
            // (codes for cache tiles, TMA for current-segment tiles): with a single
            // filler in tile order every parity wait on the stage ring is exact.
            if (!kInt8) {
                int armed_phase[kStages] = {-1, -1};
                for (int i = 0; i < n; ++i) {
                    const int st = i % kStages;
                    if (i >= kStages && !mbar_wait(bar(B_KVEMPTY + st), ((i / kStages) & 1) ^ 1, ctl)) break;
                    load_kv_tile(a, t_begin + i, head, sbase + kOffK + st * kTileBytes, sbase + kOffV + st * kTileBytes,
                                 bar(B_KFULL + st), bar(B_VFULL + st), &tm_kc, &tm_vc, &tm_kcur, &tm_vcur);
                    armed_phase[st] = (i / kStages) & 1;
                }
                drain_armed(armed_phase, bar(B_KFULL), bar(B_VFULL));
            }
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, kD, false, true);
            const uint32_t q_tile[2] = {sbase + kOffQ, sbase + kOffQ + kTileBytes};
            const uint32_t tm_s[2] = {tmem, tmem + 128};
            const uint32_t tm_o[2] = {tmem + 256, tmem + 384};
            const int nq_tiles = has_q1 ? 2 : 1;
            bool ok = mbar_wait(bar(B_QFULL), 0, ctl);
            tc_fence_after();
            auto issue_s = [&](int w, int st) {
                const uint32_t ktile = sbase + kOffK + st * kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    mma_ss(tm_s[w], desc_kmajor(q_tile[w], kk), desc_kmajor(ktile, kk), idesc_qk, kk > 0 ? 1u : 0u);
            };
            auto issue_pv = [&](int w, int st, bool first_tile) {
                const uint32_t vtile = sbase + kOffV + st * kTileBytes;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    mma_ts(tm_o[w], tm_s[w] + kk * 8, desc_mnmajor(vtile, kk), idesc_pv,
                           (first_tile && kk == 0) ? 0u : 1u);
            };
            if (ok) ok = mbar_wait(bar(B_KFULL + 0), 0, ctl);
            if (ok) {
                tc_fence_after();
                for (int w = 0; w < nq_tiles; ++w) {
                    issue_s(w, 0);
                    mma_commit(bar(B_SFULL + w));
                }
            }
            for (int i = 0; ok && i < n; ++i) {
                const int st = i % kStages;
                const uint32_t ph = (i / kStages) & 1;
                const int st1 = (i + 1) % kStages;
                const uint32_t ph1 = ((i + 1) / kStages) & 1;
                const bool last = (i + 1 == n);
                if (!(ok = mbar_wait(bar(B_VFULL + st), ph, ctl))) break;
                if (!last && !(ok = mbar_wait(bar(B_KFULL + st1), ph1, ctl))) break;
                for (int w = 0; w < nq_tiles; ++w) {
                    if (!(ok = mbar_wait(bar(B_PFULL + w), i & 1, ctl))) break;
                    tc_fence_after();
                    issue_pv(w, st, i == 0);
                    if (w == nq_tiles - 1 && !last) mma_commit(bar(B_KVEMPTY + st));
                    if (!last) {
                        issue_s(w, st1);
                        mma_commit(bar(B_SFULL + w));
                    } else {
                        mma_commit(bar(B_OFULL + w));
                    }
                }
            }
            // drain: every MMA issued above has completed before teardown
            mma_commit(bar(B_DRAIN));
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar(B_DRAIN), 0)) {
                if (global_timer_ns() - t0 > NOMAS_WAIT_NS) break;
            }
        }
    } else if (warp >= 4 && warp < 12) {
        // ================================================================ softmax
        const int w = (warp - 4) >> 2;
        const int quad = warp & 3;
        const int r = quad * 32 + lane; // row inside the Q tile
        if (w == 0 || has_q1) {
            const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
            const uint32_t t_s = tmem + lane_off + w * 128;
            const uint32_t t_o = tmem + lane_off + 256 + w * 128;
            const float sl2 = a.scale_log2;
            float m_ref = -INFINITY; // reference max, log2 units
            float l = 0.0f;
            bool ok = true;
            for (int i = 0; i < n; ++i) {
                if (!(ok = mbar_wait(bar(B_SFULL + w), i & 1, ctl))) break;
                tc_fence_after();
                const int vc = tile_valid(a, t_begin + i);
                // pass 1: row max of the raw scores
                float mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t s[32];
                    tmem_ld32(t_s + c * 32, s);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float x = __uint_as_float(s[e]);
                        mx = (c * 32 + e < vc) ? fmaxf(mx, x) : mx;
                    }
                }
                const float mxl = mx * sl2;
                const bool resc = mxl > m_ref + kRescaleThreshold;
                const float m_new = resc ? mxl : m_ref;
                const float alpha = resc ? ex2_approx(m_ref - m_new) : 1.0f; // 0 on the first tile
                if (i > 0 && __any_sync(0xFFFFFFFFu, resc)) {
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        tmem_ld32(t_o + c * 32, o);
    #pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(t_o + c * 32, o);
                    }
                    tmem_st_wait();
                }
                l *= alpha;
                m_ref = m_new;
                // pass 2: P = 2^(s*scale - m), BF16, into the first 64 columns of S
                const float neg_m = -m_ref;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t s[32];
                    tmem_ld32(t_s + c * 32, s);
                    uint32_t p[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int col = c * 32 + 2 * e;
                        float p0 = ex2_approx(fmaf(__uint_as_float(s[2 * e]), sl2, neg_m));
                        float p1 = ex2_approx(fmaf(__uint_as_float(s[2 * e + 1]), sl2, neg_m));
                        p0 = col < vc ? p0 : 0.0f;
                        p1 = col + 1 < vc ? p1 : 0.0f;
                        l += p0 + p1;
                        p[e] = pack_bf16x2(p0, p1);
                    }
                    // P columns [16c, 16c+16): S columns below 32(c+1) are already in registers
                    asm volatile(
                        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
                        "%11, %12, %13, %14, %15, %16};" ::"r"(t_s + c * 16),
                        "r"(p[0]), "r"(p[1]), "r"(p[2]), "r"(p[3]), "r"(p[4]), "r"(p[5]), "r"(p[6]), "r"(p[7]),
                        "r"(p[8]), "r"(p[9]), "r"(p[10]), "r"(p[11]), "r"(p[12]), "r"(p[13]), "r"(p[14]),
                        "r"(p[15])
                        : "memory");
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_PFULL + w));
            }
            // ---- epilogue
            if (ok) ok = mbar_wait(bar(B_OFULL + w), 0, ctl);
            if (ok) {
                tc_fence_after();
                const int qrow = (qt0 + w) * BM + r;
                const bool row_ok = qrow < a.nq;
                if (a.splits == 1) {
                    const float inv_l = 1.0f / l;
                    uint16_t* dst = a.out + (static_cast<int64_t>(qrow) * a.heads + head) * kD;
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
                    if (row_ok && a.lse) a.lse[static_cast<int64_t>(head) * a.nq + qrow] = (m_ref + log2f(l)) * 0.69314718055994531f;
                } else {
                    const int64_t prow = (static_cast<int64_t>(split) * a.heads + head) * (a.pairs * 2 * BM) +
                                         static_cast<int64_t>(pair) * 2 * BM + w * BM + r;
                    float* dst = a.part_o + prow * kD;
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        tmem_ld32(t_o + c * 32, o);
                            if (row_ok) {
                            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                            for (int e = 0; e < 8; ++e) d4[e] = make_uint4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
                        }
                    }
                    if (row_ok) a.part_ml[prow] = make_float2(m_ref, l);
                }
            }
        }
    } else if (kInt8 && warp >= 12) {
        // ================================================================ INT8 dequantiser
        const int wq = warp - 12;
        const int sub = lane >> 3;   // row inside a group of 4
        const int chunk = lane & 7;  // 16-code chunk of the row
        const bool elected = (wq == 0 && lane == 0);
        int armed_phase[kStages] = {-1, -1};
        for (int i = 0; i < n; ++i) {
            const int t = t_begin + i;
            const int st = i % kStages;
            if (i >= kStages) {
                // one elected thread waits; the group learns the outcome after a
                // named barrier, so all 128 threads take the same branch
                if (elected) *dq_go = mbar_wait(bar(B_KVEMPTY + st), ((i / kStages) & 1) ^ 1, ctl) ? 1 : 0;
                named_bar_sync(1, 128);
                if (!*dq_go) break;
            }
            const uint32_t ktile = sbase + kOffK + st * kTileBytes;
            const uint32_t vtile = sbase + kOffV + st * kTileBytes;
            if (t >= a.tiles_c) {
                // current-segment tile: BF16 already, one TMA issue by the elected thread
                if (elected) {
                    load_kv_tile(a, t, head, ktile, vtile, bar(B_KFULL + st), bar(B_VFULL + st), &tm_kc, &tm_vc,
                                 &tm_kcur, &tm_vcur);
                    armed_phase[st] = (i / kStages) & 1;
                }
                continue;
            }
#pragma unroll 2
            for (int it = 0; it < 8; ++it) {
                const int row = wq * 32 + it * 4 + sub;
                const int key = t * BN + row;
                uint4 kc = make_uint4(0, 0, 0, 0), vcw = make_uint4(0, 0, 0, 0);
                float ks = 0.0f, vs = 0.0f;
                if (key < a.nc) {
                    const int64_t grow = static_cast<int64_t>(head) * a.cap_tok + key;
                    kc = __ldg(reinterpret_cast<const uint4*>(a.kc8 + grow * kD) + chunk);
                    vcw = __ldg(reinterpret_cast<const uint4*>(a.vc8 + grow * kD) + chunk);
                    ks = __ldg(a.ksc + grow);
                    vs = __ldg(a.vsc + grow);
                }
                const uint32_t kw[4] = {kc.x ^ 0x80808080u, kc.y ^ 0x80808080u, kc.z ^ 0x80808080u, kc.w ^ 0x80808080u};
                const uint32_t vw[4] = {vcw.x ^ 0x80808080u, vcw.y ^ 0x80808080u, vcw.z ^ 0x80808080u,
                                        vcw.w ^ 0x80808080u};
                uint32_t kb[8], vb[8];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    kb[2 * q] = pack_bf16x2(dq(kw[q], 0, ks), dq(kw[q], 1, ks));
                    kb[2 * q + 1] = pack_bf16x2(dq(kw[q], 2, ks), dq(kw[q], 3, ks));
                    vb[2 * q] = pack_bf16x2(dq(vw[q], 0, vs), dq(vw[q], 1, vs));
                    vb[2 * q + 1] = pack_bf16x2(dq(vw[q], 2, vs), dq(vw[q], 3, vs));
                }
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {
                    const int c8 = 2 * chunk + hc; // 8-dim chunk, 0..15
                    const uint32_t off = (c8 >> 3) * kHalfBytes + row * 128 + (((c8 & 7) ^ (row & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(ktile + off), "r"(kb[4 * hc]),
                                 "r"(kb[4 * hc + 1]), "r"(kb[4 * hc + 2]), "r"(kb[4 * hc + 3])
                                 : "memory");
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(vtile + off), "r"(vb[4 * hc]),
                                 "r"(vb[4 * hc + 1]), "r"(vb[4 * hc + 2]), "r"(vb[4 * hc + 3])
                                 : "memory");
                }
            }
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (elected) {
                mbar_arrive(bar(B_KFULL + st));
                mbar_arrive(bar(B_VFULL + st));
            }
        }
        if (elected) drain_armed(armed_phase, bar(B_KFULL), bar(B_VFULL));
    }

    // ---- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

__global__ void __launch_bounds__(256) combine_kernel(const __grid_constant__ CombineArgs a) {
    // one warp per (head, query row); each lane owns 4 of the 128 dims
    const int64_t gw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= static_cast<int64_t>(a.heads) * a.nq) return;
    const int head = static_cast<int>(gw / a.nq);
    const int qrow = static_cast<int>(gw % a.nq);
    const int64_t rows_per_head = static_cast<int64_t>(a.pairs) * 2 * BM;
    float mmax = -INFINITY;
    for (int s = 0; s < a.splits; ++s)
        mmax = fmaxf(mmax, a.part_ml[(static_cast<int64_t>(s) * a.heads + head) * rows_per_head + qrow].x);
    float L = 0.0f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < a.splits; ++s) {
        const int64_t prow = (static_cast<int64_t>(s) * a.heads + head) * rows_per_head + qrow;
        const float2 ml = a.part_ml[prow];
        const float wgt = exp2f(ml.x - mmax);
        L += ml.y * wgt;
        const float4 o = reinterpret_cast<const float4*>(a.part_o + prow * kD)[lane];
        acc.x += o.x * wgt;
        acc.y += o.y * wgt;
        acc.z += o.z * wgt;
        acc.w += o.w * wgt;
    }
    const float inv = 1.0f / L;
    uint2 b;
    b.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    b.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(a.out + (static_cast<int64_t>(qrow) * a.heads + head) * kD)[lane] = b;
    if (lane == 0 && a.lse) a.lse[static_cast<int64_t>(head) * a.nq + qrow] = (mmax + log2f(L)) * 0.69314718055994531f;
}

} // namespace

cudaError_t launch_attn(const AttnArgs& a, bool int8_cache, const CUtensorMap& tm_q, const CUtensorMap& tm_kcur,
                        const CUtensorMap& tm_vcur, const CUtensorMap& tm_kc, const CUtensorMap& tm_vc,
                        cudaStream_t s) {
    const int grid = a.heads * a.pairs * a.splits;
    if (int8_cache) {
        static bool attr_set = false;
        if (!attr_set) {
            cudaError_t e = cudaFuncSetAttribute(attn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kSmemBytes);
            if (e != cudaSuccess) return e;
            attr_set = true;
        }
        attn_kernel<true><<<grid, 512, kSmemBytes, s>>>(a, tm_q, tm_kcur, tm_vcur, tm_kc, tm_vc);
    } else {
        static bool attr_set = false;
        if (!attr_set) {
            cudaError_t e = cudaFuncSetAttribute(attn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kSmemBytes);
            if (e != cudaSuccess) return e;
            attr_set = true;
        }
        attn_kernel<false><<<grid, 384, kSmemBytes, s>>>(a, tm_q, tm_kcur, tm_vcur, tm_kc, tm_vc);
    }
    return cudaGetLastError();
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
    const int64_t warps = static_cast<int64_t>(a.heads) * a.nq;
    const int64_t blocks = (warps * 32 + 255) / 256;
    combine_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(a);
    return cudaGetLastError();
}

} // namespace nomas
