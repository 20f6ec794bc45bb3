// C ABI of the library (declared in include/nomas.h): argument and state
// validation, RoPE tables, TMA descriptors, split selection and launches.
// Every check runs before the first launch, so an error return leaves the
// stream and the cache untouched.
#include "nomas_internal.h"

#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>

using namespace nomas;

namespace {

constexpr int kBM = 128;
constexpr int kAssumedSms = 148;       // split choice is a pure function of the shape
constexpr size_t kWsHeader = 256;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

uint64_t fnv(uint64_t h, const void* p, size_t n) {
    const auto* b = static_cast<const uint8_t*>(p);
    for (size_t i = 0; i < n; ++i) {
        h ^= b[i];
        h *= 0x100000001B3ull;
    }
    return h;
}

uint64_t config_stamp(const nomas_cache* c) {
    uint64_t h = 0xCBF29CE484222325ull;
    h = fnv(h, &c->mode, sizeof(int32_t) * 7);
    h = fnv(h, &c->rope_theta, sizeof(float));
    h = fnv(h, &c->k, sizeof(void*) * 2);
    h = fnv(h, &c->k_scale, sizeof(float*) * 2);
    return h | 1ull; // never 0, so a zeroed descriptor never validates
}

int validate_config(const nomas_cache* c) {
    if (!c) return NOMAS_ERR_ARG;
    if (c->mode != NOMAS_CACHE_BF16 && c->mode != NOMAS_CACHE_INT8) return NOMAS_ERR_ARG;
    if (c->heads <= 0 || c->head_dim != NOMAS_HEAD_DIM) return NOMAS_ERR_ARG;
    if (c->grid_h <= 0 || c->grid_w <= 0 || c->grid_h + c->grid_w > NOMAS_MAX_GRID_HW) return NOMAS_ERR_ARG;
    if (c->capacity_frames <= 0 || c->window_frames < 0) return NOMAS_ERR_ARG;
    if (c->window_frames > 0 && c->capacity_frames != c->window_frames) return NOMAS_ERR_ARG;
    if (!(c->rope_theta > 0.0f) || !std::isfinite(c->rope_theta)) return NOMAS_ERR_ARG;
    const int64_t tpf = static_cast<int64_t>(c->grid_h) * c->grid_w;
    if (static_cast<int64_t>(c->capacity_frames) * tpf > (int64_t(1) << 31) - 1) return NOMAS_ERR_ARG;
    if (!c->k || !c->v) return NOMAS_ERR_ARG;
    if (c->mode == NOMAS_CACHE_INT8 && (!c->k_scale || !c->v_scale)) return NOMAS_ERR_ARG;
    if (c->mode == NOMAS_CACHE_BF16 && (c->k_scale || c->v_scale)) return NOMAS_ERR_ARG;
    if (!aligned(c->k, 16) || !aligned(c->v, 16)) return NOMAS_ERR_ALIGN;
    if (c->mode == NOMAS_CACHE_INT8 && (!aligned(c->k_scale, 16) || !aligned(c->v_scale, 16))) return NOMAS_ERR_ALIGN;
    return NOMAS_OK;
}

int validate_state(const nomas_cache* c) {
    int rc = validate_config(c);
    if (rc != NOMAS_OK) return rc;
    if (c->check != config_stamp(c)) return NOMAS_ERR_STATE;
    if (c->frames_committed < 0 || c->valid_frames < 0 || c->valid_frames > c->capacity_frames)
        return NOMAS_ERR_STATE;
    return NOMAS_OK;
}

// ---------------------------------------------------------------- RoPE tables
// c, s = fp32 roundings of the double-precision cos/sin of pos * theta^(-2j/d).
double inv_freq(double theta, int j, int d) { return pow(theta, -2.0 * static_cast<double>(j) / static_cast<double>(d)); }

float2 rope_cs(double pos, double theta, int j, int d) {
    const double ang = pos * inv_freq(theta, j, d);
    return make_float2(static_cast<float>(cos(ang)), static_cast<float>(sin(ang)));
}

// Device address of the spatial rows (grid rows, then grid columns) of a
// configuration; computed here and uploaded by rope_hw_device on first use.
int spatial_rows(float theta, int gh, int gw, const float2** dev) {
    RopeHW h;
    for (int r = 0; r < gh; ++r)
        for (int j = 0; j < kHWPairs; ++j) h.hw[r][j] = rope_cs(static_cast<double>(r), theta, j, 56);
    for (int col = 0; col < gw; ++col)
        for (int j = 0; j < kHWPairs; ++j) h.hw[gh + col][j] = rope_cs(static_cast<double>(col), theta, j, 56);
    const cudaError_t e = rope_hw_device(h, theta, gh, gw, dev);
    if (e == cudaErrorMemoryAllocation) return NOMAS_ERR_ARG; // too many distinct configurations on this device
    return e == cudaSuccess ? NOMAS_OK : NOMAS_ERR_CUDA;
}

void fill_t(RopeTab& tab, float theta, int64_t abs_frame0, int n_frames) {
    for (int i = 0; i < n_frames; ++i)
        for (int j = 0; j < kTPairs; ++j) tab.t[i][j] = rope_cs(static_cast<double>(abs_frame0 + i), theta, j, 16);
}

// ---------------------------------------------------------------- device checks
int check_device() {
    static std::mutex mu;
    static int ok_dev[64] = {0}; // 0 unknown, 1 ok, -1 bad
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NOMAS_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (ok_dev[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return NOMAS_ERR_CUDA;
        ok_dev[dev] = (major == 10 && minor == 0) ? 1 : -1;
    }
    return ok_dev[dev] == 1 ? NOMAS_OK : NOMAS_ERR_DEVICE;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 3D BF16 tensor map, 128B swizzle, box {64, b1, b2}; out-of-range rows read as zero.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
               uint64_t stride2_bytes, uint32_t b1, uint32_t b2) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    const cuuint32_t box[3] = {64, b1, b2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- attention plan
struct Plan {
    int64_t tpf, nv, nq, nc;
    int tiles_c, tiles_q, pairs, splits, tiles_per_split;
    bool window;  // INT8 cache read through an FP16 copy of its visible window
    size_t off_qt, off_kt, off_te, off_qs, off_po, off_pml, off_cnt, off_kd, off_vd;
    size_t total; // workspace bytes of this plan
};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Split count minimising a makespan model: waves x (tiles per split + fixed
// per-CTA cost), for a 148-SM part with one CTA per SM; at most max_splits.
void choose_splits(int units, int tiles, int max_splits, int& splits, int& tps) {
    double best = 1e300;
    splits = 1;
    tps = tiles > 0 ? tiles : 1;
    if (tiles <= 0) return;
    for (int s = 1; s <= max_splits; ++s) {
        const int t = (tiles + s - 1) / s;
        const int s_eff = (tiles + t - 1) / t;
        if (s > 1 && t < 4) break;
        const int64_t ctas = static_cast<int64_t>(units) * s_eff;
        const int64_t waves = (ctas + kAssumedSms - 1) / kAssumedSms;
        const double cost = static_cast<double>(waves) * (t + 3.0) + (s_eff > 1 ? 2.0 : 0.0);
        if (cost < best - 1e-9) {
            best = cost;
            splits = s_eff;
            tps = t;
        }
    }
}

// The window copy's dequantisation kernel counts its (tensor, head, tile)
// tasks and the attention kernel its tiles in 32 bits.
bool window_copy_fits(int heads, int64_t nc) { return static_cast<int64_t>(heads) * nc < (int64_t(1) << 27); }

// Workspace layout of a plan: status header, rotated Q and K (head-major; BF16,
// or FP16 for an INT8 cache); for an INT8 cache the tile records
// [heads][tiles_c + tiles_q] float4 and the Q row factors [heads][nq] fp32;
// with splits > 1 the split partials [splits][units][16][256] (8 FP16 dims per
// 16-byte word), their (max, sum, 2^e) records [splits][units][256] float4 and
// one arrival counter per unit; with
// the window form the FP16 copy of the visible window, K then V [heads][nc][128].
Plan make_plan(const nomas_cache* c, int32_t n_video_frames, int32_t n_text, int max_splits, bool window) {
    Plan p{};
    p.tpf = static_cast<int64_t>(c->grid_h) * c->grid_w;
    p.nv = static_cast<int64_t>(n_video_frames) * p.tpf;
    p.nq = p.nv + n_text;
    p.nc = static_cast<int64_t>(c->valid_frames) * p.tpf;
    p.tiles_c = static_cast<int>((p.nc + kBM - 1) / kBM);
    p.tiles_q = static_cast<int>((p.nq + kBM - 1) / kBM);
    p.pairs = (p.tiles_q + 1) / 2;
    p.window = window;
    const int units = c->heads * p.pairs;
    choose_splits(units, p.tiles_c + p.tiles_q, max_splits, p.splits, p.tiles_per_split);
    const size_t qk_bytes = static_cast<size_t>(c->heads) * p.nq * kD * 2;
    const size_t prow = static_cast<size_t>(p.splits) * units * 2 * kBM;
    const bool sp = p.splits > 1;
    const bool int8 = c->mode == NOMAS_CACHE_INT8;
    p.off_qt = kWsHeader;
    p.off_kt = round_up(p.off_qt + qk_bytes, 256);
    p.off_te = round_up(p.off_kt + qk_bytes, 256);
    p.off_qs = round_up(p.off_te + (int8 ? static_cast<size_t>(c->heads) * (p.tiles_c + p.tiles_q) * 16 : 0), 256);
    p.off_po = round_up(p.off_qs + (int8 ? static_cast<size_t>(c->heads) * p.nq * 4 : 0), 256);
    p.off_pml = p.off_po + (sp ? prow * kD * 2 : 0);
    p.off_cnt = round_up(p.off_pml + (sp ? prow * 16 : 0), 256);
    p.off_kd = p.off_vd = p.total = round_up(p.off_cnt + (sp ? static_cast<size_t>(units) * sizeof(unsigned) : 0), 256);
    if (window) {
        const size_t copy = round_up(static_cast<size_t>(c->heads) * p.nc * kD * 2, 256);
        p.off_vd = p.off_kd + copy;
        p.total = p.off_vd + copy;
    }
    return p;
}

constexpr int kMaxSplits = 32;

// An INT8 cache with a visible history can use the window form.
bool window_form(const nomas_cache* c) {
    const int64_t nc = static_cast<int64_t>(c->valid_frames) * c->grid_h * c->grid_w;
    return c->mode == NOMAS_CACHE_INT8 && nc > 0 && window_copy_fits(c->heads, nc);
}

// The fastest plan whose workspace fits in `bytes`: for an INT8 cache the
// window form before the in-shared-memory form, and within a form more splits
// before fewer (fewer need less room: splits = 1 keeps no partials). False
// when nothing fits.
bool fit_plan(const nomas_cache* c, int32_t n_video_frames, int32_t n_text, size_t bytes, Plan& out) {
    for (int form = window_form(c) ? 1 : 0; form >= 0; --form) {
        int cap = kMaxSplits;
        while (true) {
            out = make_plan(c, n_video_frames, n_text, cap, form == 1);
            if (out.total <= bytes) return true;
            if (out.splits <= 1) break;
            cap = out.splits - 1;
        }
    }
    return false;
}

} // namespace

extern "C" {

int nomas_cache_reset(nomas_cache* c) {
    const int rc = validate_config(c);
    if (rc != NOMAS_OK) return rc;
    c->frames_committed = 0;
    c->valid_frames = 0;
    c->head_slot = 0;
    c->check = config_stamp(c);
    return NOMAS_OK;
}

// Commit of one finished segment into n layer caches that share configuration
// and state (the single-layer call is n == 1). Everything is validated before
// anything is enqueued; the host counters of every cache advance together.
static int commit_layers(nomas_cache* const* cs, const void* const* ks, const void* const* vs, int64_t token_stride,
                         int32_t n_layers, int32_t n_frames, void* stream) {
    if (!cs || n_layers < 1) return NOMAS_ERR_ARG;
    for (int i = 0; i < n_layers; ++i)
        if (!cs[i]) return NOMAS_ERR_ARG;
    const nomas_cache* c = cs[0];
    int rc = validate_state(c);
    if (rc != NOMAS_OK) return rc;
    for (int i = 1; i < n_layers; ++i) {
        const nomas_cache* o = cs[i];
        if ((rc = validate_state(o)) != NOMAS_OK) return rc;
        if (o->mode != c->mode || o->heads != c->heads || o->grid_h != c->grid_h || o->grid_w != c->grid_w ||
            o->window_frames != c->window_frames || o->capacity_frames != c->capacity_frames ||
            o->rope_theta != c->rope_theta || o->frames_committed != c->frames_committed ||
            o->valid_frames != c->valid_frames || o->head_slot != c->head_slot)
            return NOMAS_ERR_STATE;
        for (int j = 0; j < i; ++j)
            if (cs[j] == o || cs[j]->k == o->k || cs[j]->v == o->v) return NOMAS_ERR_ARG; // one cache twice
    }
    if (n_frames < 0) return NOMAS_ERR_ARG;
    if (n_frames == 0) return NOMAS_OK;
    if (!ks || !vs) return NOMAS_ERR_ARG;
    if (token_stride < static_cast<int64_t>(c->heads) * kD || token_stride % 8 != 0) return NOMAS_ERR_ARG;
    for (int i = 0; i < n_layers; ++i) {
        if (!ks[i] || !vs[i]) return NOMAS_ERR_ARG;
        if (!aligned(ks[i], 16) || !aligned(vs[i], 16)) return NOMAS_ERR_ALIGN;
    }
    const int W = c->window_frames;
    if (W == 0 && c->frames_committed + n_frames > c->capacity_frames) return NOMAS_ERR_CAPACITY;
    const int64_t layers_per_launch = n_layers < kMaxLayersPerLaunch ? n_layers : kMaxLayersPerLaunch;
    if (static_cast<int64_t>(kMaxFramesPerLaunch) * c->grid_h * c->grid_w * c->heads * layers_per_launch >=
        (int64_t(1) << 31))
        return NOMAS_ERR_ARG; // one launch's (layer, token, head) rows must fit 31 bits
    if ((rc = check_device()) != NOMAS_OK) return rc;

    const int tpf = c->grid_h * c->grid_w;
    const int first = (W > 0 && n_frames > W) ? n_frames - W : 0;
    const float2* hw = nullptr;
    if ((rc = spatial_rows(c->rope_theta, c->grid_h, c->grid_w, &hw)) != NOMAS_OK) return rc;
    RopeTab tab;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    for (int f0 = first; f0 < n_frames; f0 += kMaxFramesPerLaunch) {
        const int nf = (n_frames - f0) < kMaxFramesPerLaunch ? (n_frames - f0) : kMaxFramesPerLaunch;
        CommitArgs a{};
        a.token_stride = token_stride;
        a.cap_tok = static_cast<int64_t>(c->capacity_frames) * tpf;
        a.heads = c->heads;
        a.tpf = tpf;
        a.grid_h = c->grid_h;
        a.grid_w = c->grid_w;
        a.n_frames = nf;
        a.in_frame0 = f0;
        a.abs_frame0 = c->frames_committed + f0;
        a.window = W;
        a.slot0 = W > 0 ? static_cast<int32_t>(a.abs_frame0 % W) : 0;
        a.int8_mode = c->mode == NOMAS_CACHE_INT8;
        a.div_heads = make_fastdiv(static_cast<uint32_t>(c->heads));
        a.div_tpf = make_fastdiv(static_cast<uint32_t>(tpf));
        a.div_gw = make_fastdiv(static_cast<uint32_t>(c->grid_w));
        a.hw = hw;
        fill_t(tab, c->rope_theta, a.abs_frame0, nf);
        // launches of equal size when the layers need more than one
        const int n_launch = (n_layers + kMaxLayersPerLaunch - 1) / kMaxLayersPerLaunch;
        const int per_launch = (n_layers + n_launch - 1) / n_launch;
        for (int l0 = 0; l0 < n_layers; l0 += per_launch) {
            const int nl = (n_layers - l0) < per_launch ? (n_layers - l0) : per_launch;
            CommitLayers L{};
            for (int i = 0; i < nl; ++i) {
                const nomas_cache* ci = cs[l0 + i];
                L.l[i].k = static_cast<const uint16_t*>(ks[l0 + i]);
                L.l[i].v = static_cast<const uint16_t*>(vs[l0 + i]);
                L.l[i].ck = ci->k;
                L.l[i].cv = ci->v;
                L.l[i].cks = ci->k_scale;
                L.l[i].cvs = ci->v_scale;
            }
            a.n_layers = nl;
            if (launch_commit(a, L, tab, s) != cudaSuccess) return NOMAS_ERR_CUDA;
        }
    }
    for (int i = 0; i < n_layers; ++i) {
        nomas_cache* ci = cs[i];
        ci->frames_committed += n_frames;
        if (W > 0) {
            ci->valid_frames = static_cast<int32_t>(ci->frames_committed < W ? ci->frames_committed : W);
            ci->head_slot = static_cast<int32_t>(ci->frames_committed % W);
        } else {
            ci->valid_frames = static_cast<int32_t>(ci->frames_committed);
            ci->head_slot = static_cast<int32_t>(ci->frames_committed);
        }
    }
    return NOMAS_OK;
}

int nomas_kv_commit(nomas_cache* c, const void* k, const void* v, int64_t token_stride, int32_t n_frames,
                    void* stream) {
    return commit_layers(&c, &k, &v, token_stride, 1, n_frames, stream);
}

int nomas_kv_commit_layers(nomas_cache* const* caches, const void* const* k, const void* const* v,
                           int64_t token_stride, int32_t n_layers, int32_t n_frames, void* stream) {
    return commit_layers(caches, k, v, token_stride, n_layers, n_frames, stream);
}

// ------------------------------------------- camera cross-attention per frame
int nomas_camera_attn(const void* q, int64_t q_stride, int32_t n_frames, int32_t tokens_per_frame, int32_t heads,
                      const void* k_cam, const void* v_cam, int32_t n_cam, int32_t chunk_frames, void* out,
                      int64_t out_stride, void* stream) {
    if (n_frames < 0 || tokens_per_frame <= 0 || heads <= 0 || n_cam < 1 || n_cam > NOMAS_MAX_CAMERA_TOKENS ||
        chunk_frames < 1)
        return NOMAS_ERR_ARG;
    const int64_t rows = static_cast<int64_t>(n_frames) * tokens_per_frame * heads;
    if (rows > (int64_t(1) << 31) - 1) return NOMAS_ERR_ARG;
    if (rows == 0) return NOMAS_OK;
    if (!q || !k_cam || !v_cam || !out) return NOMAS_ERR_ARG;
    const int64_t row_elems = static_cast<int64_t>(heads) * kD;
    if (q_stride < row_elems || out_stride < row_elems) return NOMAS_ERR_ARG;
    if (q_stride % 8 != 0 || out_stride % 8 != 0) return NOMAS_ERR_ALIGN;
    if (!aligned(q, 16) || !aligned(k_cam, 16) || !aligned(v_cam, 16) || !aligned(out, 16)) return NOMAS_ERR_ALIGN;
    int rc = check_device();
    if (rc != NOMAS_OK) return rc;
    CamArgs a{};
    a.q = static_cast<const uint16_t*>(q);
    a.q_stride = q_stride;
    a.k_cam = static_cast<const uint16_t*>(k_cam);
    a.v_cam = static_cast<const uint16_t*>(v_cam);
    a.out = static_cast<uint16_t*>(out);
    a.out_stride = out_stride;
    a.rows = rows;
    a.heads = heads;
    a.n_cam = n_cam;
    a.div_heads = make_fastdiv(static_cast<uint32_t>(heads));
    a.div_tpf = make_fastdiv(static_cast<uint32_t>(tokens_per_frame));
    a.div_chunk = make_fastdiv(static_cast<uint32_t>(chunk_frames));
    a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kD)));
    return launch_camera_attn(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? NOMAS_OK : NOMAS_ERR_CUDA;
}

// ------------------------------------------------- archive of evicted frames
// A commit of n frames into a window of W leaves the last min(W, committed)
// frames of the whole sequence in the window. The frames it drops are those of
// the current window [committed - valid, committed) that precede the new
// window's first frame: consecutive, oldest first.
static void evicted_range(const nomas_cache* c, int32_t n_frames, int32_t* count, int64_t* first) {
    const int64_t fc = c->frames_committed, W = c->window_frames;
    *first = fc - c->valid_frames;
    *count = 0;
    if (W == 0 || n_frames <= 0) return;
    const int64_t after = fc + n_frames;
    const int64_t kept_from = after - (after < W ? after : W);
    const int64_t end = fc < kept_from ? fc : kept_from;
    if (end > *first) *count = static_cast<int32_t>(end - *first);
}

int nomas_kv_evicted_frames(const nomas_cache* c, int32_t n_frames, int32_t* count, int64_t* first_frame) {
    int rc = validate_state(c);
    if (rc != NOMAS_OK) return rc;
    if (n_frames < 0 || !count || !first_frame) return NOMAS_ERR_ARG;
    evicted_range(c, n_frames, count, first_frame);
    return NOMAS_OK;
}

int nomas_kv_archive_evicted(const nomas_cache* c, int32_t n_frames, void* host_k, void* host_v,
                             float* host_k_scale, float* host_v_scale, int32_t max_frames, int32_t* count,
                             int64_t* first_frame, void* stream) {
    int rc = validate_state(c);
    if (rc != NOMAS_OK) return rc;
    if (n_frames < 0 || max_frames < 0 || !count || !first_frame) return NOMAS_ERR_ARG;
    evicted_range(c, n_frames, count, first_frame);
    const int32_t m = *count;
    if (m > max_frames) return NOMAS_ERR_CAPACITY;
    if (m == 0) return NOMAS_OK;
    const bool int8 = c->mode == NOMAS_CACHE_INT8;
    if (!host_k || !host_v || (int8 && (!host_k_scale || !host_v_scale))) return NOMAS_ERR_ARG;
    if ((rc = check_device()) != NOMAS_OK) return rc;
    // One frame of one head is tokens_per_frame consecutive rows of that head's
    // slab, so a frame is `heads` equal runs pitched by the slab: one 2D copy per
    // frame and tensor, gathered by the copy engine into the frame-major archive.
    const size_t tpf = static_cast<size_t>(c->grid_h) * c->grid_w;
    const size_t cap_tok = static_cast<size_t>(c->capacity_frames) * tpf;
    const size_t es = int8 ? 1 : 2;
    const size_t run = tpf * kD * es, pitch = cap_tok * kD * es;
    const size_t srun = tpf * sizeof(float), spitch = cap_tok * sizeof(float);
    const size_t H = static_cast<size_t>(c->heads);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    for (int32_t i = 0; i < m; ++i) {
        const size_t slot = static_cast<size_t>((*first_frame + i) % c->window_frames);
        const auto d2h = [&](void* dst, size_t dst_frame_bytes, const void* src, size_t width, size_t src_pitch) {
            return cudaMemcpy2DAsync(static_cast<char*>(dst) + static_cast<size_t>(i) * dst_frame_bytes, width,
                                     static_cast<const char*>(src) + slot * width, src_pitch, width, H,
                                     cudaMemcpyDeviceToHost, s);
        };
        if (d2h(host_k, H * run, c->k, run, pitch) != cudaSuccess ||
            d2h(host_v, H * run, c->v, run, pitch) != cudaSuccess)
            return NOMAS_ERR_CUDA;
        if (int8 && (d2h(host_k_scale, H * srun, c->k_scale, srun, spitch) != cudaSuccess ||
                     d2h(host_v_scale, H * srun, c->v_scale, srun, spitch) != cudaSuccess))
            return NOMAS_ERR_CUDA;
    }
    return NOMAS_OK;
}

size_t nomas_seg_attn_workspace_bytes(const nomas_cache* c, int32_t n_video_frames, int32_t n_text) {
    if (validate_state(c) != NOMAS_OK || n_video_frames < 0 || n_text < 0) return 0;
    return make_plan(c, n_video_frames, n_text, kMaxSplits, window_form(c)).total;
}

size_t nomas_seg_attn_workspace_min_bytes(const nomas_cache* c, int32_t n_video_frames, int32_t n_text) {
    if (validate_state(c) != NOMAS_OK || n_video_frames < 0 || n_text < 0) return 0;
    return make_plan(c, n_video_frames, n_text, 1, false).total;
}

int nomas_seg_attn(const nomas_cache* c, const void* q, const void* k, const void* v, int64_t token_stride,
                   int32_t n_video_frames, int32_t n_text, void* out, float* lse, void* workspace,
                   size_t workspace_bytes, void* stream) {
    int rc = validate_state(c);
    if (rc != NOMAS_OK) return rc;
    if (n_video_frames < 0 || n_text < 0) return NOMAS_ERR_ARG;
    Plan p = make_plan(c, n_video_frames, n_text, 1, false);
    if (p.nq == 0) return NOMAS_OK;
    if (p.nq > (int64_t(1) << 30) || p.nq * c->heads >= (int64_t(1) << 31)) return NOMAS_ERR_ARG;
    if (!q || !k || !v || !out) return NOMAS_ERR_ARG;
    if (token_stride < static_cast<int64_t>(c->heads) * kD || token_stride % 8 != 0) return NOMAS_ERR_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return NOMAS_ERR_ALIGN;
    if (lse && !aligned(lse, 4)) return NOMAS_ERR_ALIGN;
    if (!workspace || !fit_plan(c, n_video_frames, n_text, workspace_bytes, p)) return NOMAS_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return NOMAS_ERR_ALIGN;
    if ((rc = check_device()) != NOMAS_OK) return rc;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint16_t* qt = reinterpret_cast<uint16_t*>(ws + p.off_qt);
    uint16_t* kt = reinterpret_cast<uint16_t*>(ws + p.off_kt);
    unsigned* counters = reinterpret_cast<unsigned*>(ws + p.off_cnt);
    float4* te = reinterpret_cast<float4*>(ws + p.off_te);
    float* qs = reinterpret_cast<float*>(ws + p.off_qs);
    const int units = c->heads * p.pairs;
    const bool int8 = c->mode == NOMAS_CACHE_INT8;
    const int64_t cap_tok = static_cast<int64_t>(c->capacity_frames) * p.tpf;

    // 1) RoPE + relayout of the current Q and K (video frames in chunks); the
    //    first launch also zeroes the split-KV arrival counters and, for an
    //    INT8 cache, writes the cache tiles' records
    const float2* hw = nullptr;
    if ((rc = spatial_rows(c->rope_theta, c->grid_h, c->grid_w, &hw)) != NOMAS_OK) return rc;
    RopeTab tab;
    {
        int f0 = 0;
        do {
            const int nf = (n_video_frames - f0) < kMaxFramesPerLaunch ? (n_video_frames - f0) : kMaxFramesPerLaunch;
            PrepArgs a{};
            a.q = static_cast<const uint16_t*>(q);
            a.k = static_cast<const uint16_t*>(k);
            a.token_stride = token_stride;
            a.qt = qt;
            a.kt = kt;
            a.heads = c->heads;
            a.tpf = static_cast<int32_t>(p.tpf);
            a.grid_h = c->grid_h;
            a.grid_w = c->grid_w;
            a.nq = static_cast<int32_t>(p.nq);
            a.nv = static_cast<int32_t>(p.nv);
            a.tok0 = static_cast<int32_t>(f0 * p.tpf);
            const bool last = f0 + nf >= n_video_frames;
            a.tok1 = last ? static_cast<int32_t>(p.nq) : static_cast<int32_t>((f0 + nf) * p.tpf);
            a.frame0 = f0;
            a.div_heads = make_fastdiv(static_cast<uint32_t>(c->heads));
            a.div_tpf = make_fastdiv(static_cast<uint32_t>(p.tpf));
            a.div_gw = make_fastdiv(static_cast<uint32_t>(c->grid_w));
            a.counters = counters;
            a.n_counters = (f0 == 0 && p.splits > 1) ? units : 0;
            a.hw = hw;
            if (int8) {
                a.te = te;
                a.qs = qs;
                a.ksc = c->k_scale;
                a.vsc = c->v_scale;
                a.cap_tok = cap_tok;
                a.nc = static_cast<int32_t>(p.nc);
                a.tiles_c = p.tiles_c;
                a.tiles_q = p.tiles_q;
                a.te_cache_tasks = f0 == 0 ? c->heads * p.tiles_c : 0;
            }
            if (nf > 0) fill_t(tab, c->rope_theta, c->frames_committed + f0, nf);
            if (a.tok1 > a.tok0 && launch_prep(a, tab, s) != cudaSuccess) return NOMAS_ERR_CUDA;
            f0 += nf;
            if (last) break;
        } while (true);
    }

    // 2) an INT8 window is dequantised once into its FP16 copy (window form)
    uint16_t* kd = reinterpret_cast<uint16_t*>(ws + p.off_kd);
    uint16_t* vd = reinterpret_cast<uint16_t*>(ws + p.off_vd);
    if (p.window) {
        DequantArgs d{};
        d.kc = static_cast<const int8_t*>(c->k);
        d.vc = static_cast<const int8_t*>(c->v);
        d.ks = c->k_scale;
        d.vs = c->v_scale;
        d.kd = kd;
        d.vd = vd;
        d.cap_tok = cap_tok;
        d.nc = static_cast<int32_t>(p.nc);
        d.heads = c->heads;
        d.tiles_c = p.tiles_c;
        if (launch_dequant_window(d, s) != cudaSuccess) return NOMAS_ERR_CUDA;
    }

    // 3) tensor maps
    CUtensorMap tm_q, tm_kcur, tm_vcur, tm_kc, tm_vc;
    const uint64_t row_bytes = kD * 2;
    bool ok = make_tmap(&tm_q, qt, kD, p.nq, c->heads, row_bytes, p.nq * row_bytes, kBM, 1) &&
              make_tmap(&tm_kcur, kt, kD, p.nq, c->heads, row_bytes, p.nq * row_bytes, kBM, 1) &&
              make_tmap(&tm_vcur, v, kD, c->heads, p.nq, row_bytes, token_stride * 2, 1, kBM);
    if (!int8) {
        const uint64_t nc_ext = p.nc > 0 ? p.nc : 1;
        ok = ok && make_tmap(&tm_kc, c->k, kD, nc_ext, c->heads, row_bytes, cap_tok * row_bytes, kBM, 1) &&
             make_tmap(&tm_vc, c->v, kD, nc_ext, c->heads, row_bytes, cap_tok * row_bytes, kBM, 1);
    } else if (p.window) {
        ok = ok && make_tmap(&tm_kc, kd, kD, p.nc, c->heads, row_bytes, p.nc * row_bytes, kBM, 1) &&
             make_tmap(&tm_vc, vd, kD, p.nc, c->heads, row_bytes, p.nc * row_bytes, kBM, 1);
    } else {
        tm_kc = tm_q; // unused: the fused form converts cache tiles itself
        tm_vc = tm_q;
    }
    if (!ok) return NOMAS_ERR_CUDA;

    // 3) attention; with splits > 1 the last CTA of each unit merges the splits
    AttnArgs a{};
    a.heads = c->heads;
    a.nq = static_cast<int32_t>(p.nq);
    a.nc = static_cast<int32_t>(p.nc);
    a.tiles_c = p.tiles_c;
    a.tiles_q = p.tiles_q;
    a.pairs = p.pairs;
    a.splits = p.splits;
    a.tiles_per_split = p.tiles_per_split;
    a.cap_tok = cap_tok;
    a.kc8 = static_cast<const int8_t*>(c->k);
    a.vc8 = static_cast<const int8_t*>(c->v);
    a.ksc = c->k_scale;
    a.vsc = c->v_scale;
    a.out = static_cast<uint16_t*>(out);
    a.lse = lse;
    a.part_o = reinterpret_cast<uint4*>(ws + p.off_po);
    a.part_ml = reinterpret_cast<float4*>(ws + p.off_pml);
    a.counters = counters;
    a.err = reinterpret_cast<unsigned*>(ws);
    a.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(kD)));
    a.te = int8 ? te : nullptr;
    a.qs = int8 ? qs : nullptr;
    const AttnForm form = !int8 ? AttnForm::kBf16Cache : p.window ? AttnForm::kInt8Window : AttnForm::kInt8Fused;
    if (launch_attn(a, form, tm_q, tm_kcur, tm_vcur, tm_kc, tm_vc, s) != cudaSuccess) return NOMAS_ERR_CUDA;
    return NOMAS_OK;
}

int nomas_device_status(void* workspace, void* stream) {
    if (!workspace) return NOMAS_ERR_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return NOMAS_ERR_CUDA;
    unsigned word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return NOMAS_ERR_CUDA;
    if (word == 0) return NOMAS_OK;
    if (cudaMemset(workspace, 0, sizeof(word)) != cudaSuccess) return NOMAS_ERR_CUDA;
    return NOMAS_ERR_DEVICE_TIMEOUT;
}

const char* nomas_status_string(int status) {
    switch (status) {
    case NOMAS_OK: return "NOMAS_OK";
    case NOMAS_ERR_ARG: return "NOMAS_ERR_ARG: invalid argument";
    case NOMAS_ERR_ALIGN: return "NOMAS_ERR_ALIGN: pointer or stride not aligned";
    case NOMAS_ERR_STATE: return "NOMAS_ERR_STATE: cache descriptor not reset or changed";
    case NOMAS_ERR_CAPACITY: return "NOMAS_ERR_CAPACITY: full-history cache is full";
    case NOMAS_ERR_WORKSPACE: return "NOMAS_ERR_WORKSPACE: workspace missing or too small";
    case NOMAS_ERR_CUDA: return "NOMAS_ERR_CUDA: CUDA call failed";
    case NOMAS_ERR_DEVICE: return "NOMAS_ERR_DEVICE: current device is not sm_100";
    case NOMAS_ERR_DEVICE_TIMEOUT: return "NOMAS_ERR_DEVICE_TIMEOUT: a kernel abandoned a bounded wait";
    default: return "unknown nomas status";
    }
}

} // extern "C"
