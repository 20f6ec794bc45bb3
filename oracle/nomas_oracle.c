/*
 * CPU oracle for segment-causal joint attention over a lifelong K/V cache.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
 * load this file: only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline leg use it. It shares no code, header, table or constant
 * generator with the CUDA library (segment_causal_kv_b200/); its only common
 * ground with it is the seeded input generator in synth/, which holds none
 * of the method's arithmetic.
 *
 * Plain, slow, obviously correct: fp64 attention with a two-pass softmax
 * (max, then sum of exponentials), no tiling, no online rescaling. The cache
 * commit is written in fp32 exactly as specified below so that INT8 codes,
 * fp32 scales and BF16 cache values can be compared bit for bit.
 *
 * What it follows (page titles and sections):
 *  - Hy-Nomas model card, "Segment-Autoregressive Diffusion Transformer":
 *    joint attention of a segment's text and video tokens, 3D RoPE on video
 *    positions, a per-layer K/V cache of earlier segments; architecture
 *    table: 16 heads of 128 dims, RoPE split [16,56,56] over (t,h,w),
 *    theta 256; attention causal across segments, cached K/V reused.
 *  - same card, "Single-GPU Low-Memory Inference": INT8 K/V storage with
 *    BF16 attention math; a GPU history budget of 18 latent frames.
 *  - same card: full history (max_cache_segments=null, no sliding window).
 *  - "Hy-Nomas Explained" blog, "Segment-wise causal joint attention":
 *    causal between segments, bidirectional inside one; RoPE rotates
 *    queries and keys (RoFormer formulation).
 *  - blog "Step 3: The Video Latent": 22 x 40 = 880 tokens per latent frame.
 *  - model card, "Text and Camera Conditioning", and the blog's "Camera
 *    conditioning": video tokens query projected camera features by
 *    cross-attention; with per-chunk camera attention and a chunk of one
 *    latent frame, each latent frame's video tokens see only the camera
 *    tokens of their own chunk (one token per latent frame in the blog's
 *    reading of the 64-d grouped extrinsics).
 *
 * Readings where the pages are silent:
 *  - RoPE pairs are interleaved (2j, 2j+1) inside each axis block; block t
 *    = dims [0,16), h = [16,72), w = [72,128); pair j of a block of width d
 *    turns by pos * theta^(-2j/d). Text tokens are not rotated.
 *  - t is the absolute latent-frame index since the session began; h, w are
 *    grid indices; token order inside a frame is row-major (h, then w);
 *    video tokens come first in a segment, text tokens after them.
 *  - cached keys are stored after rotation; only video tokens are cached.
 *  - no mask inside a segment; every cached token is visible.
 *  - softmax scale 1/sqrt(128).
 *  - commit in fp32: c, s = (float)cos/sin((double)pos * pow(theta, -2j/d));
 *    y0 = fma(x0, c, -(x1*s)), y1 = fma(x0, s, x1*c), products rounded to
 *    fp32. INT8: per (token, head) absmax over 128 dims, scale = absmax/127
 *    (IEEE fp32 division), code = round-half-even(x/scale) clamped to
 *    [-127,127]; absmax 0 gives scale 0 and all codes 0. BF16: RNE of the
 *    rotated fp32 key; V is not rotated.
 *  - eviction: keep the last `window` committed latent frames (FIFO, frame
 *    granularity); frame f lives in slot f mod window. window 0 = keep all
 *    (full history) and commits beyond capacity are an error.
 *  - camera cross-attention: no RoPE, softmax scale 1/sqrt(128), only video
 *    tokens take part; video token i belongs to latent frame i / F and to
 *    chunk (i / F) / chunk_frames; each chunk has n_cam camera tokens.
 *
 * Mode 2 (ORC_MODE_F64) is oracle-only: the cache keeps fp64 rotated keys
 * and exact values, so incremental attention can be compared with a masked
 * full-sequence computation to rounding level.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_D 128
#define ORC_MODE_BF16 0
#define ORC_MODE_INT8 1
#define ORC_MODE_F64 2

typedef struct {
    int32_t mode;
    int32_t heads;
    int32_t grid_h, grid_w;
    int32_t window_frames;   /* 0 = unbounded */
    int32_t capacity_frames; /* slots */
    double theta;
    uint16_t *k_bf16, *v_bf16; /* [H][cap*F][128] */
    int8_t *k_code, *v_code;   /* [H][cap*F][128] */
    float *k_scale, *v_scale;  /* [H][cap*F] */
    double *k_f64, *v_f64;     /* [H][cap*F][128] */
    int64_t *slot_frame;       /* [cap], -1 = empty */
    int64_t frames_committed;
    int32_t valid_frames;
} orc_cache;

/* ------------------------------------------------------------------ */
/* BF16 helpers                                                        */
/* ------------------------------------------------------------------ */

static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* round-half-to-even of an fp32 value to BF16 (inputs are finite) */
uint16_t orc_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
}

/* ------------------------------------------------------------------ */
/* 3D RoPE (architecture table: split [16,56,56], theta 256)            */
/* ------------------------------------------------------------------ */

/* Axis block of dimension pair p (0..63): returns width d and index j. */
static int pair_axis(int p, int *d, int *j) {
    if (p < 8) { *d = 16; *j = p; return 0; }
    if (p < 36) { *d = 56; *j = p - 8; return 1; }
    *d = 56; *j = p - 36; return 2;
}

/* Rotation angle of pair j in a block of width d at integer position pos. */
double orc_rope_angle(int d, int j, double pos, double theta) {
    double inv_freq = pow(theta, -2.0 * (double)j / (double)d);
    return pos * inv_freq;
}

/* fp32 cos/sin used by the bit-exact commit: double libm, rounded once. */
void orc_rope_cs_f32(int d, int j, double pos, double theta, float *c, float *s) {
    double a = orc_rope_angle(d, j, pos, theta);
    *c = (float)cos(a);
    *s = (float)sin(a);
}

/* Position (t,h,w) of video token n of a segment whose first frame is t0. */
static void video_pos(int64_t n, int64_t t0, int gh, int gw, double pos[3]) {
    int64_t F = (int64_t)gh * gw;
    int64_t frame = n / F, r = n % F;
    pos[0] = (double)(t0 + frame);
    pos[1] = (double)(r / gw);
    pos[2] = (double)(r % gw);
    (void)gh;
}

/* cos/sin (double) of the 64 pairs at position pos: cs[2p] = cos, cs[2p+1] = sin. */
static void rope_cs_f64_all(const double pos[3], double theta, double *cs) {
    for (int p = 0; p < ORC_D / 2; ++p) {
        int d, j;
        int ax = pair_axis(p, &d, &j);
        double a = orc_rope_angle(d, j, pos[ax], theta);
        cs[2 * p] = cos(a);
        cs[2 * p + 1] = sin(a);
    }
}

static void rotate_f64_cs(const double *x, const double *cs, double *y) {
    for (int p = 0; p < ORC_D / 2; ++p) {
        double c = cs[2 * p], s = cs[2 * p + 1];
        double x0 = x[2 * p], x1 = x[2 * p + 1];
        y[2 * p] = x0 * c - x1 * s;
        y[2 * p + 1] = x0 * s + x1 * c;
    }
}

/* fp64 rotation of one 128-vector at position pos (exact cos/sin). */
void orc_rope_rotate_f64(const double *x, const double pos[3], double theta, double *y) {
    double cs[ORC_D];
    rope_cs_f64_all(pos, theta, cs);
    rotate_f64_cs(x, cs, y);
}

/* fp32 cos/sin of the 64 pairs at position pos (commit table). */
static void rope_cs_f32_all(const double pos[3], double theta, float *cs) {
    for (int p = 0; p < ORC_D / 2; ++p) {
        int d, j;
        int ax = pair_axis(p, &d, &j);
        orc_rope_cs_f32(d, j, pos[ax], theta, &cs[2 * p], &cs[2 * p + 1]);
    }
}

static void rotate_f32_cs(const float *x, const float *cs, float *y) {
    for (int p = 0; p < ORC_D / 2; ++p) {
        float c = cs[2 * p], s = cs[2 * p + 1];
        float x0 = x[2 * p], x1 = x[2 * p + 1];
        float x1s = x1 * s; /* rounded to fp32 (compiled with -ffp-contract=off) */
        float x1c = x1 * c;
        y[2 * p] = fmaf(x0, c, -x1s);
        y[2 * p + 1] = fmaf(x0, s, x1c);
    }
}

/* fp32 rotation with the commit's exact expression. */
void orc_rope_rotate_f32(const float *x, const double pos[3], double theta, float *y) {
    float cs[ORC_D];
    rope_cs_f32_all(pos, theta, cs);
    rotate_f32_cs(x, cs, y);
}

/* ------------------------------------------------------------------ */
/* INT8 quantisation of one (token, head) row                          */
/* ------------------------------------------------------------------ */

void orc_quantize_row(const float *x, int8_t *code, float *scale) {
    float amax = 0.0f;
    for (int i = 0; i < ORC_D; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        *scale = 0.0f;
        memset(code, 0, ORC_D);
        return;
    }
    float s = amax / 127.0f;
    *scale = s;
    for (int i = 0; i < ORC_D; ++i) {
        float r = rintf(x[i] / s); /* default rounding mode: half to even */
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        code[i] = (int8_t)r;
    }
}

/* ------------------------------------------------------------------ */
/* Cache state: reset and commit                                       */
/* ------------------------------------------------------------------ */

int orc_cache_reset(orc_cache *c) {
    if (c->heads <= 0 || c->grid_h <= 0 || c->grid_w <= 0 || c->capacity_frames <= 0) return -1;
    if (c->window_frames < 0) return -1;
    if (c->window_frames > 0 && c->capacity_frames != c->window_frames) return -1;
    for (int s = 0; s < c->capacity_frames; ++s) c->slot_frame[s] = -1;
    c->frames_committed = 0;
    c->valid_frames = 0;
    return 0;
}

/* Commit a finished segment of n_frames latent frames (video tokens only).
 * k, v: BF16 bits, token-major [n_frames*F][H][128], token_stride elements
 * between consecutive tokens. Positions t = frames_committed + i. */
int orc_commit(orc_cache *c, const uint16_t *k, const uint16_t *v, int64_t token_stride, int n_frames) {
    if (n_frames < 0) return -1;
    const int64_t F = (int64_t)c->grid_h * c->grid_w;
    const int H = c->heads;
    const int64_t cap_tok = (int64_t)c->capacity_frames * F;
    const int W = c->window_frames;
    if (W == 0 && c->frames_committed + n_frames > c->capacity_frames) return -2;
    /* frames of this commit that are already outside the window at its end
     * are never stored */
    int first = (W > 0 && n_frames > W) ? n_frames - W : 0;
    float xf[ORC_D], yf[ORC_D];
    double xd[ORC_D], yd[ORC_D];
    for (int i = first; i < n_frames; ++i) {
        int64_t f = c->frames_committed + i;
        int64_t slot = (W > 0) ? (f % W) : f;
        for (int64_t r = 0; r < F; ++r) {
            int64_t n = (int64_t)i * F + r; /* token inside the segment */
            double pos[3];
            video_pos(n, c->frames_committed, c->grid_h, c->grid_w, pos);
            float csf[ORC_D];
            double csd[ORC_D];
            if (c->mode == ORC_MODE_F64)
                rope_cs_f64_all(pos, c->theta, csd);
            else
                rope_cs_f32_all(pos, c->theta, csf);
            for (int h = 0; h < H; ++h) {
                const uint16_t *kr = k + n * token_stride + (int64_t)h * ORC_D;
                const uint16_t *vr = v + n * token_stride + (int64_t)h * ORC_D;
                int64_t row = (int64_t)h * cap_tok + slot * F + r;
                if (c->mode == ORC_MODE_F64) {
                    for (int e = 0; e < ORC_D; ++e) xd[e] = (double)bf16_to_f32(kr[e]);
                    rotate_f64_cs(xd, csd, yd);
                    for (int e = 0; e < ORC_D; ++e) {
                        c->k_f64[row * ORC_D + e] = yd[e];
                        c->v_f64[row * ORC_D + e] = (double)bf16_to_f32(vr[e]);
                    }
                    continue;
                }
                for (int e = 0; e < ORC_D; ++e) xf[e] = bf16_to_f32(kr[e]);
                rotate_f32_cs(xf, csf, yf);
                if (c->mode == ORC_MODE_BF16) {
                    for (int e = 0; e < ORC_D; ++e) {
                        c->k_bf16[row * ORC_D + e] = orc_f32_to_bf16(yf[e]);
                        c->v_bf16[row * ORC_D + e] = vr[e];
                    }
                } else {
                    orc_quantize_row(yf, c->k_code + row * ORC_D, c->k_scale + row);
                    for (int e = 0; e < ORC_D; ++e) xf[e] = bf16_to_f32(vr[e]);
                    orc_quantize_row(xf, c->v_code + row * ORC_D, c->v_scale + row);
                }
            }
        }
        c->slot_frame[slot] = f;
    }
    c->frames_committed += n_frames;
    if (W > 0)
        c->valid_frames = (int32_t)(c->frames_committed < W ? c->frames_committed : W);
    else
        c->valid_frames = (int32_t)c->frames_committed;
    return 0;
}

/* ------------------------------------------------------------------ */
/* fp64 attention                                                      */
/* ------------------------------------------------------------------ */

typedef struct {
    int64_t nk;
    const double *keys; /* [nk][128] */
    const double *vals; /* [nk][128] */
} key_set;

/* Two-pass softmax attention of one rotated query over a key set. */
static void attend_row(const double *q, const key_set *ks, double *o, double *lse, double *scores) {
    const double inv_sqrt_d = 1.0 / sqrt((double)ORC_D);
    double m = -INFINITY;
    for (int64_t j = 0; j < ks->nk; ++j) {
        const double *kj = ks->keys + j * ORC_D;
        double acc = 0.0;
        for (int e = 0; e < ORC_D; ++e) acc += q[e] * kj[e];
        scores[j] = acc * inv_sqrt_d;
        if (scores[j] > m) m = scores[j];
    }
    double den = 0.0;
    for (int e = 0; e < ORC_D; ++e) o[e] = 0.0;
    for (int64_t j = 0; j < ks->nk; ++j) {
        double p = exp(scores[j] - m);
        den += p;
        const double *vj = ks->vals + j * ORC_D;
        for (int e = 0; e < ORC_D; ++e) o[e] += p * vj[e];
    }
    for (int e = 0; e < ORC_D; ++e) o[e] /= den;
    *lse = m + log(den);
}

typedef struct {
    const key_set *ks;
    const double *qrot; /* [nrows][128] */
    int64_t nrows;
    double *o;   /* [nrows][128] */
    double *lse; /* [nrows] */
    int tid, nthreads;
} attend_job;

static void *attend_worker(void *arg) {
    attend_job *jb = (attend_job *)arg;
    double *scores = (double *)malloc(sizeof(double) * (size_t)(jb->ks->nk > 0 ? jb->ks->nk : 1));
    for (int64_t r = jb->tid; r < jb->nrows; r += jb->nthreads)
        attend_row(jb->qrot + r * ORC_D, jb->ks, jb->o + r * ORC_D, jb->lse + r, scores);
    free(scores);
    return NULL;
}

static void attend_rows_parallel(const key_set *ks, const double *qrot, int64_t nrows, double *o, double *lse,
                                 int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    attend_job jobs[256];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = (attend_job){ks, qrot, nrows, o, lse, t, nthreads};
        if (nthreads == 1) {
            attend_worker(&jobs[t]);
        } else {
            pthread_create(&th[t], NULL, attend_worker, &jobs[t]);
        }
    }
    if (nthreads > 1)
        for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
}

/* cos/sin tables of a segment's video tokens: [nv][128] (t0 + frame, h, w). */
static double *segment_cs(int64_t nv, int64_t t0, int gh, int gw, double theta) {
    double *cs = (double *)malloc(sizeof(double) * (size_t)(nv > 0 ? nv : 1) * ORC_D);
    if (!cs) return NULL;
    for (int64_t n = 0; n < nv; ++n) {
        double pos[3];
        video_pos(n, t0, gh, gw, pos);
        rope_cs_f64_all(pos, theta, cs + n * ORC_D);
    }
    return cs;
}

/* Rotated fp64 copy of rows `rows` (NULL: 0..nrows-1) of a segment's tensor
 * for head h: video tokens (index < nv) rotated with the tables `cs`, text
 * tokens unchanged. */
static void rotate_segment(const uint16_t *x, int64_t token_stride, int h, int64_t nv, const int64_t *rows,
                           int64_t nrows, const double *cs, double *out) {
    double tmp[ORC_D];
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t n = rows ? rows[r] : r;
        const uint16_t *xr = x + n * token_stride + (int64_t)h * ORC_D;
        for (int e = 0; e < ORC_D; ++e) tmp[e] = (double)bf16_to_f32(xr[e]);
        if (n < nv)
            rotate_f64_cs(tmp, cs + n * ORC_D, out + r * ORC_D);
        else
            memcpy(out + r * ORC_D, tmp, sizeof(tmp));
    }
}

static void plain_segment(const uint16_t *x, int64_t token_stride, int h, int64_t nq, double *out) {
    for (int64_t n = 0; n < nq; ++n) {
        const uint16_t *xr = x + n * token_stride + (int64_t)h * ORC_D;
        for (int e = 0; e < ORC_D; ++e) out[n * ORC_D + e] = (double)bf16_to_f32(xr[e]);
    }
}

/* Dequantised cache key/value of one slot row (fp64). */
static void cache_row(const orc_cache *c, int64_t row, double *k, double *v) {
    for (int e = 0; e < ORC_D; ++e) {
        switch (c->mode) {
        case ORC_MODE_BF16:
            k[e] = (double)bf16_to_f32(c->k_bf16[row * ORC_D + e]);
            v[e] = (double)bf16_to_f32(c->v_bf16[row * ORC_D + e]);
            break;
        case ORC_MODE_INT8:
            k[e] = (double)c->k_code[row * ORC_D + e] * (double)c->k_scale[row];
            v[e] = (double)c->v_code[row * ORC_D + e] * (double)c->v_scale[row];
            break;
        default:
            k[e] = c->k_f64[row * ORC_D + e];
            v[e] = c->v_f64[row * ORC_D + e];
        }
    }
}

/* Number of cache tokens visible to the current segment: all tokens of the
 * slots that hold one of the last `window` committed frames. */
int64_t orc_visible_cache_tokens(const orc_cache *c) {
    const int64_t F = (int64_t)c->grid_h * c->grid_w;
    int64_t lo = (c->window_frames > 0) ? c->frames_committed - c->window_frames : 0;
    int64_t n = 0;
    for (int s = 0; s < c->capacity_frames; ++s)
        if (c->slot_frame[s] >= 0 && c->slot_frame[s] >= lo) n += F;
    return n;
}

/* Segment attention of the current segment over [visible cache ; current].
 * q, k, v: BF16 bits, token-major [Nq][H][128] (video first, then text).
 * rows: query indices to evaluate (NULL = all Nq); out: [n_rows][H][128]
 * (row order of `rows`); lse: [H][n_rows] natural-log sum-exp of scaled
 * scores. */
int orc_seg_attn(const orc_cache *c, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                 int64_t token_stride, int n_video_frames, int n_text, const int64_t *rows, int64_t n_rows,
                 double *out, double *lse, int nthreads) {
    const int64_t F = (int64_t)c->grid_h * c->grid_w;
    const int64_t nv = (int64_t)n_video_frames * F;
    const int64_t nq = nv + n_text;
    const int H = c->heads;
    const int64_t cap_tok = (int64_t)c->capacity_frames * F;
    const int64_t t0 = c->frames_committed;
    if (rows == NULL) n_rows = nq;
    const int64_t nc = orc_visible_cache_tokens(c);
    const int64_t nk = nc + nq;
    int64_t lo = (c->window_frames > 0) ? c->frames_committed - c->window_frames : 0;

    double *keys = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1) * ORC_D);
    double *vals = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1) * ORC_D);
    double *cs = segment_cs(nv, t0, c->grid_h, c->grid_w, c->theta);
    double *qsel = (double *)malloc(sizeof(double) * (size_t)(n_rows > 0 ? n_rows : 1) * ORC_D);
    double *osel = (double *)malloc(sizeof(double) * (size_t)(n_rows > 0 ? n_rows : 1) * ORC_D);
    double *lsel = (double *)malloc(sizeof(double) * (size_t)(n_rows > 0 ? n_rows : 1));
    if (!keys || !vals || !cs || !qsel || !osel || !lsel) {
        free(keys); free(vals); free(cs); free(qsel); free(osel); free(lsel);
        return -3;
    }
    for (int h = 0; h < H; ++h) {
        int64_t j = 0;
        for (int s = 0; s < c->capacity_frames; ++s) {
            if (c->slot_frame[s] < 0 || c->slot_frame[s] < lo) continue;
            for (int64_t r = 0; r < F; ++r, ++j)
                cache_row(c, (int64_t)h * cap_tok + (int64_t)s * F + r, keys + j * ORC_D, vals + j * ORC_D);
        }
        rotate_segment(k, token_stride, h, nv, NULL, nq, cs, keys + nc * ORC_D);
        plain_segment(v, token_stride, h, nq, vals + nc * ORC_D);
        rotate_segment(q, token_stride, h, nv, rows, n_rows, cs, qsel);
        key_set ks = {nk, keys, vals};
        attend_rows_parallel(&ks, qsel, n_rows, osel, lsel, nthreads);
        for (int64_t r = 0; r < n_rows; ++r) {
            memcpy(out + (r * H + h) * ORC_D, osel + r * ORC_D, sizeof(double) * ORC_D);
            if (lse) lse[(int64_t)h * n_rows + r] = lsel[r];
        }
    }
    free(keys); free(vals); free(cs); free(qsel); free(osel); free(lsel);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Masked full-sequence attention (no cache)                            */
/* ------------------------------------------------------------------ */

/* The whole session as one sequence of segments: segment s has n_video[s]
 * latent frames and n_text[s] text tokens, BF16 q/k/v token-major
 * [N_s][H][128] with stride H*128. Its video frames sit at t0_s = sum of
 * earlier segments' frames. A query of segment `target` sees every token of
 * its own segment and the video tokens of earlier segments whose frame
 * index is >= t0_target - window (window 0: all earlier frames); nothing of
 * later segments. Returns out [N_target][H][128]. */
int orc_full_seq_attn(int n_seg, const uint16_t *const *qs, const uint16_t *const *ks_, const uint16_t *const *vs,
                      const int32_t *n_video, const int32_t *n_text, int heads, int gh, int gw, double theta,
                      int window, int target, double *out, double *lse, int nthreads) {
    const int64_t F = (int64_t)gh * gw;
    const int64_t stride = (int64_t)heads * ORC_D;
    int64_t t0_target = 0;
    for (int s = 0; s < target; ++s) t0_target += n_video[s];
    const int64_t lo = window > 0 ? t0_target - window : 0;
    int64_t nk = 0;
    for (int s = 0; s < target; ++s) {
        int64_t t0 = 0;
        for (int u = 0; u < s; ++u) t0 += n_video[u];
        for (int64_t fi = 0; fi < n_video[s]; ++fi)
            if (t0 + fi >= lo) nk += F;
    }
    const int64_t nq = (int64_t)n_video[target] * F + n_text[target];
    nk += nq;
    double *keys = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1) * ORC_D);
    double *vals = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1) * ORC_D);
    double *qr = (double *)malloc(sizeof(double) * (size_t)(nq > 0 ? nq : 1) * ORC_D);
    double *ob = (double *)malloc(sizeof(double) * (size_t)(nq > 0 ? nq : 1) * ORC_D);
    double *lb = (double *)malloc(sizeof(double) * (size_t)(nq > 0 ? nq : 1));
    int64_t max_nvs = 1;
    for (int s = 0; s < target; ++s)
        if ((int64_t)n_video[s] * F > max_nvs) max_nvs = (int64_t)n_video[s] * F;
    double *tmp = (double *)malloc(sizeof(double) * (size_t)(2 * max_nvs) * ORC_D);
    if (!keys || !vals || !qr || !ob || !lb || !tmp) {
        free(keys); free(vals); free(qr); free(ob); free(lb); free(tmp);
        return -3;
    }
    for (int h = 0; h < heads; ++h) {
        int64_t j = 0, t0 = 0;
        for (int s = 0; s < target; ++s) {
            int64_t nvs = (int64_t)n_video[s] * F;
            double *cs_s = segment_cs(nvs, t0, gh, gw, theta);
            rotate_segment(ks_[s], stride, h, nvs, NULL, nvs, cs_s, tmp);
            free(cs_s);
            plain_segment(vs[s], stride, h, nvs, tmp + nvs * ORC_D);
            for (int64_t n = 0; n < nvs; ++n) {
                if (t0 + n / F < lo) continue;
                memcpy(keys + j * ORC_D, tmp + n * ORC_D, sizeof(double) * ORC_D);
                memcpy(vals + j * ORC_D, tmp + (nvs + n) * ORC_D, sizeof(double) * ORC_D);
                ++j;
            }
            t0 += n_video[s];
        }
        int64_t nvt = (int64_t)n_video[target] * F;
        double *cs_t = segment_cs(nvt, t0_target, gh, gw, theta);
        rotate_segment(ks_[target], stride, h, nvt, NULL, nq, cs_t, keys + j * ORC_D);
        plain_segment(vs[target], stride, h, nq, vals + j * ORC_D);
        rotate_segment(qs[target], stride, h, nvt, NULL, nq, cs_t, qr);
        free(cs_t);
        key_set kset = {nk, keys, vals};
        attend_rows_parallel(&kset, qr, nq, ob, lb, nthreads);
        for (int64_t r = 0; r < nq; ++r) {
            memcpy(out + (r * heads + h) * ORC_D, ob + r * ORC_D, sizeof(double) * ORC_D);
            if (lse) lse[(int64_t)h * nq + r] = lb[r];
        }
    }
    free(keys); free(vals); free(qr); free(ob); free(lb); free(tmp);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Per-latent-frame camera cross-attention                             */
/* ------------------------------------------------------------------ */

/* out[i][h] = softmax_j(<q_i,h, k_c,j,h> / sqrt(128)) . v_c,j,h over the
 * n_cam camera tokens j of chunk c = (i / tpf) / chunk_frames, for every
 * video token i < n_frames * tpf and head h. q: BF16 [n_video][heads][128]
 * with token stride q_stride; k_cam, v_cam: BF16 [n_chunks][n_cam][heads][128];
 * out: fp64 [n_video][heads][128]. fp64 two-pass softmax (attend_row). */
int orc_camera_attn(const uint16_t *q, int64_t q_stride, int n_frames, int tpf, int heads,
                    const uint16_t *k_cam, const uint16_t *v_cam, int n_cam, int chunk_frames, double *out) {
    if (n_frames < 0 || tpf <= 0 || heads <= 0 || n_cam <= 0 || chunk_frames <= 0) return -1;
    double *keys = malloc(sizeof(double) * (size_t)n_cam * ORC_D);
    double *vals = malloc(sizeof(double) * (size_t)n_cam * ORC_D);
    double *scores = malloc(sizeof(double) * (size_t)n_cam);
    double qd[ORC_D];
    if (!keys || !vals || !scores) {
        free(keys); free(vals); free(scores);
        return -2;
    }
    const int64_t nv = (int64_t)n_frames * tpf;
    for (int64_t i = 0; i < nv; ++i) {
        const int64_t chunk = (i / tpf) / chunk_frames;
        for (int h = 0; h < heads; ++h) {
            for (int j = 0; j < n_cam; ++j) {
                const int64_t base = ((chunk * n_cam + j) * heads + h) * ORC_D;
                for (int e = 0; e < ORC_D; ++e) {
                    keys[(int64_t)j * ORC_D + e] = bf16_to_f32(k_cam[base + e]);
                    vals[(int64_t)j * ORC_D + e] = bf16_to_f32(v_cam[base + e]);
                }
            }
            for (int e = 0; e < ORC_D; ++e) qd[e] = bf16_to_f32(q[i * q_stride + (int64_t)h * ORC_D + e]);
            key_set ks = {n_cam, keys, vals};
            double lse;
            attend_row(qd, &ks, out + (i * heads + h) * ORC_D, &lse, scores);
        }
    }
    free(keys); free(vals); free(scores);
    return 0;
}
