/*
 * vsa_oracle.c -- plain, slow, obviously-correct CPU oracle for block-sparse
 * video attention (VSA-style fine pass plus the SLA/RoLA-style linear branch).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant with the
 * CUDA library.
 *
 * Arithmetic is carried out in REAL (double by default; the build also makes
 * a float copy, used only to show that the tolerance budget is loose compared
 * with fp32-vs-fp64 differences).  Inputs arrive as raw bf16 bit patterns and
 * are widened exactly.
 *
 * What the pages fix, and where:
 *  - "FastVideo 稀疏蒸馏技术深度解析" (omica.com.cn), section "2. 视频稀疏注意力VSA":
 *    VSA picks the key attention blocks dynamically and evaluates only 10-20 %
 *    of the attention weights (sparsity 0.8-0.9), in a way that stays
 *    compatible with Flash-Attention-style exact softmax attention.
 *  - SparkDiffusion news item (bazainvestora.ru), paragraphs 2-3: at 97 %
 *    sparsity only 3 % of the blocks survive; RoLA pairs the block-sparse branch
 *    with a low-rank linear branch that keeps global context.
 *  - TurboDiffusion article (dolphinsci.com), section "稀疏、蒸馏与全链路量化":
 *    SLA = trainable sparse attention plus a linear-attention branch.
 * Everything the pages leave open (the 4x4x4 cube tiles, mean pooling over
 * the valid tokens, the scaled coarse scores, top-k with ties to the lower
 * tile id, elu+1 feature map) follows the plainest reading of that outline;
 * each such reading is named at the function that makes it.
 *
 * Conventions (all arrays contiguous, row-major):
 *   token n = (t*H + h)*W + w         for a T x H x W latent grid
 *   q, k, v, out : [B][N][heads][d]   bf16 bit patterns (out: REAL)
 *   tile j = (it*nh + ih)*nw + iw     nt = nT*nh*nw, nT = ceil(T/tt) ...
 *   slot s = (dt*th + dh)*tw + dw     inside a tt x th x tw tile
 *   a slot is valid iff its (t,h,w) lies inside the grid
 *   block_idx : [B][heads][nt][k]     int32, each row ascending
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef REAL
#define REAL double
#endif
#ifndef ORACLE_EXP
#define ORACLE_EXP exp
#endif
#ifndef ORACLE_SQRT
#define ORACLE_SQRT sqrt
#endif

/* ---------------------------------------------------------------- helpers */

static REAL bf16_to_real(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (REAL)f;
}

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

typedef struct {
    int T, H, W, tt, th, tw;
    int nT, nh, nw, nt, vol;
    int64_t N;
} grid_t;

static grid_t make_grid(int T, int H, int W, int tt, int th, int tw)
{
    grid_t g;
    g.T = T; g.H = H; g.W = W; g.tt = tt; g.th = th; g.tw = tw;
    g.nT = ceil_div(T, tt); g.nh = ceil_div(H, th); g.nw = ceil_div(W, tw);
    g.nt = g.nT * g.nh * g.nw;
    g.vol = tt * th * tw;
    g.N = (int64_t)T * H * W;
    return g;
}

/* Token index held by slot s of tile j, or -1 when the slot lies outside
 * the grid (a padded slot of a ragged edge tile). */
static int64_t slot_token(const grid_t *g, int j, int s)
{
    int it = j / (g->nh * g->nw);
    int ih = (j / g->nw) % g->nh;
    int iw = j % g->nw;
    int dt = s / (g->th * g->tw);
    int dh = (s / g->tw) % g->th;
    int dw = s % g->tw;
    int t = it * g->tt + dt, h = ih * g->th + dh, w = iw * g->tw + dw;
    if (t >= g->T || h >= g->H || w >= g->W) return -1;
    return ((int64_t)t * g->H + h) * g->W + w;
}

static const uint16_t *row_ptr(const uint16_t *x, int64_t N, int heads, int d,
                               int b, int64_t n, int hd)
{
    return x + (((int64_t)b * N + n) * heads + hd) * d;
}

/* ------------------------------------------------------- tiling map (step 1) */

int oracle_num_tiles(int T, int H, int W, int tt, int th, int tw)
{
    grid_t g = make_grid(T, H, W, tt, th, tw);
    return g.nt;
}

/* token_of_slot[j*vol + s] = token index, or -1 for a padded slot. */
void oracle_tile_slots(int T, int H, int W, int tt, int th, int tw,
                       int64_t *token_of_slot)
{
    grid_t g = make_grid(T, H, W, tt, th, tw);
    for (int j = 0; j < g.nt; ++j)
        for (int s = 0; s < g.vol; ++s)
            token_of_slot[(int64_t)j * g.vol + s] = slot_token(&g, j, s);
}

/* Grid order -> tile-major [B][heads][nt][vol][d]; padded slots are zero. */
void oracle_gather(const uint16_t *x, uint16_t *tiles, int B, int heads, int d,
                   int T, int H, int W, int tt, int th, int tw)
{
    grid_t g = make_grid(T, H, W, tt, th, tw);
    for (int b = 0; b < B; ++b)
        for (int hd = 0; hd < heads; ++hd)
            for (int j = 0; j < g.nt; ++j)
                for (int s = 0; s < g.vol; ++s) {
                    uint16_t *dst = tiles + ((((int64_t)b * heads + hd) * g.nt + j) * g.vol + s) * d;
                    int64_t n = slot_token(&g, j, s);
                    if (n < 0) { memset(dst, 0, sizeof(uint16_t) * d); continue; }
                    memcpy(dst, row_ptr(x, g.N, heads, d, b, n, hd), sizeof(uint16_t) * d);
                }
}

/* Tile-major -> grid order, valid slots only. */
void oracle_scatter(const uint16_t *tiles, uint16_t *x, int B, int heads, int d,
                    int T, int H, int W, int tt, int th, int tw)
{
    grid_t g = make_grid(T, H, W, tt, th, tw);
    for (int b = 0; b < B; ++b)
        for (int hd = 0; hd < heads; ++hd)
            for (int j = 0; j < g.nt; ++j)
                for (int s = 0; s < g.vol; ++s) {
                    int64_t n = slot_token(&g, j, s);
                    if (n < 0) continue;
                    const uint16_t *src = tiles + ((((int64_t)b * heads + hd) * g.nt + j) * g.vol + s) * d;
                    memcpy((uint16_t *)row_ptr(x, g.N, heads, d, b, n, hd), src, sizeof(uint16_t) * d);
                }
}

/* ------------------------------------------------------------ pool (step 2)
 * Mean of each tile over its VALID tokens only (a ragged edge tile divides by
 * its own valid count).  pooled: [B][heads][nt][d]. */
void oracle_pool(const uint16_t *x, int B, int heads, int d,
                 int T, int H, int W, int tt, int th, int tw, REAL *pooled)
{
    grid_t g = make_grid(T, H, W, tt, th, tw);
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int hd = 0; hd < heads; ++hd)
            for (int j = 0; j < g.nt; ++j) {
                REAL *out = pooled + (((int64_t)b * heads + hd) * g.nt + j) * d;
                int count = 0;
                for (int c = 0; c < d; ++c) out[c] = 0;
                for (int s = 0; s < g.vol; ++s) {
                    int64_t n = slot_token(&g, j, s);
                    if (n < 0) continue;
                    const uint16_t *r = row_ptr(x, g.N, heads, d, b, n, hd);
                    for (int c = 0; c < d; ++c) out[c] += bf16_to_real(r[c]);
                    ++count;
                }
                for (int c = 0; c < d; ++c) out[c] /= (REAL)count;
            }
}

/* ---------------------------------------------------------- coarse (step 3)
 * scores[i][j] = Qp[i] . Kp[j] / sqrt(d), per (b, head).  probs (optional) is
 * the row softmax over key tiles; selection uses only the scores, because
 * softmax is monotone within a row. */
void oracle_coarse(const REAL *qp, const REAL *kp, int B, int heads, int nt, int d,
                   REAL *scores, REAL *probs)
{
    REAL inv_sqrt_d = (REAL)1 / ORACLE_SQRT((REAL)d);
#pragma omp parallel for collapse(2) schedule(static)
    for (int bh = 0; bh < B * heads; ++bh)
        for (int i = 0; i < nt; ++i) {
            const REAL *qi = qp + ((int64_t)bh * nt + i) * d;
            REAL *row = scores + ((int64_t)bh * nt + i) * nt;
            for (int j = 0; j < nt; ++j) {
                const REAL *kj = kp + ((int64_t)bh * nt + j) * d;
                REAL acc = 0;
                for (int c = 0; c < d; ++c) acc += qi[c] * kj[c];
                row[j] = acc * inv_sqrt_d;
            }
            if (probs) {
                REAL *p = probs + ((int64_t)bh * nt + i) * nt;
                REAL mx = row[0], sum = 0;
                for (int j = 1; j < nt; ++j) if (row[j] > mx) mx = row[j];
                for (int j = 0; j < nt; ++j) { p[j] = ORACLE_EXP(row[j] - mx); sum += p[j]; }
                for (int j = 0; j < nt; ++j) p[j] /= sum;
            }
        }
}

/* ----------------------------------------------------------- top-k (step 4)
 * Rank key tiles by (score descending, tile id ascending), keep the first k,
 * emit them in ascending tile order. */
typedef struct { REAL s; int j; } scored_t;

static int by_score_then_id(const void *pa, const void *pb)
{
    const scored_t *a = (const scored_t *)pa, *b = (const scored_t *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

static int by_int(const void *pa, const void *pb)
{
    int a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

void oracle_topk(const REAL *scores, int B, int heads, int nt, int k, int32_t *idx)
{
#pragma omp parallel
    {
        scored_t *buf = (scored_t *)malloc(sizeof(scored_t) * (size_t)nt);
#pragma omp for schedule(static)
        for (int64_t r = 0; r < (int64_t)B * heads * nt; ++r) {
            const REAL *row = scores + r * nt;
            for (int j = 0; j < nt; ++j) { buf[j].s = row[j]; buf[j].j = j; }
            qsort(buf, (size_t)nt, sizeof(scored_t), by_score_then_id);
            int32_t *out = idx + r * k;
            for (int m = 0; m < k; ++m) out[m] = buf[m].j;
            qsort(out, (size_t)k, sizeof(int32_t), by_int);
        }
        free(buf);
    }
}

/* pool + coarse + top-k in one call; scores (optional) receives the coarse
 * logits [B][heads][nt][nt]. */
void oracle_select(const uint16_t *q, const uint16_t *kk, int B, int heads, int d,
                   int T, int H, int W, int tt, int th, int tw, int k,
                   int32_t *idx, REAL *scores_out)
{
    grid_t g = make_grid(T, H, W, tt, th, tw);
    size_t np = (size_t)B * heads * g.nt * d;
    REAL *qp = (REAL *)malloc(sizeof(REAL) * np);
    REAL *kp = (REAL *)malloc(sizeof(REAL) * np);
    REAL *sc = scores_out ? scores_out
                          : (REAL *)malloc(sizeof(REAL) * (size_t)B * heads * g.nt * g.nt);
    oracle_pool(q, B, heads, d, T, H, W, tt, th, tw, qp);
    oracle_pool(kk, B, heads, d, T, H, W, tt, th, tw, kp);
    oracle_coarse(qp, kp, B, heads, g.nt, d, sc, NULL);
    oracle_topk(sc, B, heads, g.nt, k, idx);
    free(qp); free(kp);
    if (!scores_out) free(sc);
}

/* ------------------------------------------------------------ fine (step 5)
 * For every valid query n of tile i: softmax over the valid tokens of the
 * selected key tiles idx[i][0..k) of q_n . k_m / sqrt(d), then the weighted
 * sum of v_m.  The scale 1/sqrt(d) is the plainest reading (the pages do not
 * state the scale of the fine pass). */
static void fine_one_tile(const grid_t *g, const uint16_t *q, const uint16_t *kk,
                          const uint16_t *v, const int32_t *sel, int k,
                          int heads, int d, int b, int hd, int i,
                          int64_t *tok_buf, REAL *s_buf,
                          REAL *out_rows /* [vol][d], padded rows left 0 */)
{
    REAL inv_sqrt_d = (REAL)1 / ORACLE_SQRT((REAL)d);
    int nk = 0;
    for (int m = 0; m < k; ++m)
        for (int s = 0; s < g->vol; ++s) {
            int64_t n = slot_token(g, sel[m], s);
            if (n >= 0) tok_buf[nk++] = n;
        }
    for (int s = 0; s < g->vol; ++s) {
        REAL *o = out_rows + (int64_t)s * d;
        for (int c = 0; c < d; ++c) o[c] = 0;
        int64_t nq = slot_token(g, i, s);
        if (nq < 0) continue;
        const uint16_t *qr = row_ptr(q, g->N, heads, d, b, nq, hd);
        REAL mx = -INFINITY;
        for (int m = 0; m < nk; ++m) {
            const uint16_t *kr = row_ptr(kk, g->N, heads, d, b, tok_buf[m], hd);
            REAL acc = 0;
            for (int c = 0; c < d; ++c) acc += bf16_to_real(qr[c]) * bf16_to_real(kr[c]);
            s_buf[m] = acc * inv_sqrt_d;
            if (s_buf[m] > mx) mx = s_buf[m];
        }
        REAL sum = 0;
        for (int m = 0; m < nk; ++m) { s_buf[m] = ORACLE_EXP(s_buf[m] - mx); sum += s_buf[m]; }
        for (int m = 0; m < nk; ++m) {
            const uint16_t *vr = row_ptr(v, g->N, heads, d, b, tok_buf[m], hd);
            REAL p = s_buf[m] / sum;
            for (int c = 0; c < d; ++c) o[c] += p * bf16_to_real(vr[c]);
        }
    }
}

/* Fine pass for a list of query tiles.  rows[r] = (b*heads + head)*nt + i;
 * out_rows: [nrows][vol][d] in slot order (padded slots stay 0). */
void oracle_fine_tiles(const uint16_t *q, const uint16_t *kk, const uint16_t *v,
                       const int32_t *idx, int B, int heads, int d,
                       int T, int H, int W, int tt, int th, int tw, int k,
                       const int64_t *rows, int64_t nrows, REAL *out_rows)
{
    grid_t g = make_grid(T, H, W, tt, th, tw);
    (void)B;
#pragma omp parallel
    {
        int64_t *tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)k * g.vol);
        REAL *sb = (REAL *)malloc(sizeof(REAL) * (size_t)k * g.vol);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t row = rows[r];
            int i = (int)(row % g.nt);
            int bh = (int)(row / g.nt);
            int b = bh / heads, hd = bh % heads;
            fine_one_tile(&g, q, kk, v, idx + row * k, k, heads, d, b, hd, i,
                          tok, sb, out_rows + r * g.vol * d);
        }
        free(tok); free(sb);
    }
}

/* Fine pass for every query tile, written in grid order out[B][N][heads][d]. */
void oracle_fine(const uint16_t *q, const uint16_t *kk, const uint16_t *v,
                 const int32_t *idx, int B, int heads, int d,
                 int T, int H, int W, int tt, int th, int tw, int k, REAL *out)
{
    grid_t g = make_grid(T, H, W, tt, th, tw);
#pragma omp parallel
    {
        int64_t *tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)k * g.vol);
        REAL *sb = (REAL *)malloc(sizeof(REAL) * (size_t)k * g.vol);
        REAL *tile = (REAL *)malloc(sizeof(REAL) * (size_t)g.vol * d);
#pragma omp for schedule(dynamic, 1)
        for (int64_t row = 0; row < (int64_t)B * heads * g.nt; ++row) {
            int i = (int)(row % g.nt);
            int bh = (int)(row / g.nt);
            int b = bh / heads, hd = bh % heads;
            fine_one_tile(&g, q, kk, v, idx + row * k, k, heads, d, b, hd, i,
                          tok, sb, tile);
            for (int s = 0; s < g.vol; ++s) {
                int64_t n = slot_token(&g, i, s);
                if (n < 0) continue;
                memcpy(out + (((int64_t)b * g.N + n) * heads + hd) * d,
                       tile + (int64_t)s * d, sizeof(REAL) * d);
            }
        }
        free(tok); free(sb); free(tile);
    }
}

/* ----------------------------------------------- low-precision fine pass
 * The low-precision variant quantises q and k to FP8 E4M3 before Q K^T, one
 * scale per (b, head, cube) ("sparse is orthogonal to low-bit tensor cores":
 * TurboDiffusion article, section "稀疏、蒸馏与全链路量化", SageSLA built on
 * SageAttention's quantised products).  E4M3 as the OCP 8-bit floating-point
 * format defines it ("fn" flavour, no infinities): 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits; normal values 1.m x 2^(e-7) for e = 1..15
 * except e = 15, m = 7 (NaN), so the largest is 1.75 x 2^8 = 448; subnormals
 * m x 2^-9 (e = 0).  Rounding: to nearest, ties to even; magnitudes above 448
 * saturate to 448.  Reading made here: scale = amax / 448 in fp32 over the
 * cube's valid tokens and all d features (1 for an all-zero cube), code =
 * E4M3(x * inv) with inv = 1 / scale, both rounded to nearest fp32 (the
 * dequantised value is code * scale). */
uint8_t oracle_e4m3_encode_one(float x)
{
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs((double)x);
    if (a > 448.0) return sign | 0x7E;
    if (a < 0.015625) {                       /* below 2^-6: quantum 2^-9 */
        double m = nearbyint(a * 512.0);      /* 8 carries into 2^-6 = code 8 */
        return sign | (uint8_t)m;
    }
    int e2;
    frexp(a, &e2);                            /* a = f 2^e2, f in [0.5, 1) */
    int E = e2 - 1;                           /* 2^E <= a < 2^(E+1) */
    double m = nearbyint(a / ldexp(1.0, E - 3));   /* 8 .. 16 */
    if (m == 16.0) { m = 8.0; E += 1; }
    return sign | (uint8_t)(((E + 7) << 3) | ((int)m - 8));
}

REAL oracle_e4m3_decode_one(uint8_t c)
{
    int e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    REAL v = e == 0 ? (REAL)ldexp((double)m, -9) : (REAL)ldexp((double)(8 + m), e - 10);
    return (c & 0x80) ? -v : v;
}

void oracle_e4m3_encode(const float *x, int64_t n, uint8_t *codes)
{
    for (int64_t i = 0; i < n; ++i) codes[i] = oracle_e4m3_encode_one(x[i]);
}

void oracle_e4m3_decode(const uint8_t *codes, int64_t n, REAL *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_decode_one(codes[i]);
}

/* Per-cube quantisation of x [B][N][heads][d] (bf16 bits): codes in the same
 * layout (valid tokens only), scales [B][heads][nt]. */
void oracle_quant_e4m3_cubes(const uint16_t *x, int B, int heads, int d, int T, int H, int W,
                             int tt, int th, int tw, uint8_t *codes, float *scales)
{
    grid_t g = make_grid(T, H, W, tt, th, tw);
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int hd = 0; hd < heads; ++hd)
            for (int j = 0; j < g.nt; ++j) {
                float amax = 0.0f;
                for (int s = 0; s < g.vol; ++s) {
                    int64_t n = slot_token(&g, j, s);
                    if (n < 0) continue;
                    const uint16_t *xr = row_ptr(x, g.N, heads, d, b, n, hd);
                    for (int c = 0; c < d; ++c) {
                        float v = fabsf((float)bf16_to_real(xr[c]));
                        if (v > amax) amax = v;
                    }
                }
                volatile float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
                volatile float inv = 1.0f / scale;
                scales[((int64_t)b * heads + hd) * g.nt + j] = scale;
                for (int s = 0; s < g.vol; ++s) {
                    int64_t n = slot_token(&g, j, s);
                    if (n < 0) continue;
                    const uint16_t *xr = row_ptr(x, g.N, heads, d, b, n, hd);
                    uint8_t *cr = codes + (((int64_t)b * g.N + n) * heads + hd) * d;
                    for (int c = 0; c < d; ++c) {
                        volatile float y = (float)bf16_to_real(xr[c]) * inv;
                        cr[c] = oracle_e4m3_encode_one(y);
                    }
                }
            }
}

/* Fine pass (as oracle_fine_tiles) with real-valued q and k [B][N][heads][d]
 * (e.g. the dequantised codes times their cube scales) and bf16 v. */
void oracle_fine_tiles_real(const REAL *q, const REAL *kk, const uint16_t *v,
                            const int32_t *idx, int B, int heads, int d,
                            int T, int H, int W, int tt, int th, int tw, int k,
                            const int64_t *rows, int64_t nrows, REAL *out_rows)
{
    grid_t g = make_grid(T, H, W, tt, th, tw);
    (void)B;
    REAL inv_sqrt_d = (REAL)1 / ORACLE_SQRT((REAL)d);
#pragma omp parallel
    {
        int64_t *tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)k * g.vol);
        REAL *sb = (REAL *)malloc(sizeof(REAL) * (size_t)k * g.vol);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t row = rows[r];
            int i = (int)(row % g.nt);
            int bh = (int)(row / g.nt);
            int b = bh / heads, hd = bh % heads;
            const int32_t *sel = idx + row * k;
            REAL *out = out_rows + r * g.vol * d;
            int nk = 0;
            for (int m = 0; m < k; ++m)
                for (int s = 0; s < g.vol; ++s) {
                    int64_t n = slot_token(&g, sel[m], s);
                    if (n >= 0) tok[nk++] = n;
                }
            for (int s = 0; s < g.vol; ++s) {
                REAL *o = out + (int64_t)s * d;
                for (int c = 0; c < d; ++c) o[c] = 0;
                int64_t nq = slot_token(&g, i, s);
                if (nq < 0) continue;
                const REAL *qr = q + (((int64_t)b * g.N + nq) * heads + hd) * d;
                REAL mx = -INFINITY;
                for (int m = 0; m < nk; ++m) {
                    const REAL *kr = kk + (((int64_t)b * g.N + tok[m]) * heads + hd) * d;
                    REAL acc = 0;
                    for (int c = 0; c < d; ++c) acc += qr[c] * kr[c];
                    sb[m] = acc * inv_sqrt_d;
                    if (sb[m] > mx) mx = sb[m];
                }
                REAL sum = 0;
                for (int m = 0; m < nk; ++m) { sb[m] = ORACLE_EXP(sb[m] - mx); sum += sb[m]; }
                for (int m = 0; m < nk; ++m) {
                    const uint16_t *vr = row_ptr(v, g.N, heads, d, b, tok[m], hd);
                    REAL p = sb[m] / sum;
                    for (int c = 0; c < d; ++c) o[c] += p * bf16_to_real(vr[c]);
                }
            }
        }
        free(tok); free(sb);
    }
}

/* Attention weights of one query (b, head, token n) over ALL N keys in grid
 * order: zero outside the selected tiles.  Used to check that each row sums
 * to one and vanishes off the selection. */
void oracle_weights(const uint16_t *q, const uint16_t *kk, const int32_t *idx,
                    int B, int heads, int d, int T, int H, int W,
                    int tt, int th, int tw, int k, int b, int hd, int64_t n,
                    REAL *w /* [N] */)
{
    grid_t g = make_grid(T, H, W, tt, th, tw);
    (void)B;
    REAL inv_sqrt_d = (REAL)1 / ORACLE_SQRT((REAL)d);
    int t = (int)(n / ((int64_t)H * W)), h = (int)((n / W) % H), ww = (int)(n % W);
    int i = ((t / tt) * g.nh + h / th) * g.nw + ww / tw;
    const int32_t *sel = idx + (((int64_t)b * heads + hd) * g.nt + i) * k;
    const uint16_t *qr = row_ptr(q, g.N, heads, d, b, n, hd);
    for (int64_t m = 0; m < g.N; ++m) w[m] = 0;
    REAL mx = -INFINITY;
    for (int a = 0; a < k; ++a)
        for (int s = 0; s < g.vol; ++s) {
            int64_t m = slot_token(&g, sel[a], s);
            if (m < 0) continue;
            const uint16_t *kr = row_ptr(kk, g.N, heads, d, b, m, hd);
            REAL acc = 0;
            for (int c = 0; c < d; ++c) acc += bf16_to_real(qr[c]) * bf16_to_real(kr[c]);
            w[m] = acc * inv_sqrt_d;
            if (w[m] > mx) mx = w[m];
        }
    REAL sum = 0;
    for (int a = 0; a < k; ++a)
        for (int s = 0; s < g.vol; ++s) {
            int64_t m = slot_token(&g, sel[a], s);
            if (m < 0) continue;
            w[m] = ORACLE_EXP(w[m] - mx);
            sum += w[m];
        }
    for (int a = 0; a < k; ++a)
        for (int s = 0; s < g.vol; ++s) {
            int64_t m = slot_token(&g, sel[a], s);
            if (m >= 0) w[m] /= sum;
        }
}

/* ------------------------------------------------------ fine pass, backward
 * Gradients of the fine pass (trainable sparse attention: "FastVideo
 * 稀疏蒸馏技术深度解析", section "2. 视频稀疏注意力VSA", and the TurboDiffusion
 * article, section "稀疏、蒸馏与全链路量化", train the sparse branch).  The
 * selection is a fixed input here, as in the forward fine pass.  For each
 * valid query token n with kept keys m (valid tokens of its selected tiles),
 * given the output gradient dO_n, straight from the chain rule through
 * s_m = q_n.k_m / sqrt(d), p = softmax(s), o_n = sum_m p_m v_m:
 *     dv_m += p_m dO_n
 *     dp_m  = dO_n . v_m
 *     ds_m  = p_m (dp_m - sum_m' p_m' dp_m')
 *     dq_n  = sum_m ds_m k_m / sqrt(d)
 *     dk_m += ds_m q_n / sqrt(d)
 * dout is bf16 (bit patterns, like q, k, v); dq, dk, dv are REAL, fully
 * overwritten.  One (b, head) per OpenMP iteration, so the dk / dv sums of a
 * key never race. */
void oracle_fine_bwd(const uint16_t *q, const uint16_t *kk, const uint16_t *v,
                     const uint16_t *dout, const int32_t *idx, int B, int heads, int d,
                     int T, int H, int W, int tt, int th, int tw, int k,
                     REAL *dq, REAL *dk, REAL *dv)
{
    grid_t g = make_grid(T, H, W, tt, th, tw);
    REAL inv_sqrt_d = (REAL)1 / ORACLE_SQRT((REAL)d);
    size_t total = (size_t)B * g.N * heads * d;
    memset(dq, 0, sizeof(REAL) * total);
    memset(dk, 0, sizeof(REAL) * total);
    memset(dv, 0, sizeof(REAL) * total);
#pragma omp parallel
    {
        int64_t *tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)k * g.vol);
        REAL *p = (REAL *)malloc(sizeof(REAL) * (size_t)k * g.vol);
        REAL *dp = (REAL *)malloc(sizeof(REAL) * (size_t)k * g.vol);
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < (int64_t)B * heads; ++bh) {
            int b = (int)(bh / heads), hd = (int)(bh % heads);
            for (int i = 0; i < g.nt; ++i) {
                const int32_t *sel = idx + (bh * g.nt + i) * k;
                int nk = 0;
                for (int a = 0; a < k; ++a)
                    for (int s = 0; s < g.vol; ++s) {
                        int64_t m = slot_token(&g, sel[a], s);
                        if (m >= 0) tok[nk++] = m;
                    }
                for (int s = 0; s < g.vol; ++s) {
                    int64_t n = slot_token(&g, i, s);
                    if (n < 0) continue;
                    const uint16_t *qr = row_ptr(q, g.N, heads, d, b, n, hd);
                    const uint16_t *gr = row_ptr(dout, g.N, heads, d, b, n, hd);
                    /* p = softmax(s) */
                    REAL mx = -INFINITY;
                    for (int m = 0; m < nk; ++m) {
                        const uint16_t *kr = row_ptr(kk, g.N, heads, d, b, tok[m], hd);
                        REAL acc = 0;
                        for (int c = 0; c < d; ++c) acc += bf16_to_real(qr[c]) * bf16_to_real(kr[c]);
                        p[m] = acc * inv_sqrt_d;
                        if (p[m] > mx) mx = p[m];
                    }
                    REAL sum = 0;
                    for (int m = 0; m < nk; ++m) { p[m] = ORACLE_EXP(p[m] - mx); sum += p[m]; }
                    for (int m = 0; m < nk; ++m) p[m] /= sum;
                    /* dp_m = dO_n . v_m and the row term sum_m p_m dp_m */
                    REAL row = 0;
                    for (int m = 0; m < nk; ++m) {
                        const uint16_t *vr = row_ptr(v, g.N, heads, d, b, tok[m], hd);
                        REAL acc = 0;
                        for (int c = 0; c < d; ++c) acc += bf16_to_real(gr[c]) * bf16_to_real(vr[c]);
                        dp[m] = acc;
                        row += p[m] * acc;
                    }
                    REAL *dqr = dq + (((int64_t)b * g.N + n) * heads + hd) * d;
                    for (int m = 0; m < nk; ++m) {
                        REAL ds = p[m] * (dp[m] - row);
                        const uint16_t *kr = row_ptr(kk, g.N, heads, d, b, tok[m], hd);
                        REAL *dkr = dk + (((int64_t)b * g.N + tok[m]) * heads + hd) * d;
                        REAL *dvr = dv + (((int64_t)b * g.N + tok[m]) * heads + hd) * d;
                        for (int c = 0; c < d; ++c) {
                            dqr[c] += ds * bf16_to_real(kr[c]) * inv_sqrt_d;
                            dkr[c] += ds * bf16_to_real(qr[c]) * inv_sqrt_d;
                            dvr[c] += p[m] * bf16_to_real(gr[c]);
                        }
                    }
                }
            }
        }
        free(tok); free(p); free(dp);
    }
}

/* ----------------------------------------------------- linear branch (step 6)
 * phi(x) = elu(x) + 1 = x + 1 for x > 0, exp(x) otherwise, applied to the raw
 * q and k (no projection, weight one).  The state sums run over ALL valid
 * tokens:  S = sum_n phi(k_n)^T v_n  (d x d),  z = sum_n phi(k_n)  (d).
 * lin_n = phi(q_n) S / (phi(q_n) . z). */
static REAL phi(REAL x) { return x > 0 ? x + 1 : ORACLE_EXP(x); }

void oracle_linear_state(const uint16_t *kk, const uint16_t *v, int B, int heads,
                         int d, int64_t N, REAL *S, REAL *z)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int hd = 0; hd < heads; ++hd) {
            REAL *Sb = S + ((int64_t)b * heads + hd) * d * d;
            REAL *zb = z + ((int64_t)b * heads + hd) * d;
            for (int a = 0; a < d * d; ++a) Sb[a] = 0;
            for (int a = 0; a < d; ++a) zb[a] = 0;
            for (int64_t n = 0; n < N; ++n) {
                const uint16_t *kr = row_ptr(kk, N, heads, d, b, n, hd);
                const uint16_t *vr = row_ptr(v, N, heads, d, b, n, hd);
                for (int a = 0; a < d; ++a) {
                    REAL pk = phi(bf16_to_real(kr[a]));
                    zb[a] += pk;
                    for (int c = 0; c < d; ++c) Sb[a * d + c] += pk * bf16_to_real(vr[c]);
                }
            }
        }
}

void oracle_linear_apply(const uint16_t *q, const REAL *S, const REAL *z, int B,
                         int heads, int d, int64_t N, REAL *lin /* [B][N][heads][d] */)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int64_t n = 0; n < N; ++n)
            for (int hd = 0; hd < heads; ++hd) {
                const REAL *Sb = S + ((int64_t)b * heads + hd) * d * d;
                const REAL *zb = z + ((int64_t)b * heads + hd) * d;
                const uint16_t *qr = row_ptr(q, N, heads, d, b, n, hd);
                REAL *o = lin + (((int64_t)b * N + n) * heads + hd) * d;
                REAL den = 0;
                for (int c = 0; c < d; ++c) o[c] = 0;
                for (int a = 0; a < d; ++a) {
                    REAL pq = phi(bf16_to_real(qr[a]));
                    den += pq * zb[a];
                    for (int c = 0; c < d; ++c) o[c] += pq * Sb[a * d + c];
                }
                for (int c = 0; c < d; ++c) o[c] /= den;
            }
}

/* ---------------------------------------------------- linear branch, backward
 * Gradients of the linear branch (SLA: the sparse and the linear branch are
 * trained together, TurboDiffusion article, section "稀疏、蒸馏与全链路量化").
 * With phi = elu + 1, per (b, head): S = sum_m phi(k_m)^T v_m, z = sum_m
 * phi(k_m), and for every token lin_n = num_n / den_n with num_n = phi(q_n) S,
 * den_n = phi(q_n) . z.  Given dlin_n (the output gradient), by the chain rule:
 *     dnum_n = dlin_n / den_n,   dden_n = -(dlin_n . lin_n) / den_n
 *     dphi(q_n) = S dnum_n + dden_n z             dq_n = dphi(q_n) o phi'(q_n)
 *     dS = sum_n phi(q_n)^T dnum_n,  dz = sum_n dden_n phi(q_n)
 *     dphi(k_m) = dS v_m + dz,  dv_m = dS^T phi(k_m)
 *     dk_m = dphi(k_m) o phi'(k_m)                 phi'(x) = 1 (x > 0), e^x
 * dout is bf16 bits; dq, dk, dv are REAL [B][N][heads][d], overwritten. */
static REAL dphi(REAL x) { return x > 0 ? 1 : ORACLE_EXP(x); }

void oracle_linear_bwd(const uint16_t *q, const uint16_t *kk, const uint16_t *v,
                       const uint16_t *dout, int B, int heads, int d, int64_t N,
                       REAL *dq, REAL *dk, REAL *dv)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int hd = 0; hd < heads; ++hd) {
            REAL *S = (REAL *)calloc((size_t)d * d, sizeof(REAL));
            REAL *z = (REAL *)calloc((size_t)d, sizeof(REAL));
            REAL *dS = (REAL *)calloc((size_t)d * d, sizeof(REAL));
            REAL *dz = (REAL *)calloc((size_t)d, sizeof(REAL));
            REAL *pq = (REAL *)malloc(sizeof(REAL) * d);
            REAL *num = (REAL *)malloc(sizeof(REAL) * d);
            REAL *dnum = (REAL *)malloc(sizeof(REAL) * d);
            /* forward state */
            for (int64_t m = 0; m < N; ++m) {
                const uint16_t *kr = row_ptr(kk, N, heads, d, b, m, hd);
                const uint16_t *vr = row_ptr(v, N, heads, d, b, m, hd);
                for (int a = 0; a < d; ++a) {
                    REAL pk = phi(bf16_to_real(kr[a]));
                    z[a] += pk;
                    for (int c = 0; c < d; ++c) S[a * d + c] += pk * bf16_to_real(vr[c]);
                }
            }
            /* query side: dq and the sums dS, dz */
            for (int64_t n = 0; n < N; ++n) {
                const uint16_t *qr = row_ptr(q, N, heads, d, b, n, hd);
                const uint16_t *gr = row_ptr(dout, N, heads, d, b, n, hd);
                REAL den = 0;
                for (int a = 0; a < d; ++a) { pq[a] = phi(bf16_to_real(qr[a])); den += pq[a] * z[a]; }
                for (int c = 0; c < d; ++c) {
                    REAL acc = 0;
                    for (int a = 0; a < d; ++a) acc += pq[a] * S[a * d + c];
                    num[c] = acc;
                }
                REAL gl = 0;
                for (int c = 0; c < d; ++c) gl += bf16_to_real(gr[c]) * num[c] / den;
                REAL dden = -gl / den;
                for (int c = 0; c < d; ++c) dnum[c] = bf16_to_real(gr[c]) / den;
                REAL *dqr = dq + (((int64_t)b * N + n) * heads + hd) * d;
                for (int a = 0; a < d; ++a) {
                    REAL acc = dden * z[a];
                    for (int c = 0; c < d; ++c) acc += S[a * d + c] * dnum[c];
                    dqr[a] = acc * dphi(bf16_to_real(qr[a]));
                    dz[a] += dden * pq[a];
                    for (int c = 0; c < d; ++c) dS[a * d + c] += pq[a] * dnum[c];
                }
            }
            /* key side: dk, dv */
            for (int64_t m = 0; m < N; ++m) {
                const uint16_t *kr = row_ptr(kk, N, heads, d, b, m, hd);
                const uint16_t *vr = row_ptr(v, N, heads, d, b, m, hd);
                REAL *dkr = dk + (((int64_t)b * N + m) * heads + hd) * d;
                REAL *dvr = dv + (((int64_t)b * N + m) * heads + hd) * d;
                for (int a = 0; a < d; ++a) {
                    REAL acc = dz[a];
                    for (int c = 0; c < d; ++c) acc += dS[a * d + c] * bf16_to_real(vr[c]);
                    dkr[a] = acc * dphi(bf16_to_real(kr[a]));
                }
                for (int c = 0; c < d; ++c) {
                    REAL acc = 0;
                    for (int a = 0; a < d; ++a) acc += dS[a * d + c] * phi(bf16_to_real(kr[a]));
                    dvr[c] = acc;
                }
            }
            free(S); free(z); free(dS); free(dz); free(pq); free(num); free(dnum);
        }
}

/* ------------------------------------------------------------ dense (pin)
 * Plain dense softmax attention over all N tokens of the grid; with k equal
 * to the tile count the block-sparse fine pass must reduce to this. */
void oracle_dense(const uint16_t *q, const uint16_t *kk, const uint16_t *v,
                  int B, int heads, int d, int64_t N, REAL *out)
{
    REAL inv_sqrt_d = (REAL)1 / ORACLE_SQRT((REAL)d);
#pragma omp parallel
    {
        REAL *s = (REAL *)malloc(sizeof(REAL) * (size_t)N);
#pragma omp for collapse(2) schedule(static)
        for (int bh = 0; bh < B * heads; ++bh)
            for (int64_t n = 0; n < N; ++n) {
                int b = bh / heads, hd = bh % heads;
                const uint16_t *qr = row_ptr(q, N, heads, d, b, n, hd);
                REAL mx = -INFINITY, sum = 0;
                for (int64_t m = 0; m < N; ++m) {
                    const uint16_t *kr = row_ptr(kk, N, heads, d, b, m, hd);
                    REAL acc = 0;
                    for (int c = 0; c < d; ++c) acc += bf16_to_real(qr[c]) * bf16_to_real(kr[c]);
                    s[m] = acc * inv_sqrt_d;
                    if (s[m] > mx) mx = s[m];
                }
                for (int64_t m = 0; m < N; ++m) { s[m] = ORACLE_EXP(s[m] - mx); sum += s[m]; }
                REAL *o = out + (((int64_t)b * N + n) * heads + hd) * d;
                for (int c = 0; c < d; ++c) o[c] = 0;
                for (int64_t m = 0; m < N; ++m) {
                    const uint16_t *vr = row_ptr(v, N, heads, d, b, m, hd);
                    for (int c = 0; c < d; ++c) o[c] += (s[m] / sum) * bf16_to_real(vr[c]);
                }
            }
        free(s);
    }
}

/* Number of OpenMP threads the oracle runs on (reported with CPU timings). */
int oracle_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
