/*
 * ds4moe oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, CPU implementation of the routed Mixture-of-Experts FFN with
 * 2-bit block-quantized experts described on the ds4 pages: only the routed
 * experts are quantized (up/gate in an IQ2_XXS-style codebook layout, down in
 * a Q2_K-style layout) while the shared expert and the router stay in high
 * precision (ds4 news summary, "model weights" section; upppp.jp article,
 * "asymmetric 2-bit quantization" section).  A 4-bit Q4_K-style variant is
 * the "q4" model of the same pages (ds4 news summary, "speed benchmarks").
 *
 * Only the tests, the package's smoke check and the benchmark's CPU baseline
 * may load this file.  It shares no code with the CUDA library: no header, no
 * table, no helper.  Dequantization is done in fp32 in the op order of the
 * block definitions, contraction and everything after it in fp64.
 *
 * Block layouts (little endian; 256 weights per block; matrices are
 * [rows x cols] with blocks running along cols):
 *   IQ2X 66 B : fp16 d | 8 x { idx[4] u8, aux u32 }.  aux bits 7j..7j+6 are
 *               the signs of elements 0..6 of 8-vector j (1 = negative), the
 *               sign of element 7 is the parity of those 7 bits, aux bits
 *               28..31 are the 4-bit scale s.  weight 32g+8j+i =
 *               ((d * (0.5 + s)) * 0.25) * grid[idx[j]][i] * sign.
 *   Q2K  84 B : scales[16] (low nibble sc, high nibble m, one per 16 weights)
 *               | qs[64] (weight i in byte i>>2, bits 2*(i&3)) | fp16 d
 *               | fp16 dmin.  w = d*sc*q - dmin*m.
 *   Q4K 144 B : fp16 d | fp16 dmin | 12 scale bytes = 96-bit little-endian
 *               bit string, sc_j at bits 6j..6j+5, m_j at bits 48+6j..48+6j+5
 *               (one per 32 weights) | qs[128] (weight i in byte i>>1, low
 *               nibble for even i).  w = d*sc*q - dmin*m.
 *
 * Gating (the pages leave the router function open; the reading used here):
 *   l_e = sum_i W_r[e,i] x_i + b_e,  s_e = 1 / (1 + exp(-l_e)),
 *   the k largest s_e (ties -> smaller e) in descending order,
 *   w_j = s_j / sum_j' s_j'.
 * Expert j: h = silu(G x) * (U x), y_j = D h.  Shared expert (bf16 weights,
 * weight 1, outside the renormalisation) y_s likewise.
 * out = y_s + sum_j w_j y_j.
 *
 * Pins: the closed-form block tests, gating invariants and the dense numpy
 * brute force under tests/ exercise every function exported here.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_IQ2X = 0, ORC_Q2K = 1, ORC_Q4K = 2 };

/* ---- scalar decoding, written from the IEEE 754 binary16 / bfloat16 definitions ---- */

static float half_bits_to_float(uint16_t h) {
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1F;
    int mant = h & 0x3FF;
    float v;
    if (expo == 0) {
        v = ldexpf((float)mant, -24); /* subnormal: mant * 2^-24 */
    } else if (expo == 31) {
        v = mant ? NAN : INFINITY;
    } else {
        v = ldexpf((float)(mant + 1024), expo - 25); /* (1024+mant) * 2^(e-15-10) */
    }
    return sign ? -v : v;
}

static float bf16_bits_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float v;
    memcpy(&v, &u, 4);
    return v;
}

static uint16_t rd16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static uint32_t rd32(const uint8_t *p) {
    return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}

int orc_block_bytes(int fmt) {
    switch (fmt) {
    case ORC_IQ2X: return 66;
    case ORC_Q2K: return 84;
    case ORC_Q4K: return 144;
    default: return -1;
    }
}

/* ---- block dequantization (fp32, definition op order) ---- */

static void dequant_iq2x_block(const uint8_t *b, const uint8_t *grid, float *out) {
    float d = half_bits_to_float(rd16(b));
    for (int g = 0; g < 8; g++) {
        const uint8_t *grp = b + 2 + 8 * g;
        uint32_t aux = rd32(grp + 4);
        int s = (int)(aux >> 28);
        float dl = (d * (0.5f + (float)s)) * 0.25f;
        for (int j = 0; j < 4; j++) {
            const uint8_t *gv = grid + 8 * grp[j];
            int bits7 = (int)((aux >> (7 * j)) & 0x7F);
            int parity = 0;
            for (int t = 0; t < 7; t++) parity ^= (bits7 >> t) & 1;
            for (int i = 0; i < 8; i++) {
                int neg = (i < 7) ? ((bits7 >> i) & 1) : parity;
                float w = dl * (float)gv[i];
                out[32 * g + 8 * j + i] = neg ? -w : w;
            }
        }
    }
}

static void dequant_q2k_block(const uint8_t *b, float *out) {
    float d = half_bits_to_float(rd16(b + 80));
    float dmin = half_bits_to_float(rd16(b + 82));
    for (int i = 0; i < 256; i++) {
        int sub = i / 16;
        int sc = b[sub] & 0xF;
        int m = b[sub] >> 4;
        int q = (b[16 + (i >> 2)] >> (2 * (i & 3))) & 3;
        float a = d * (float)sc;
        float c = dmin * (float)m;
        out[i] = a * (float)q - c;
    }
}

static int q4k_field6(const uint8_t *sc12, int bit) {
    int v = 0;
    for (int t = 0; t < 6; t++) {
        int pos = bit + t;
        v |= ((sc12[pos >> 3] >> (pos & 7)) & 1) << t;
    }
    return v;
}

static void dequant_q4k_block(const uint8_t *b, float *out) {
    float d = half_bits_to_float(rd16(b));
    float dmin = half_bits_to_float(rd16(b + 2));
    const uint8_t *sc12 = b + 4;
    const uint8_t *qs = b + 16;
    for (int i = 0; i < 256; i++) {
        int sub = i / 32;
        int sc = q4k_field6(sc12, 6 * sub);
        int m = q4k_field6(sc12, 48 + 6 * sub);
        int q = (i & 1) ? (qs[i >> 1] >> 4) : (qs[i >> 1] & 0xF);
        float a = d * (float)sc;
        float c = dmin * (float)m;
        out[i] = a * (float)q - c;
    }
}

static void dequant_block(int fmt, const uint8_t *b, const uint8_t *grid, float *out) {
    if (fmt == ORC_IQ2X) dequant_iq2x_block(b, grid, out);
    else if (fmt == ORC_Q2K) dequant_q2k_block(b, out);
    else dequant_q4k_block(b, out);
}

/* Dequantize n_blocks consecutive canonical blocks into out[n_blocks*256]. */
int orc_dequant(int fmt, const uint8_t *blocks, int64_t n_blocks, const uint8_t *grid, float *out) {
    int bb = orc_block_bytes(fmt);
    if (bb < 0 || !blocks || !out || n_blocks < 0) return -1;
    if (fmt == ORC_IQ2X && !grid) return -1;
    for (int64_t n = 0; n < n_blocks; n++) dequant_block(fmt, blocks + n * bb, grid, out + n * 256);
    return 0;
}

/* ---- routing ---- */

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* Scores of one token; s[E]. */
static void token_scores(const uint16_t *x, int d, const uint16_t *wr, const float *bias, int E, double *s) {
    for (int e = 0; e < E; e++) {
        double acc = 0.0;
        const uint16_t *row = wr + (size_t)e * d;
        for (int i = 0; i < d; i++) acc += (double)half_bits_to_float(row[i]) * (double)bf16_bits_to_float(x[i]);
        if (bias) acc += (double)bias[e];
        s[e] = sigmoid(acc);
    }
}

/* k-selection in descending score order, ties to the smaller expert id.
 * alt != 0 takes the (k+1)-th ranked expert in place of the k-th.
 * gap = s_(k) - s_(k+1) (HUGE_VAL when k == E). */
static void select_topk(const double *s, int E, int k, int alt, int32_t *ids, double *w, double *gap) {
    char *taken = (char *)calloc((size_t)E, 1);
    int32_t *rank = (int32_t *)malloc(sizeof(int32_t) * (size_t)(k + 1));
    int nrank = (k < E) ? k + 1 : k;
    for (int j = 0; j < nrank; j++) {
        int best = -1;
        for (int e = 0; e < E; e++) {
            if (taken[e]) continue;
            if (best < 0 || s[e] > s[best]) best = e; /* strict '>' keeps the smaller id on ties */
        }
        taken[best] = 1;
        rank[j] = best;
    }
    for (int j = 0; j < k; j++) ids[j] = rank[j];
    if (alt && k < E) ids[k - 1] = rank[k];
    if (gap) *gap = (k < E) ? s[rank[k - 1]] - s[rank[k]] : HUGE_VAL;
    double tot = 0.0;
    for (int j = 0; j < k; j++) tot += s[ids[j]];
    for (int j = 0; j < k; j++) w[j] = s[ids[j]] / tot;
    free(taken);
    free(rank);
}

int orc_route(const uint16_t *x, int T, int d, const uint16_t *wr, const float *bias, int E, int k, int alt,
              int32_t *ids, double *w, double *scores, double *gap) {
    if (!x || !wr || !ids || !w || T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E) return -1;
    double *s = (double *)malloc(sizeof(double) * (size_t)E);
    for (int t = 0; t < T; t++) {
        token_scores(x + (size_t)t * d, d, wr, bias, E, s);
        if (scores) memcpy(scores + (size_t)t * E, s, sizeof(double) * (size_t)E);
        select_topk(s, E, k, alt, ids + (size_t)t * k, w + (size_t)t * k, gap ? gap + t : NULL);
    }
    free(s);
    return 0;
}

/* ---- whole layer ---- */

typedef struct {
    int d, f, E, k, f_shared;
    int fmt_gate, fmt_up, fmt_down;
    const uint8_t *const *gate; /* per expert canonical matrix [f x d], NULL if absent */
    const uint8_t *const *up;   /* [f x d] */
    const uint8_t *const *down; /* [d x f] */
    const uint8_t *grid;        /* 256 x 8 */
    const uint16_t *sh_gate;    /* bf16 [f_shared x d] or NULL */
    const uint16_t *sh_up;
    const uint16_t *sh_down;    /* bf16 [d x f_shared] */
    const uint16_t *wr;         /* fp16 [E x d] */
    const float *bias;          /* [E] or NULL */
} orc_layer;

/* y[r] = sum_c W[r, c] v[c] for a canonical quantized matrix [rows x cols]. */
static void qmatvec(int fmt, const uint8_t *mat, int rows, int cols, const uint8_t *grid, const double *v,
                    double *y, float *rowbuf) {
    int nb = cols / 256;
    int bb = orc_block_bytes(fmt);
    for (int r = 0; r < rows; r++) {
        const uint8_t *rowp = mat + (size_t)r * nb * bb;
        for (int b = 0; b < nb; b++) dequant_block(fmt, rowp + (size_t)b * bb, grid, rowbuf + 256 * b);
        double acc = 0.0;
        for (int c = 0; c < cols; c++) acc += (double)rowbuf[c] * v[c];
        y[r] = acc;
    }
}

static void bmatvec(const uint16_t *mat, int rows, int cols, const double *v, double *y) {
    for (int r = 0; r < rows; r++) {
        double acc = 0.0;
        const uint16_t *row = mat + (size_t)r * cols;
        for (int c = 0; c < cols; c++) acc += (double)bf16_bits_to_float(row[c]) * v[c];
        y[r] = acc;
    }
}

static double silu(double g) { return g * sigmoid(g); }

typedef struct {
    const orc_layer *L;
    const uint16_t *x;
    int T, alt;
    int32_t *ids;
    double *w, *gap, *out;
    int t0, t1, status;
} orc_job;

static void *layer_worker(void *arg) {
    orc_job *jb = (orc_job *)arg;
    const orc_layer *L = jb->L;
    int d = L->d, f = L->f, fs = L->f_shared, k = L->k;
    int fmax = f > fs ? f : fs;
    int cmax = d > fmax ? d : fmax;
    double *xv = (double *)malloc(sizeof(double) * (size_t)d);
    double *g = (double *)malloc(sizeof(double) * (size_t)fmax);
    double *u = (double *)malloc(sizeof(double) * (size_t)fmax);
    double *y = (double *)malloc(sizeof(double) * (size_t)d);
    double *s = (double *)malloc(sizeof(double) * (size_t)L->E);
    float *rowbuf = (float *)malloc(sizeof(float) * (size_t)cmax);
    for (int t = jb->t0; t < jb->t1 && jb->status == 0; t++) {
        const uint16_t *xt = jb->x + (size_t)t * d;
        for (int i = 0; i < d; i++) xv[i] = (double)bf16_bits_to_float(xt[i]);
        int32_t *ids = jb->ids + (size_t)t * k;
        double *w = jb->w + (size_t)t * k;
        token_scores(xt, d, L->wr, L->bias, L->E, s);
        select_topk(s, L->E, k, jb->alt, ids, w, jb->gap ? jb->gap + t : NULL);
        double *out = jb->out + (size_t)t * d;
        for (int n = 0; n < d; n++) out[n] = 0.0;
        if (fs > 0 && L->sh_gate && L->sh_up && L->sh_down) {
            bmatvec(L->sh_gate, fs, d, xv, g);
            bmatvec(L->sh_up, fs, d, xv, u);
            for (int r = 0; r < fs; r++) g[r] = silu(g[r]) * u[r];
            bmatvec(L->sh_down, d, fs, g, y);
            for (int n = 0; n < d; n++) out[n] += y[n];
        }
        for (int j = 0; j < k; j++) {
            int e = ids[j];
            if (!L->gate[e] || !L->up[e] || !L->down[e]) {
                jb->status = -2 - e; /* a selected expert was not supplied */
                break;
            }
            qmatvec(L->fmt_gate, L->gate[e], f, d, L->grid, xv, g, rowbuf);
            qmatvec(L->fmt_up, L->up[e], f, d, L->grid, xv, u, rowbuf);
            for (int r = 0; r < f; r++) g[r] = silu(g[r]) * u[r];
            qmatvec(L->fmt_down, L->down[e], d, f, L->grid, g, y, rowbuf);
            for (int n = 0; n < d; n++) out[n] += w[j] * y[n];
        }
    }
    free(xv); free(g); free(u); free(y); free(s); free(rowbuf);
    return NULL;
}

/* Full layer for T tokens, threads over tokens.  out: fp64 [T x d];
 * ids [T x k], w [T x k], gap [T] (nullable). Returns 0, or <0 on error. */
int orc_layer_forward(const orc_layer *L, const uint16_t *x, int T, int alt, int nthreads, int32_t *ids, double *w,
                      double *gap, double *out) {
    if (!L || !x || !ids || !w || !out || T < 0) return -1;
    if (L->d % 256 || L->f % 256 || L->f_shared % 256 || L->k <= 0 || L->k > L->E) return -1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > T) nthreads = T > 0 ? T : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    orc_job *jobs = (orc_job *)calloc((size_t)nthreads, sizeof(orc_job));
    for (int i = 0; i < nthreads; i++) {
        jobs[i] = (orc_job){L, x, T, alt, ids, w, gap, out, (int)((int64_t)T * i / nthreads),
                            (int)((int64_t)T * (i + 1) / nthreads), 0};
        pthread_create(&th[i], NULL, layer_worker, &jobs[i]);
    }
    int status = 0;
    for (int i = 0; i < nthreads; i++) {
        pthread_join(th[i], NULL);
        if (jobs[i].status) status = jobs[i].status;
    }
    free(th);
    free(jobs);
    return status;
}
