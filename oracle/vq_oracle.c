/*
 * vq_oracle.c -- plain CPU reference ("oracle") for the bit-packed VQ/RVQ
 * linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  The product path (the CUDA library and its Python
 * binding) never links, loads or calls this file; only the tests, the smoke
 * check and the benchmark's CPU-baseline leg do.  It shares no code, header,
 * table or constant with the CUDA path and includes no CUDA header.
 *
 * Every routine is the plain definition of what the method computes, written
 * for a reader to check by eye, with no blocking, fusion or reordering:
 *
 *  - fp16 / bf16 <-> fp32 conversions from the IEEE 754 definitions
 *    (round to nearest, ties to even; subnormals kept; overflow to infinity).
 *  - unpack / pack of b-bit index fields, one bit at a time, in the row
 *    order and in the tiled order (four vectors per tile, rows consecutive).
 *  - dequantisation: w_hat = C1[i1] (+ C2[i2]), times the row scale, plus the
 *    row bias, each an fp32 operation rounded to nearest-even, in that order,
 *    then rounded once to fp16.  Follows "VPTQ Guide: Extreme 2-Bit Vector
 *    Quantization", section "2. Multi-Stage Residual Vector Quantization
 *    (RVQ)" (the reconstruction is the sum of the primary and residual
 *    centroids) and section "Step 2" (dequantize: gather both books, add,
 *    reshape to (out, in)); "Vector Quantization for LLM Weights in
 *    Production", section "2. AQLM: Additive Multi-Codebook Vector
 *    Quantization" (sum over M = 1 or 2 books) and section "1. QuIP#" (per-
 *    channel scaling).
 *  - products y = x . W_hat^T accumulated in fp64 in ascending k order
 *    ("VPTQ Guide", section "Step 3: Fused Low-Bit VPTQ Linear Layer":
 *    forward computes y = x @ W^T with the dequantised weights), plus an
 *    optional fp16 output bias b_out[o] added once in fp64 (the same
 *    section's F.linear(x, W_hat, bias)).
 *  - the normalised, damped activation Hessian H = 2 X^T X / n + damping
 *    (section "Hessian collection" below);
 *  - the randomized Hadamard transform of QuIP#-style incoherence processing
 *    (plain O(n b) sums; section "Randomized Hadamard transform" below);
 *  - nearest-centroid encoding by brute force, ties to the lowest index
 *    ("VPTQ Guide", section "The Information-Theoretic Superiority of Vector
 *    Quantization": q = argmin_k ||w - c_k||^2; section "2. Multi-Stage
 *    Residual Vector Quantization (RVQ)" for the residual stage).
 *  - the Hessian-weighted variant, D_H(v, c) = (v - c)^T H_v (v - c) with H_v
 *    the vector's sub-matrix of the layer Hessian ("VPTQ Guide", section
 *    "1. Second-Order Hessian-Weighted Optimization"), by brute force.
 *
 * Readings of points the pages leave open (stated once here):
 *  - index fields are unsigned; field j of a row occupies bits [j*b, j*b+b),
 *    bits numbered LSB-first inside little-endian 32-bit words;
 *  - nvec = ceil(in_features / d); centroid components past in_features are
 *    ignored (neither stored nor multiplied);
 *  - a missing scale skips the multiply, a missing bias skips the add.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -shared
 * -fPIC.  FLT_EVAL_METHOD must be 0 (every float operation rounds to float),
 * which holds on x86-64 (SSE) and aarch64.
 */
#include <float.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#if !defined(FLT_EVAL_METHOD) || FLT_EVAL_METHOD != 0
#error "the oracle needs FLT_EVAL_METHOD == 0 (float operations rounded to float)"
#endif

/* ---------------------------------------------------------------------- */
/* Rounding to a binary format, from the IEEE 754 definition.              */
/* ---------------------------------------------------------------------- */

/* Round the finite double v to the nearest value representable with p
 * significand bits and minimum normal exponent emin (values below 2^emin are
 * subnormal with spacing 2^(emin - p + 1)), ties to even.  Overflow is left to
 * the caller.  v must be exactly a float (so every step below is exact). */
static double round_to_format(double v, int p, int emin) {
    if (v == 0.0) return v;
    double a = fabs(v);
    int e;                      /* a = f * 2^e with f in [0.5, 1) */
    frexp(a, &e);
    int exp2 = e - 1;           /* a in [2^exp2, 2^(exp2+1)) */
    if (exp2 < emin) exp2 = emin;
    double quantum = ldexp(1.0, exp2 - (p - 1));   /* spacing in this binade */
    double q = a / quantum;                        /* exact: scaling by 2^n */
    double fl = floor(q);
    double r = q - fl;
    double n;
    if (r > 0.5) n = fl + 1.0;
    else if (r < 0.5) n = fl;
    else n = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    double out = n * quantum;
    return v < 0 ? -out : out;
}

/* fp16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
uint16_t vqo_f32_to_f16(float f) {
    if (isnan(f)) return 0x7e00u;
    uint16_t sign = signbit(f) ? 0x8000u : 0u;
    if (isinf(f)) return sign | 0x7c00u;
    double r = round_to_format((double)f, 11, -14);
    double a = fabs(r);
    if (a >= 65536.0) return sign | 0x7c00u;           /* rounded past 65504 */
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);
    int exp2 = e - 1;
    if (exp2 < -14) {                                   /* subnormal */
        uint32_t m = (uint32_t)(a / ldexp(1.0, -24));
        return sign | (uint16_t)m;
    }
    uint32_t frac = (uint32_t)(a / ldexp(1.0, exp2 - 10)) - 1024u;
    return sign | (uint16_t)((uint32_t)(exp2 + 15) << 10) | (uint16_t)frac;
}

float vqo_f16_to_f32(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(1024 + m), e - 25);
    return (float)(sign ? -v : v);
}

/* bf16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
uint16_t vqo_f32_to_bf16(float f) {
    if (isnan(f)) return 0x7fc0u;
    uint16_t sign = signbit(f) ? 0x8000u : 0u;
    if (isinf(f)) return sign | 0x7f80u;
    double r = round_to_format((double)f, 8, -126);
    double a = fabs(r);
    if (a >= ldexp(1.0, 128)) return sign | 0x7f80u;
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);
    int exp2 = e - 1;
    if (exp2 < -126) {
        uint32_t m = (uint32_t)(a / ldexp(1.0, -133));
        return sign | (uint16_t)m;
    }
    uint32_t frac = (uint32_t)(a / ldexp(1.0, exp2 - 7)) - 128u;
    return sign | (uint16_t)((uint32_t)(exp2 + 127) << 7) | (uint16_t)frac;
}

float vqo_bf16_to_f32(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 7) & 0xff;
    int m = h & 0x7f;
    double v;
    if (e == 0) v = ldexp((double)m, -133);
    else if (e == 255) v = m ? NAN : INFINITY;
    else v = ldexp((double)(128 + m), e - 134);
    return (float)(sign ? -v : v);
}

void vqo_f32_to_f16_array(const float* in, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = vqo_f32_to_f16(in[i]);
}
void vqo_f16_to_f32_array(const uint16_t* in, float* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = vqo_f16_to_f32(in[i]);
}
void vqo_f32_to_bf16_array(const float* in, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = vqo_f32_to_bf16(in[i]);
}
void vqo_bf16_to_f32_array(const uint16_t* in, float* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = vqo_bf16_to_f32(in[i]);
}

/* ---------------------------------------------------------------------- */
/* Index fields.                                                           */
/* ---------------------------------------------------------------------- */

static uint32_t get_bit(const uint32_t* words, int64_t p) {
    return (words[p >> 5] >> (p & 31)) & 1u;
}

/* Field j of one stream row: bits [j*b, j*b+b), least significant first. */
static uint32_t field(const uint32_t* row, int b, int64_t j) {
    uint32_t v = 0;
    for (int t = 0; t < b; ++t) v |= get_bit(row, j * (int64_t)b + t) << t;
    return v;
}

/* Unpack n rows of nvec b-bit fields (row stride row_words) into idx[n][nvec]. */
int vqo_unpack(const uint32_t* words, int64_t n, int64_t row_words, int b, int64_t nvec,
               uint32_t* idx) {
    if (b < 1 || b > 32 || nvec * (int64_t)b > row_words * 32) return 1;
    for (int64_t o = 0; o < n; ++o)
        for (int64_t j = 0; j < nvec; ++j)
            idx[o * nvec + j] = field(words + o * row_words, b, j);
    return 0;
}

/* Pack idx[n][nvec] into zeroed rows of row_words words.  Fields wider than b
 * bits are an error. */
int vqo_pack(const uint32_t* idx, int64_t n, int64_t nvec, int b, int64_t row_words,
             uint32_t* words) {
    if (b < 1 || b > 32 || nvec * (int64_t)b > row_words * 32) return 1;
    memset(words, 0, (size_t)(n * row_words) * sizeof(uint32_t));
    for (int64_t o = 0; o < n; ++o) {
        uint32_t* row = words + o * row_words;
        for (int64_t j = 0; j < nvec; ++j) {
            uint32_t v = idx[o * nvec + j];
            if (b < 32 && (v >> b) != 0) return 2;
            for (int t = 0; t < b; ++t) {
                int64_t p = j * (int64_t)b + t;
                row[p >> 5] |= ((v >> t) & 1u) << (p & 31);
            }
        }
    }
    return 0;
}

/* The tiled arrangement of the same fields ("tile4", this library's second
 * storage order; the pages fix only the field width).  A book's stream is a
 * sequence of tiles tile_words words apart; tile t covers vectors 4t..4t+3.
 * Inside a tile the rows follow one another, row o contributing one record of
 * four b-bit fields: those of vectors 4t, 4t+1, 4t+2, 4t+3, in that order.
 * So field (o, j) occupies bits [(4*o + j%4)*b, +b) of tile j/4, numbered as
 * in the row stream.  Fields of vectors >= nvec (the tail of the last tile)
 * are written as zero and never read. */
static int64_t tile4_count(int64_t nvec) { return (nvec + 3) / 4; }

int vqo_unpack_tile4(const uint32_t* words, int64_t n, int64_t tile_words, int b, int64_t nvec,
                     uint32_t* idx) {
    if (b < 1 || b > 32 || n * 4 * (int64_t)b > tile_words * 32) return 1;
    for (int64_t o = 0; o < n; ++o)
        for (int64_t j = 0; j < nvec; ++j)
            idx[o * nvec + j] = field(words + (j / 4) * tile_words, b, 4 * o + j % 4);
    return 0;
}

int vqo_pack_tile4(const uint32_t* idx, int64_t n, int64_t nvec, int b, int64_t tile_words,
                   uint32_t* words) {
    if (b < 1 || b > 32 || n * 4 * (int64_t)b > tile_words * 32) return 1;
    memset(words, 0, (size_t)(tile4_count(nvec) * tile_words) * sizeof(uint32_t));
    for (int64_t o = 0; o < n; ++o) {
        for (int64_t j = 0; j < nvec; ++j) {
            uint32_t v = idx[o * nvec + j];
            if (b < 32 && (v >> b) != 0) return 2;
            uint32_t* tile = words + (j / 4) * tile_words;
            for (int t = 0; t < b; ++t) {
                int64_t p = (4 * o + j % 4) * (int64_t)b + t;
                tile[p >> 5] |= ((v >> t) & 1u) << (p & 31);
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------- */
/* Layer description and dequantisation.                                   */
/* ---------------------------------------------------------------------- */

typedef struct {
    int64_t out_features;          /* N */
    int64_t in_features;           /* Kin */
    int32_t d;                     /* vector length */
    int32_t n_books;               /* 1 or 2 */
    int32_t log2k[2];              /* b per book, K = 2^b */
    const uint32_t* idx[2];        /* packed streams, [N][row_words] */
    int64_t row_words[2];
    const uint16_t* codebook[2];   /* fp16 [K][d] */
    const uint16_t* scale;         /* fp16 [N] or NULL */
    const uint16_t* bias;          /* fp16 [N] or NULL */
    const uint16_t* out_bias;      /* fp16 [N] or NULL: output-side bias of the product */
} vqo_layer;

static int64_t nvec_of(const vqo_layer* L) { return (L->in_features + L->d - 1) / L->d; }

static int check_layer(const vqo_layer* L) {
    if (L->out_features < 0 || L->in_features < 0 || L->d < 1 || L->n_books < 1 ||
        L->n_books > 2)
        return 1;
    for (int m = 0; m < L->n_books; ++m) {
        if (L->log2k[m] < 1 || L->log2k[m] > 16) return 1;
        if (nvec_of(L) * L->log2k[m] > L->row_words[m] * 32) return 1;
    }
    return 0;
}

/* One dequantised row o into w[0..Kin): the definition, element by element. */
static void dequant_row(const vqo_layer* L, int64_t o, uint16_t* w) {
    const int64_t nvec = nvec_of(L);
    const int d = L->d;
    for (int64_t j = 0; j < nvec; ++j) {
        uint32_t i1 = field(L->idx[0] + o * L->row_words[0], L->log2k[0], j);
        uint32_t i2 = 0;
        if (L->n_books == 2) i2 = field(L->idx[1] + o * L->row_words[1], L->log2k[1], j);
        for (int e = 0; e < d; ++e) {
            int64_t k = j * d + e;
            if (k >= L->in_features) break;          /* partial last vector */
            float v = vqo_f16_to_f32(L->codebook[0][(int64_t)i1 * d + e]);
            if (L->n_books == 2) {
                float c2 = vqo_f16_to_f32(L->codebook[1][(int64_t)i2 * d + e]);
                v = v + c2;                              /* fp32 add, RNE */
            }
            if (L->scale) v = v * vqo_f16_to_f32(L->scale[o]);   /* fp32 mul, RNE */
            if (L->bias) v = v + vqo_f16_to_f32(L->bias[o]);     /* fp32 add, RNE */
            w[k] = vqo_f32_to_f16(v);
        }
    }
}

/* W_hat fp16 [N][ldw]; columns >= Kin are not touched. */
int vqo_dequant(const vqo_layer* L, uint16_t* w, int64_t ldw) {
    if (check_layer(L) || ldw < L->in_features) return 1;
    int64_t n = L->out_features;
#pragma omp parallel for schedule(static)
    for (int64_t o = 0; o < n; ++o) dequant_row(L, o, w + o * ldw);
    return 0;
}

/* Dequantise only the listed rows into w[r][ldw] for r = 0..nrows-1. */
int vqo_dequant_rows(const vqo_layer* L, const int64_t* rows, int64_t nrows, uint16_t* w,
                     int64_t ldw) {
    if (check_layer(L) || ldw < L->in_features) return 1;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= L->out_features) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) dequant_row(L, rows[r], w + r * ldw);
    return 0;
}

/* ---------------------------------------------------------------------- */
/* Products in fp64.                                                       */
/* ---------------------------------------------------------------------- */

/* x: [M][ldx] activations, bf16 bits (x_is_fp16 = 0) or fp16 bits (1). */
static double act(const uint16_t* x, int x_is_fp16, int64_t i) {
    return x_is_fp16 ? (double)vqo_f16_to_f32(x[i]) : (double)vqo_bf16_to_f32(x[i]);
}

/* y[m][n] = sum_k x[m][k] * w[n][k], fp64, k ascending.  w is fp16 [N][ldw]. */
int vqo_matmul(int64_t M, int64_t N, int64_t Kin, const uint16_t* x, int x_is_fp16,
               int64_t ldx, const uint16_t* w, int64_t ldw, double* y, int64_t ldy) {
    if (M < 0 || N < 0 || Kin < 0 || ldx < Kin || ldw < Kin || ldy < N) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t m = 0; m < M; ++m) {
            double s = 0.0;
            for (int64_t k = 0; k < Kin; ++k)
                s += act(x, x_is_fp16, m * ldx + k) * (double)vqo_f16_to_f32(w[n * ldw + k]);
            y[m * ldy + n] = s;
        }
    }
    return 0;
}

/* The layer's forward pass for the listed output rows (all rows when rows is
 * NULL): dequantise row o, then y[m][c] = sum_k x[m][k] * w_hat[o][k] in fp64,
 * where c is the position of o in the list, plus out_bias[o] (when given)
 * added once, in fp64, after the sum: the layer's forward ends in
 * F.linear(x, W_hat, bias), an output-side bias over the product ("VPTQ
 * Guide", section "Step 3: Fused Low-Bit VPTQ Linear Layer").  That bias is
 * separate from the per-row bias t folded into W_hat above.  Uses one row
 * buffer per thread, so it runs on full-size layers without materialising
 * W_hat. */
int vqo_linear(const vqo_layer* L, const uint16_t* x, int x_is_fp16, int64_t M, int64_t ldx,
               const int64_t* rows, int64_t nrows, double* y, int64_t ldy) {
    if (check_layer(L) || M < 0 || ldx < L->in_features) return 1;
    const int64_t n_out = rows ? nrows : L->out_features;
    if (ldy < n_out) return 1;
    if (rows)
        for (int64_t r = 0; r < nrows; ++r)
            if (rows[r] < 0 || rows[r] >= L->out_features) return 1;
    const int64_t kin = L->in_features;
    int bad = 0;
#pragma omp parallel
    {
        uint16_t* w = (uint16_t*)malloc((size_t)(kin > 0 ? kin : 1) * sizeof(uint16_t));
        if (!w) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t c = 0; c < n_out; ++c) {
                int64_t o = rows ? rows[c] : c;
                dequant_row(L, o, w);
                for (int64_t m = 0; m < M; ++m) {
                    double s = 0.0;
                    for (int64_t k = 0; k < kin; ++k)
                        s += act(x, x_is_fp16, m * ldx + k) * (double)vqo_f16_to_f32(w[k]);
                    if (L->out_bias) s += (double)vqo_f16_to_f32(L->out_bias[o]);
                    y[m * ldy + c] = s;
                }
            }
            free(w);
        }
    }
    return bad ? 2 : 0;
}

/* ---------------------------------------------------------------------- */
/* Brute-force nearest-centroid encoding (tests only).                     */
/* ---------------------------------------------------------------------- */

/* For each of nv vectors v[i][0..d) (fp64), idx[i] = argmin_k sum_e
 * (v_e - C[k][e])^2 over the fp16 book C[K][d], ties to the lowest k. */
int vqo_encode(const double* v, int64_t nv, int d, const uint16_t* book, int64_t K,
               uint32_t* idx) {
    if (d < 1 || K < 1) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nv; ++i) {
        double best = INFINITY;
        int64_t arg = 0;
        for (int64_t k = 0; k < K; ++k) {
            double dist = 0.0;
            for (int e = 0; e < d; ++e) {
                double t = v[i * d + e] - (double)vqo_f16_to_f32(book[k * d + e]);
                dist += t * t;
            }
            if (dist < best) { best = dist; arg = k; }
        }
        idx[i] = (uint32_t)arg;
    }
    return 0;
}

/* Two-stage residual encoding, the greedy cascade: i1 = nearest centroid of
 * book 1, r = v - C1[i1], i2 = nearest centroid of book 2 to r. */
int vqo_encode_residual(const double* v, int64_t nv, int d, const uint16_t* book1, int64_t K1,
                        const uint16_t* book2, int64_t K2, uint32_t* idx1, uint32_t* idx2) {
    if (vqo_encode(v, nv, d, book1, K1, idx1)) return 1;
    double* r = (double*)malloc((size_t)(nv > 0 ? nv : 1) * (size_t)d * sizeof(double));
    if (!r) return 2;
    for (int64_t i = 0; i < nv; ++i)
        for (int e = 0; e < d; ++e)
            r[i * d + e] = v[i * d + e] - (double)vqo_f16_to_f32(book1[(int64_t)idx1[i] * d + e]);
    int rc = vqo_encode(r, nv, d, book2, K2, idx2);
    free(r);
    return rc;
}

/* Hessian-weighted encoding ("VPTQ Guide: Extreme 2-Bit Vector
 * Quantization", section "1. Second-Order Hessian-Weighted Optimization"):
 * the distance of vector v to centroid c is D_H(v, c) = (v - c)^T H_v (v - c),
 * with H_v the d x d sub-matrix of the layer's Hessian on the channels of v.
 * For each of nv vectors v[i][0..d) (fp64) with its own sub-matrix
 * hb[i][e][f] (fp64, row-major d x d), idx[i] = argmin_k D_H(v_i, C[k]) over
 * the fp16 book C[K][d], ties to the lowest k.  Evaluation order (every
 * operation rounded once in fp64, no fused multiply-add): t_e = v_e - C[k][e];
 * g_e = sum_f hb[e][f] t_f, f ascending; D = sum_e t_e g_e, e ascending.  A
 * NaN distance never wins; with no finite distance the index is 0. */
static double dist_h(const double* v, const double* h, const uint16_t* c, int d, double* t) {
    for (int e = 0; e < d; ++e) t[e] = v[e] - (double)vqo_f16_to_f32(c[e]);
    double dist = 0.0;
    for (int e = 0; e < d; ++e) {
        double g = 0.0;
        for (int f = 0; f < d; ++f) g += h[e * d + f] * t[f];
        dist += t[e] * g;
    }
    return dist;
}

int vqo_encode_h(const double* v, int64_t nv, int d, const double* hb, const uint16_t* book,
                 int64_t K, uint32_t* idx) {
    if (d < 1 || d > 64 || K < 1) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nv; ++i) {
        double t[64];
        double best = INFINITY;
        int64_t arg = 0;
        for (int64_t k = 0; k < K; ++k) {
            double dist = dist_h(v + i * d, hb + i * d * d, book + k * d, d, t);
            if (dist < best) { best = dist; arg = k; }
        }
        idx[i] = (uint32_t)arg;
    }
    return 0;
}

/* The two-stage cascade under the weighted distance: i1 = argmin_k
 * D_H(v, C1[k]); r = v - C1[i1] (fp64); i2 = argmin_k D_H(r, C2[k]) with the
 * same sub-matrix.  The page writes the residual stage with the plain
 * distance; with H_v = I the two coincide, and weighting it keeps the second
 * stage minimising the same objective for the final reconstruction. */
int vqo_encode_h_residual(const double* v, int64_t nv, int d, const double* hb,
                          const uint16_t* book1, int64_t K1, const uint16_t* book2, int64_t K2,
                          uint32_t* idx1, uint32_t* idx2) {
    if (vqo_encode_h(v, nv, d, hb, book1, K1, idx1)) return 1;
    double* r = (double*)malloc((size_t)(nv > 0 ? nv : 1) * (size_t)d * sizeof(double));
    if (!r) return 2;
    for (int64_t i = 0; i < nv; ++i)
        for (int e = 0; e < d; ++e)
            r[i * d + e] = v[i * d + e] - (double)vqo_f16_to_f32(book1[(int64_t)idx1[i] * d + e]);
    int rc = vqo_encode_h(r, nv, d, hb, book2, K2, idx2);
    free(r);
    return rc;
}

/* Joint two-book search: (i1, i2) = argmin ||v - (C1[i1] + C2[i2])||^2 over all
 * pairs, the sum taken in fp64; ties to the lowest (i1, i2) in lexicographic
 * order.  For tiny books only (K1 * K2 distance evaluations per vector). */
int vqo_encode_joint(const double* v, int64_t nv, int d, const uint16_t* book1, int64_t K1,
                     const uint16_t* book2, int64_t K2, uint32_t* idx1, uint32_t* idx2) {
    if (d < 1 || K1 < 1 || K2 < 1) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nv; ++i) {
        double best = INFINITY;
        int64_t a1 = 0, a2 = 0;
        for (int64_t k1 = 0; k1 < K1; ++k1)
            for (int64_t k2 = 0; k2 < K2; ++k2) {
                double dist = 0.0;
                for (int e = 0; e < d; ++e) {
                    double c = (double)vqo_f16_to_f32(book1[k1 * d + e]) +
                               (double)vqo_f16_to_f32(book2[k2 * d + e]);
                    double t = v[i * d + e] - c;
                    dist += t * t;
                }
                if (dist < best) { best = dist; a1 = k1; a2 = k2; }
            }
        idx1[i] = (uint32_t)a1;
        idx2[i] = (uint32_t)a2;
    }
    return 0;
}

/* ---------------------------------------------------------------------- */
/* Randomized Hadamard transform (tests only).                             */
/* ---------------------------------------------------------------------- */

/* Incoherence processing: W~ = U W V^T and x~ = V x with U, V orthogonal
 * randomized Walsh-Hadamard matrices, so y = W x = U^T (W~ x~) ("Vector
 * Quantization for LLM Weights in Production", section "1. QuIP#:
 * Incoherence Processing and Lattice Codebooks"; "Sub-4-Bit Quantization",
 * section "QuIP#: Incoherence Processing": Hadamard plus random signs).
 * Reading for lengths that are not powers of two: the transform of a row of
 * length n is block diagonal, blocks of b = the largest power of two that
 * divides n (at most 2^15), i.e. (I ⊗ H_b) diag(s) / sqrt(b).
 *   forward:  out[k*b + i] = b^-1/2 * sum_j H_b[i][j] * s[k*b + j] * in[k*b + j]
 *   inverse:  out[k*b + j] = s[k*b + j] * b^-1/2 * sum_i H_b[j][i] * in[k*b + i]
 * with H_b[i][j] = (-1)^popcount(i & j) (Sylvester's construction) and
 * s[t] = -1 where bit t of `signs` is set (LSB first in 32-bit words), +1
 * otherwise.  Plain O(n b) sums in fp64, j (or i) ascending. */
int64_t vqo_rht_block(int64_t n) {
    if (n <= 0) return 0;
    int64_t b = 1;
    while (b < 32768 && n % (2 * b) == 0) b *= 2;
    return b;
}

static double hadamard_entry(int64_t i, int64_t j) {
    return (__builtin_popcountll((unsigned long long)(i & j)) & 1) ? -1.0 : 1.0;
}

static double sign_of(const uint32_t* signs, int64_t t) {
    return (signs[t >> 5] >> (t & 31)) & 1u ? -1.0 : 1.0;
}

int vqo_rht(const double* in, int64_t rows, int64_t n, const uint32_t* signs, int inverse, double* out) {
    if (rows < 0 || n < 0) return 1;
    const int64_t b = vqo_rht_block(n);
    const double scale = b > 0 ? 1.0 / sqrt((double)b) : 0.0;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double* x = in + r * n;
        double* y = out + r * n;
        for (int64_t k0 = 0; k0 < n; k0 += b) {
            for (int64_t i = 0; i < b; ++i) {
                double acc = 0.0;
                for (int64_t j = 0; j < b; ++j) {
                    const double v = inverse ? x[k0 + j] : sign_of(signs, k0 + j) * x[k0 + j];
                    acc += hadamard_entry(i, j) * v;
                }
                y[k0 + i] = inverse ? sign_of(signs, k0 + i) * (acc * scale) : acc * scale;
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------- */
/* Hessian collection (tests only).                                        */
/* ---------------------------------------------------------------------- */

/* The normalised, damped activation Hessian of a layer's inputs ("VPTQ
 * Guide", section "Step 1: Hessian Matrix Collection", and section "1.
 * Second-Order Hessian-Weighted Optimization": H = 2 X X^T over the tokens):
 *   H[i][j] = sum_t 2 x_t[i] x_t[j]        (fp64, tokens t ascending)
 *   h = H / n_tokens;  damp = 0.01 * mean_i h[i][i];  h[i][i] += damp
 * x: n_tokens rows of d values, bf16 (x_is_fp16 = 0) or fp16 bits, row
 * stride ldx.  out: fp64 [d][d]. */
int vqo_hessian(const uint16_t* x, int x_is_fp16, int64_t n_tokens, int64_t d, int64_t ldx, double* out) {
    if (n_tokens < 1 || d < 0 || ldx < d) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d; ++i) {
        for (int64_t j = 0; j < d; ++j) {
            double acc = 0.0;
            for (int64_t t = 0; t < n_tokens; ++t)
                acc += 2.0 * act(x, x_is_fp16, t * ldx + i) * act(x, x_is_fp16, t * ldx + j);
            out[i * d + j] = acc / (double)n_tokens;
        }
    }
    double diag = 0.0;
    for (int64_t i = 0; i < d; ++i) diag += out[i * d + i];
    const double damp = d > 0 ? 0.01 * (diag / (double)d) : 0.0;
    for (int64_t i = 0; i < d; ++i) out[i * d + i] += damp;
    return 0;
}

int vqo_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
