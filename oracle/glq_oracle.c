/*
 * glq_oracle.c -- plain, slow fp64 CPU oracle for the GLQ compressed-weight
 * linear layer  y = S_out . H_m . W^ . H_n . (S_in . x).  Single-threaded,
 * except that the rows of the middle product may be dealt out to threads
 * (glq_oracle_linear_mt; every output element is the same loop either way).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package entry point's
 * smoke check and the benchmark's CPU-baseline leg may load this file.  The
 * CUDA library never links, includes or calls it, and it shares no code,
 * table or constant with the CUDA library.
 *
 * Sources (pages of the GLQ project, as cited):
 *   [glq 0.5.1 PyPI page, "How it works" 1]  65,536 vectors from the first
 *       seven shells of the E8 lattice; one 16-bit index per 8-weight group;
 *       8-bit (256-entry) or 16-bit (E8) residual codebooks refine it.
 *   [glq 0.5.1 PyPI page, "How it works" 2]  random sign flips followed by a
 *       fast Walsh-Hadamard transform (the RHT).
 *   [glq 0.5.1 PyPI page, "Bit widths"]  one global scale per layer; a
 *       non-power-of-two size uses a block-diagonal Hadamard over the binary
 *       decomposition of the size (the page's example: 2688 = 2048+512+128).
 *   [glq 0.5.1 PyPI page, "Inference kernels"]  Y = X . dequant(W)^T with the
 *       residual index/codebook and the inverse residual scale as arguments.
 *
 * Readings where the pages leave a step open (each also listed in the
 * design notes of the repository):
 *   - codebook = all E8 points of squared norm <= 12 sorted by (squared norm,
 *     x0, x1, ..., x7) ascending, first 65,536 kept (origin included);
 *   - index layout [m][n/8], group g of row r covers columns 8g..8g+7;
 *   - w^ = ws * (cb1 + rs * cb2), where rs is the multiplier applied at
 *     decode; rounding: c = fmaf(rs, cb2, cb1) (single rounding), then
 *     w^ = fp32(ws * c) (single rounding);
 *   - 5-8 bpw: the residual stages of the "Bit widths" table in its order
 *     (16-bit E8 stages, then the 8-bit stage of an odd bpw), each with its
 *     own scale, added one fmaf per stage in that order;
 *   - H_k[i][j] = (-1)^popcount(i & j) / sqrt(k) (Sylvester order); blocks in
 *     descending size at increasing offsets;
 *   - input side: sign, then H; output side: H, then sign.
 *
 * Parity pins live in the test-suite; none of the functions here is unpinned.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* scalar formats: the plain IEEE-754 binary16 and bfloat16 definitions  */
/* ------------------------------------------------------------------ */

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double glq_oracle_f16_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24); /* subnormal: f * 2^-14 * 2^-10 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16: the upper half of a binary32. */
double glq_oracle_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------ */
/* E8 shell codebook  [glq 0.5.1, "How it works" 1]                     */
/* ------------------------------------------------------------------ */

/* A lattice point is held as y = 2x (integers); E8 = D8 u (D8 + 1/2):
 * either every x_i is an integer or every x_i is an integer plus 1/2, and
 * sum(x_i) is even.  Squared norm ||x||^2 = sum(y_i^2) / 4 <= 12 means
 * sum(y_i^2) <= 48, so |y_i| <= 6.                                      */
typedef struct {
    int norm4; /* sum(y_i^2) = 4 ||x||^2 */
    int y[8];
} e8_point;

static int e8_point_cmp(const void *pa, const void *pb) {
    const e8_point *a = (const e8_point *)pa, *b = (const e8_point *)pb;
    if (a->norm4 != b->norm4) return a->norm4 < b->norm4 ? -1 : 1;
    for (int i = 0; i < 8; i++)
        if (a->y[i] != b->y[i]) return a->y[i] < b->y[i] ? -1 : 1;
    return 0;
}

/* Enumerates every E8 point with squared norm <= max_norm (max_norm <= 12),
 * sorts them by (squared norm, x0, ..., x7) and writes the first
 * min(total, max_entries) as doubles into cb[entry][8].
 * Returns the total number of points found (117,361 for max_norm 12). */
int64_t glq_oracle_e8_points(int max_norm, double *cb, int64_t max_entries) {
    if (max_norm < 0 || max_norm > 12) return -1;
    int64_t cap = 200000, count = 0;
    e8_point *pts = (e8_point *)malloc(sizeof(e8_point) * cap);
    if (!pts) return -1;
    for (int parity = 0; parity < 2; parity++) {
        /* integer points: y_i in {-6,-4,...,6}; half-integer: {-5,...,5} */
        int lo = parity ? -5 : -6;
        int nvals = parity ? 6 : 7;
        int digits[8] = {0};
        for (;;) {
            int y[8], s = 0, q = 0;
            for (int i = 0; i < 8; i++) {
                y[i] = lo + 2 * digits[i];
                s += y[i];
                q += y[i] * y[i];
            }
            /* sum(x) even  <=>  sum(y) divisible by 4 */
            if (q <= 4 * max_norm && ((s % 4) + 4) % 4 == 0) {
                if (count == cap) {
                    free(pts);
                    return -1;
                }
                pts[count].norm4 = q;
                memcpy(pts[count].y, y, sizeof y);
                count++;
            }
            int i = 0;
            while (i < 8 && ++digits[i] == nvals) digits[i++] = 0;
            if (i == 8) break;
        }
    }
    qsort(pts, (size_t)count, sizeof(e8_point), e8_point_cmp);
    int64_t nout = count < max_entries ? count : max_entries;
    for (int64_t e = 0; e < nout; e++)
        for (int i = 0; i < 8; i++) cb[e * 8 + i] = 0.5 * pts[e].y[i];
    free(pts);
    return count;
}

/* ------------------------------------------------------------------ */
/* Normalised Walsh-Hadamard, block-diagonal over the binary             */
/* decomposition of the size  [glq 0.5.1, "How it works" 2; "Bit widths"] */
/* ------------------------------------------------------------------ */

/* Writes the block sizes of n (descending powers of two) into sizes and
 * returns how many there are; -1 if n <= 0 or more than max_blocks. */
int glq_oracle_hadamard_blocks(int64_t n, int64_t *sizes, int max_blocks) {
    if (n <= 0) return -1;
    int nb = 0;
    for (int bit = 62; bit >= 0; bit--) {
        if (n & ((int64_t)1 << bit)) {
            if (nb == max_blocks) return -1;
            sizes[nb++] = (int64_t)1 << bit;
        }
    }
    return nb;
}

static int popcount64(uint64_t v) {
    int c = 0;
    while (v) {
        v &= v - 1;
        c++;
    }
    return c;
}

/* One entry of the unnormalised Sylvester Hadamard matrix of order 2^q. */
static double sylvester_entry(int64_t i, int64_t j) {
    return (popcount64((uint64_t)(i & j)) & 1) ? -1.0 : 1.0;
}

/* Dense n x n block-diagonal normalised Hadamard matrix, row-major. */
void glq_oracle_hadamard_matrix(int64_t n, double *H) {
    int64_t sizes[64];
    int nb = glq_oracle_hadamard_blocks(n, sizes, 64);
    memset(H, 0, sizeof(double) * (size_t)(n * n));
    int64_t off = 0;
    for (int b = 0; b < nb; b++) {
        int64_t k = sizes[b];
        double s = 1.0 / sqrt((double)k);
        for (int64_t i = 0; i < k; i++)
            for (int64_t j = 0; j < k; j++)
                H[(off + i) * n + (off + j)] = s * sylvester_entry(i, j);
        off += k;
    }
}

/* out = H_k v for one Sylvester block of order k, unnormalised, dense. */
static void hadamard_block_dense(int64_t k, const double *v, double *out) {
    for (int64_t i = 0; i < k; i++) {
        double acc = 0.0;
        for (int64_t j = 0; j < k; j++) acc += sylvester_entry(i, j) * v[j];
        out[i] = acc;
    }
}

/* out = H_k v, unnormalised, for k = a*b (a, b powers of two).  Since
 * popcount((i1 b + i0) & (j1 b + j0)) = popcount(i1 & j1) + popcount(i0 & j0),
 * H_k = H_a (x) H_b, so with V[j1][j0] = v[j1 b + j0]:  out = H_a V H_b^T. */
static void hadamard_block_kron(int64_t a, int64_t b, const double *v, double *out) {
    double *t = (double *)malloc(sizeof(double) * (size_t)(a * b));
    for (int64_t j1 = 0; j1 < a; j1++) hadamard_block_dense(b, v + j1 * b, t + j1 * b);
    for (int64_t i1 = 0; i1 < a; i1++)
        for (int64_t i0 = 0; i0 < b; i0++) {
            double acc = 0.0;
            for (int64_t j1 = 0; j1 < a; j1++) acc += sylvester_entry(i1, j1) * t[j1 * b + i0];
            out[i1 * b + i0] = acc;
        }
    free(t);
}

/* Largest block applied as one dense k x k product; larger blocks use the
 * Kronecker split above with two dense factors. */
#define DENSE_LIMIT 4096

/* out = H_n v with H_n the normalised block-diagonal Hadamard of order n.
 * force_dense != 0 applies every block densely whatever its size. */
void glq_oracle_hadamard_apply(int64_t n, const double *v, double *out, int force_dense) {
    int64_t sizes[64];
    int nb = glq_oracle_hadamard_blocks(n, sizes, 64);
    int64_t off = 0;
    for (int b = 0; b < nb; b++) {
        int64_t k = sizes[b];
        if (k <= DENSE_LIMIT || force_dense) {
            hadamard_block_dense(k, v + off, out + off);
        } else {
            int q = 0;
            while (((int64_t)1 << q) < k) q++;
            int64_t a = (int64_t)1 << (q / 2);
            hadamard_block_kron(a, k / a, v + off, out + off);
        }
        double s = 1.0 / sqrt((double)k);
        for (int64_t i = 0; i < k; i++) out[off + i] *= s;
        off += k;
    }
}

/* ------------------------------------------------------------------ */
/* Codeword reconstruction  [glq 0.5.1, "How it works" 1; "Bit widths";  */
/* "Inference kernels" (Qidxs2, codebook2, inv_resid_scale)]            */
/* ------------------------------------------------------------------ */

/* Residual stages of a bit width  [glq 0.5.1, "Bit widths"]: after the
 * 16-bit primary index, (bpw - 2) / 2 stages of 16-bit E8 indices and, for
 * an odd bpw, one last stage of 8-bit indices into a 256-entry table
 * (3 = 16+8, 4 = 16+16, 5 = 16+16+8, ..., 8 = 16+16+16+16).  Writes the
 * index width of each residual stage into bits[] and returns their number,
 * or -1 for a bpw outside 2..8. */
int glq_oracle_stage_bits(int bpw, int *bits) {
    if (bpw < 2 || bpw > 8) return -1;
    int k = 0;
    for (int i = 0; i < (bpw - 2) / 2; i++) bits[k++] = 16;
    if (bpw % 2) bits[k++] = 8;
    return k;
}

/* Decodes rows [r0, r1) of W^ into w[(r - r0) * n + j] (fp32 values held
 * in double).  idx_res[s] is residual stage s ([m][n/8], uint16 into cb16
 * for a 16-bit stage, uint8 into cb8[256][8] for the 8-bit one) and rs[s]
 * its scale.  Reconstruction, stage by stage in that order:
 *   c = cb1[idx1][j];  c = fmaf(rs[s], cb_s[idx_s][j], c)  (one rounding each);
 *   w^ = fp32(ws * c)  (one rounding).
 * Returns 0, or -1 on bad arguments. */
int glq_oracle_decode_stages(int64_t m, int64_t n, int bpw, const uint16_t *idx1,
                             const void *const *idx_res, const double *cb1, const double *cb16,
                             const double *cb8, float ws, const float *rs, int64_t r0, int64_t r1,
                             double *w) {
    int bits[4];
    int ns = glq_oracle_stage_bits(bpw, bits);
    if (ns < 0 || n % 8 != 0 || r0 < 0 || r1 > m) return -1;
    for (int s = 0; s < ns; s++)
        if (!idx_res || !idx_res[s] || (bits[s] == 16 && !cb16) || (bits[s] == 8 && !cb8)) return -1;
    int64_t G = n / 8;
    for (int64_t r = r0; r < r1; r++) {
        for (int64_t g = 0; g < G; g++) {
            const double *c1 = cb1 + (int64_t)idx1[r * G + g] * 8;
            for (int j = 0; j < 8; j++) {
                float c = (float)c1[j]; /* exact: codewords are multiples of 1/2 */
                for (int s = 0; s < ns; s++) {
                    const double *cs = bits[s] == 16
                        ? cb16 + (int64_t)((const uint16_t *)idx_res[s])[r * G + g] * 8
                        : cb8 + (int64_t)((const uint8_t *)idx_res[s])[r * G + g] * 8;
                    c = fmaf(rs[s], (float)cs[j], c);
                }
                /* a binary32 x binary32 product is exact in binary64 */
                w[(r - r0) * n + g * 8 + j] = (double)(float)((double)ws * (double)c);
            }
        }
    }
    return 0;
}

/* The two-stage form of the pages' matmul arguments (Qidxs2, codebook2,
 * inv_resid_scale): bpw 2: no residual; bpw 3: idx2 is uint8 into
 * cb2[256][8]; bpw 4: idx2 is uint16 into cb2[65536][8].  Returns 0, or -1
 * on a bad bpw. */
int glq_oracle_decode_rows(int64_t m, int64_t n, int bpw, const uint16_t *idx1,
                           const void *idx2, const double *cb1, const double *cb2,
                           float ws, float rs, int64_t r0, int64_t r1, double *w) {
    if (bpw < 2 || bpw > 4) return -1;
    const void *res[1] = {idx2};
    return glq_oracle_decode_stages(m, n, bpw, idx1, res, cb1, bpw == 4 ? cb2 : 0, bpw == 3 ? cb2 : 0, ws,
                                    &rs, r0, r1, w);
}

/* ------------------------------------------------------------------ */
/* The layer:  y = S_out . H_m . W^ . H_n . (S_in . x)                  */
/* ------------------------------------------------------------------ */

/* The middle product z = W^ xr for rows [r0, r1): W^ is decoded one row at
 * a time (explicitly) and multiplied by a naive dot product. */
typedef struct {
    int64_t m, n, B, r0, r1;
    int bpw;
    const uint16_t *idx1;
    const void *const *idx_res;
    const double *cb1, *cb16, *cb8;
    float ws;
    const float *rs;
    const double *xr;
    double *z;
    int rc;
} rows_job;

static void *rows_product(void *arg) {
    rows_job *j = (rows_job *)arg;
    double *w = (double *)malloc(sizeof(double) * (size_t)j->n);
    if (!w) {
        j->rc = -1;
        return 0;
    }
    for (int64_t r = j->r0; r < j->r1; r++) {
        if (glq_oracle_decode_stages(j->m, j->n, j->bpw, j->idx1, j->idx_res, j->cb1, j->cb16, j->cb8, j->ws,
                                     j->rs, r, r + 1, w) != 0) {
            free(w);
            j->rc = -1;
            return 0;
        }
        for (int64_t b = 0; b < j->B; b++) {
            double acc = 0.0;
            const double *xb = j->xr + b * j->n;
            for (int64_t k = 0; k < j->n; k++) acc += w[k] * xb[k];
            j->z[b * j->m + r] = acc;
        }
    }
    free(w);
    j->rc = 0;
    return 0;
}

/* x[B][n] as fp16 (x_is_bf16 == 0) or bf16 bits; y[B][m] in double.
 * W^ is decoded one row at a time (explicitly) and multiplied by a naive
 * dot product.  The rows of the middle product are dealt out in contiguous
 * ranges to `nthreads` POSIX threads (each output element is computed by
 * the same loop whatever the thread count, so the result is identical).
 * Returns 0 or -1 on bad arguments / allocation failure. */
int glq_oracle_linear_stages_mt(int64_t m, int64_t n, int bpw, const uint16_t *idx1,
                                const void *const *idx_res, const double *cb1, const double *cb16,
                                const double *cb8, float ws, const float *rs, const int8_t *s_in,
                                const int8_t *s_out, const uint16_t *x, int x_is_bf16, int64_t B, double *y,
                                int nthreads) {
    if (m <= 0 || n <= 0 || n % 8 != 0 || B < 0) return -1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nthreads > m) nthreads = (int)m;
    double *xs = (double *)malloc(sizeof(double) * (size_t)n);
    double *xr = (double *)malloc(sizeof(double) * (size_t)(B * n + 1));
    double *z = (double *)malloc(sizeof(double) * (size_t)(B * m + 1));
    double *zb = (double *)malloc(sizeof(double) * (size_t)m);
    double *hb = (double *)malloc(sizeof(double) * (size_t)m);
    rows_job *jobs = (rows_job *)malloc(sizeof(rows_job) * (size_t)nthreads);
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!xs || !xr || !z || !zb || !hb || !jobs || !tid) {
        free(xs); free(xr); free(z); free(zb); free(hb); free(jobs); free(tid);
        return -1;
    }
    /* input RHT: sign, then H_n */
    for (int64_t b = 0; b < B; b++) {
        for (int64_t j = 0; j < n; j++) {
            uint16_t bits = x[b * n + j];
            double v = x_is_bf16 ? glq_oracle_bf16_to_double(bits) : glq_oracle_f16_to_double(bits);
            xs[j] = (double)s_in[j] * v;
        }
        glq_oracle_hadamard_apply(n, xs, xr + b * n, 0);
    }
    /* z = W^ xr, one decoded row at a time, rows split over the threads */
    int rc = 0, started = 0;
    for (int t = 0; t < nthreads; t++) {
        rows_job *j = &jobs[t];
        j->m = m; j->n = n; j->B = B; j->bpw = bpw;
        j->r0 = m * t / nthreads;
        j->r1 = m * (t + 1) / nthreads;
        j->idx1 = idx1; j->idx_res = idx_res; j->cb1 = cb1; j->cb16 = cb16; j->cb8 = cb8;
        j->ws = ws; j->rs = rs; j->xr = xr; j->z = z; j->rc = -1;
    }
    for (int t = 1; t < nthreads; t++) {
        if (pthread_create(&tid[t], 0, rows_product, &jobs[t]) != 0) break;
        started = t;
    }
    rows_product(&jobs[0]);
    for (int t = 1; t <= started; t++) pthread_join(tid[t], 0);
    for (int t = started + 1; t < nthreads; t++) rows_product(&jobs[t]); /* threads that did not start */
    for (int t = 0; t < nthreads; t++) rc |= jobs[t].rc;
    /* output RHT: H_m, then sign */
    for (int64_t b = 0; b < B && rc == 0; b++) {
        memcpy(zb, z + b * m, sizeof(double) * (size_t)m);
        glq_oracle_hadamard_apply(m, zb, hb, 0);
        for (int64_t r = 0; r < m; r++) y[b * m + r] = (double)s_out[r] * hb[r];
    }
    free(xs); free(xr); free(z); free(zb); free(hb); free(jobs); free(tid);
    return rc;
}

/* The two-stage form (bpw 2..4, see glq_oracle_decode_rows). */
int glq_oracle_linear_mt(int64_t m, int64_t n, int bpw, const uint16_t *idx1, const void *idx2,
                         const double *cb1, const double *cb2, float ws, float rs,
                         const int8_t *s_in, const int8_t *s_out, const uint16_t *x, int x_is_bf16,
                         int64_t B, double *y, int nthreads) {
    if (bpw < 2 || bpw > 4) return -1;
    const void *res[1] = {idx2};
    return glq_oracle_linear_stages_mt(m, n, bpw, idx1, res, cb1, bpw == 4 ? cb2 : 0, bpw == 3 ? cb2 : 0, ws, &rs,
                                       s_in, s_out, x, x_is_bf16, B, y, nthreads);
}

/* The single-threaded two-stage form. */
int glq_oracle_linear(int64_t m, int64_t n, int bpw, const uint16_t *idx1, const void *idx2,
                      const double *cb1, const double *cb2, float ws, float rs,
                      const int8_t *s_in, const int8_t *s_out, const uint16_t *x, int x_is_bf16,
                      int64_t B, double *y) {
    return glq_oracle_linear_mt(m, n, bpw, idx1, idx2, cb1, cb2, ws, rs, s_in, s_out, x, x_is_bf16, B, y, 1);
}
