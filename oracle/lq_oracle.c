/*
 * Float64 CPU oracle for the LiftQuant lift-then-project linear layer.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or
 * call this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it. It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes (LiftQuant: Continuous Bit-Width LLM via Dimensional
 * Lifting and Projection, ICML 2026 paper note, "Key designs" 1 and 4):
 *
 *   o = diag(s) . W_q . (blockdiag(M^T) . T^{-1} . a)
 *
 *   - a weight block w in R^d is represented as w ~= M y with y in {+-1}^D,
 *     M in R^{d x D}, so that w_i = sum_j M_ij y_j  (design 1);
 *   - storage is D sign bits per d weights, bit-width D/d  (design 1);
 *   - the whitening T acts on the activation side; in its Kronecker form
 *     T = diag(s1)(P1 kron P2)diag(s2), s2 constant per block  (design 3);
 *   - encoding a block means finding the nearest lifted codeword M y, which a
 *     pseudo-inverse start plus a 2^{D-d} search over an auxiliary vector
 *     approximates  (design 2);
 *   - at inference the decode matrix T* = M T^{-1} is applied to the
 *     activations once, followed by a 1-bit x float matmul with W_q and the
 *     per-row scale diag(s)  (design 4).
 *
 * Readings taken where the page is silent (each also listed in the design
 * notes): M T^{-1} a is read as M^T applied to each consecutive d-block of
 * T^{-1} a, the lifted coordinates of block b occupying [b*D, (b+1)*D) of a
 * lifted axis of length K = (in/d)*D rounded up to a multiple of 32, padded
 * with zeros; T^{-1} is given (block diagonal, tblk x tblk blocks, or the
 * identity); signs are stored 32 per uint32, least significant bit first
 * along the lifted axis, bit 1 meaning +1.
 *
 * Every routine is a direct loop over its definition, in float64, with no
 * blocking, fusion or reordering.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* K = (in/d)*D rounded up to a multiple of 32; -1 if d does not divide in.
 * Bit-width D/d: D sign bits stored per d weights (design 1). */
int lqo_lifted_dim(int in, int d, int D) {
    if (in <= 0 || d <= 0 || D <= 0 || in % d != 0) return -1;
    long long k = (long long)(in / d) * D;
    k = (k + 31) / 32 * 32;
    if (k > 0x7fffffffLL) return -1;
    return (int)k;
}

/* sigma[r][k] = +1 if bit (k mod 32) of word packed[r][k/32] is set, else -1. */
static inline int lqo_sign(const uint32_t* packed, int64_t K, int64_t r, int64_t k) {
    uint32_t w = packed[r * (K / 32) + k / 32];
    return ((w >> (k % 32)) & 1u) ? +1 : -1;
}

/* Pack +-1 signs [out][K] into words [out][K/32] (1-bit W_q storage, design 4). */
void lqo_pack_signs(const int8_t* signs, int64_t out, int64_t K, uint32_t* packed) {
    for (int64_t r = 0; r < out; ++r)
        for (int64_t q = 0; q < K / 32; ++q) {
            uint32_t w = 0;
            for (int b = 0; b < 32; ++b)
                if (signs[r * K + q * 32 + b] > 0) w |= (1u << b);
            packed[r * (K / 32) + q] = w;
        }
}

void lqo_unpack_signs(const uint32_t* packed, int64_t out, int64_t K, int8_t* signs) {
    for (int64_t r = 0; r < out; ++r)
        for (int64_t k = 0; k < K; ++k)
            signs[r * K + k] = (int8_t)lqo_sign(packed, K, r, k);
}

/* a' = T^{-1} a, block by block: a'[c][blk*tblk+i] = sum_j Tinv[blk][i][j] a[c][blk*tblk+j].
 * tinv == NULL means T = identity (design 3: T acts on the activations). */
void lqo_whiten(const double* a, int64_t batch, int64_t in, const double* tinv, int64_t tblk,
                double* ap) {
    for (int64_t c = 0; c < batch; ++c) {
        if (tinv == NULL) {
            for (int64_t i = 0; i < in; ++i) ap[c * in + i] = a[c * in + i];
            continue;
        }
        for (int64_t blk = 0; blk < in / tblk; ++blk)
            for (int64_t i = 0; i < tblk; ++i) {
                double acc = 0.0;
                for (int64_t j = 0; j < tblk; ++j)
                    acc += tinv[(blk * tblk + i) * tblk + j] * a[c * in + blk * tblk + j];
                ap[c * in + blk * tblk + i] = acc;
            }
    }
}

/* Kronecker-factored whitening (design 3: T = diag(s1) (P1 kron P2) diag(s2), with s2
 * constant over each d-block), applied through the factors of its inverse
 *   T^{-1} = diag(r2) (Q1 kron Q2) diag(r1),  r1 = 1/s1, Q1 = P1^{-1}, Q2 = P2^{-1}, r2 = 1/s2.
 * in = n1 * n2. Kronecker entry (i, j) with i = i1*n2 + i2, j = j1*n2 + j2 is
 * Q1[i1][j1] * Q2[i2][j2], so
 *   a'[c][i] = r2[i / d] * sum_j Q1[i/n2][j/n2] * Q2[i%n2][j%n2] * r1[j] * a[c][j].
 * r1 == NULL or r2 == NULL means all ones. O(in^2) per token: the definition, not a
 * fast transform. */
void lqo_whiten_kron(const double* a, int64_t batch, int64_t in, const double* r1, const double* q1,
                     int64_t n1, const double* q2, int64_t n2, const double* r2, int64_t d, double* ap) {
    for (int64_t c = 0; c < batch; ++c)
        for (int64_t i = 0; i < in; ++i) {
            const int64_t i1 = i / n2, i2 = i % n2;
            double acc = 0.0;
            for (int64_t j = 0; j < in; ++j) {
                const int64_t j1 = j / n2, j2 = j % n2;
                const double x = (r1 ? r1[j] : 1.0) * a[c * in + j];
                acc += q1[i1 * n1 + j1] * q2[i2 * n2 + j2] * x;
            }
            ap[c * in + i] = (r2 ? r2[i / d] : 1.0) * acc;
        }
}

/* Lift: u[c][blk*D+j] = sum_{i<d} M[i][j] a'[c][blk*d+i]; entries past (in/d)*D are 0.
 * This is M^T applied per d-block, i.e. the small matmul T* a of design 4, read
 * through w_i = sum_j M_ij y_j of design 1. */
void lqo_lift(const double* ap, int64_t batch, int64_t in, const double* M, int d, int D,
              int64_t K, double* u) {
    for (int64_t c = 0; c < batch; ++c) {
        for (int64_t k = 0; k < K; ++k) u[c * K + k] = 0.0;
        for (int64_t blk = 0; blk < in / d; ++blk)
            for (int j = 0; j < D; ++j) {
                double acc = 0.0;
                for (int i = 0; i < d; ++i) acc += M[i * D + j] * ap[c * in + blk * d + i];
                u[c * K + blk * D + j] = acc;
            }
    }
}

/* o[c][r] = s[r] * sum_k sigma[r][k] u[c][k]  (1-bit x float matmul and diag(s), design 4). */
typedef struct {
    const uint32_t* packed; const double* s; int64_t out, K; const double* u; int64_t batch;
    double* o; int64_t r0, r1;
} lqo_contract_job;

static void* lqo_contract_worker(void* p) {
    lqo_contract_job* j = (lqo_contract_job*)p;
    for (int64_t r = j->r0; r < j->r1; ++r)
        for (int64_t c = 0; c < j->batch; ++c) {
            double acc = 0.0;
            for (int64_t k = 0; k < j->K; ++k)
                acc += (double)lqo_sign(j->packed, j->K, r, k) * j->u[c * j->K + k];
            j->o[c * j->out + r] = j->s[r] * acc;
        }
    return NULL;
}

/* nthreads <= 1 runs on the calling thread; otherwise rows are split evenly. */
void lqo_contract(const uint32_t* packed, const double* s, int64_t out, int64_t K,
                  const double* u, int64_t batch, double* o, int nthreads) {
    if (nthreads <= 1) {
        lqo_contract_job j = {packed, s, out, K, u, batch, o, 0, out};
        lqo_contract_worker(&j);
        return;
    }
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    lqo_contract_job* jobs = (lqo_contract_job*)malloc(sizeof(lqo_contract_job) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) {
        int64_t r0 = out * t / nthreads, r1 = out * (t + 1) / nthreads;
        lqo_contract_job j = {packed, s, out, K, u, batch, o, r0, r1};
        jobs[t] = j;
        pthread_create(&th[t], NULL, lqo_contract_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
    free(jobs);
}

/* Same contraction on a chosen list of rows: o[c][n] for row rows[n]. Used to
 * check sampled outputs of full-size layers. */
void lqo_contract_rows(const uint32_t* packed, const double* s, int64_t out, int64_t K,
                       const double* u, int64_t batch, const int64_t* rows, int64_t nrows,
                       double* o) {
    (void)out;
    for (int64_t n = 0; n < nrows; ++n) {
        int64_t r = rows[n];
        for (int64_t c = 0; c < batch; ++c) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += (double)lqo_sign(packed, K, r, k) * u[c * K + k];
            o[c * nrows + n] = s[r] * acc;
        }
    }
}

/* Second route through the dense reconstruction: W'[r][blk*d+i] = sum_j M[i][j]
 * sigma[r][blk*D+j] (w = M y, design 1), then o2[c][r] = s[r] sum_i W'[r][i] a'[c][i].
 * Equal to the lifted route by w.a' = y^T (M^T a'). */
void lqo_dense_route(const uint32_t* packed, const double* s, int64_t out, int64_t K,
                     const double* M, int d, int D, const double* ap, int64_t batch, int64_t in,
                     double* o) {
    double* wrow = (double*)malloc(sizeof(double) * (size_t)in);
    for (int64_t r = 0; r < out; ++r) {
        for (int64_t blk = 0; blk < in / d; ++blk)
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int j = 0; j < D; ++j) acc += M[i * D + j] * (double)lqo_sign(packed, K, r, blk * D + j);
                wrow[blk * d + i] = acc;
            }
        for (int64_t c = 0; c < batch; ++c) {
            double acc = 0.0;
            for (int64_t i = 0; i < in; ++i) acc += wrow[i] * ap[c * in + i];
            o[c * out + r] = s[r] * acc;
        }
    }
    free(wrow);
}

/* Whole layer: whiten, lift, contract. Scratch is allocated here (oracle only). */
int lqo_forward(const uint32_t* packed, const double* s, int64_t out, int64_t K,
                const double* a, int64_t batch, int64_t in, const double* tinv, int64_t tblk,
                const double* M, int d, int D, double* u_out, double* o, int nthreads) {
    double* ap = (double*)malloc(sizeof(double) * (size_t)(batch * in));
    double* u = u_out ? u_out : (double*)malloc(sizeof(double) * (size_t)(batch * K));
    if (!ap || !u) return -1;
    lqo_whiten(a, batch, in, tinv, tblk, ap);
    lqo_lift(ap, batch, in, M, d, D, K, u);
    lqo_contract(packed, s, out, K, u, batch, o, nthreads);
    free(ap);
    if (!u_out) free(u);
    return 0;
}

/* Codebook of one block: all 2^D sign patterns y, codeword My. Returns the exact
 * first moment mean[i] = 2^-D sum_y (My)_i and second moment
 * second[i][i'] = 2^-D sum_y (My)_i (My)_{i'}. By symmetry of y these equal 0 and
 * (M M^T)[i][i'] (the CLT-codebook moments of design 1). */
void lqo_codebook_moments(const double* M, int d, int D, double* mean, double* second) {
    for (int i = 0; i < d; ++i) {
        mean[i] = 0.0;
        for (int i2 = 0; i2 < d; ++i2) second[i * d + i2] = 0.0;
    }
    double* w = (double*)malloc(sizeof(double) * (size_t)d);
    uint64_t n = 1ull << D;
    for (uint64_t y = 0; y < n; ++y) {
        for (int i = 0; i < d; ++i) {
            double acc = 0.0;
            for (int j = 0; j < D; ++j) acc += M[i * D + j] * (((y >> j) & 1u) ? 1.0 : -1.0);
            w[i] = acc;
        }
        for (int i = 0; i < d; ++i) {
            mean[i] += w[i];
            for (int i2 = 0; i2 < d; ++i2) second[i * d + i2] += w[i] * w[i2];
        }
    }
    for (int i = 0; i < d; ++i) {
        mean[i] /= (double)n;
        for (int i2 = 0; i2 < d; ++i2) second[i * d + i2] /= (double)n;
    }
    free(w);
}

/* Largest |y.(M^T a') - (M y).a'| over all 2^D patterns of one block: the
 * identity w.a' = y^T (M^T a') behind the fused decode, checked by enumeration. */
double lqo_block_identity_maxerr(const double* M, int d, int D, const double* ap_blk) {
    double* mt = (double*)malloc(sizeof(double) * (size_t)D);
    for (int j = 0; j < D; ++j) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += M[i * D + j] * ap_blk[i];
        mt[j] = acc;
    }
    double worst = 0.0;
    uint64_t n = 1ull << D;
    for (uint64_t y = 0; y < n; ++y) {
        double lhs = 0.0, rhs = 0.0;
        for (int j = 0; j < D; ++j) lhs += (((y >> j) & 1u) ? 1.0 : -1.0) * mt[j];
        for (int i = 0; i < d; ++i) {
            double wi = 0.0;
            for (int j = 0; j < D; ++j) wi += M[i * D + j] * (((y >> j) & 1u) ? 1.0 : -1.0);
            rhs += wi * ap_blk[i];
        }
        double e = lhs - rhs;
        if (e < 0) e = -e;
        if (e > worst) worst = e;
    }
    free(mt);
    return worst;
}

/* ---------------------------------------------------------------- encoder
 * "Key designs" 2: quantising a block w of d weights means finding the nearest
 * point M y of the lifted codebook, y in {+-1}^D. Sign patterns are bit masks:
 * bit j set <=> y_j = +1. Errors are squared Euclidean distances ||w - M y||^2. */

static double lqo_code_err(const double* M, int d, int D, const double* w, uint64_t y) {
    double e = 0.0;
    for (int i = 0; i < d; ++i) {
        double acc = w[i];
        for (int j = 0; j < D; ++j) acc -= M[i * D + j] * (((y >> j) & 1u) ? 1.0 : -1.0);
        e += acc * acc;
    }
    return e;
}

/* The naive search: all 2^D patterns; the lowest pattern wins a tie. */
uint64_t lqo_encode_brute(const double* M, int d, int D, const double* w, double* err) {
    uint64_t best = 0;
    double best_e = lqo_code_err(M, d, D, w, 0);
    for (uint64_t y = 1; y < (1ull << D); ++y) {
        const double e = lqo_code_err(M, d, D, w, y);
        if (e < best_e) {
            best_e = e;
            best = y;
        }
    }
    *err = best_e;
    return best;
}

/* x = A^{-1} b for a small dense n x n A (row-major), by Gauss-Jordan elimination
 * with partial pivoting on copies. Returns 0 when A is singular. */
static int lqo_solve(const double* A_in, const double* b_in, int n, double* x) {
    double* A = (double*)malloc(sizeof(double) * (size_t)n * n);
    memcpy(A, A_in, sizeof(double) * (size_t)n * n);
    memcpy(x, b_in, sizeof(double) * (size_t)n);
    int ok = 1;
    for (int c = 0; c < n && ok; ++c) {
        int piv = c;
        for (int r = c + 1; r < n; ++r)
            if (fabs(A[r * n + c]) > fabs(A[piv * n + c])) piv = r;
        if (A[piv * n + c] == 0.0) {
            ok = 0;
            break;
        }
        if (piv != c) {
            for (int k = 0; k < n; ++k) {
                const double t = A[c * n + k];
                A[c * n + k] = A[piv * n + k];
                A[piv * n + k] = t;
            }
            const double t = x[c];
            x[c] = x[piv];
            x[piv] = t;
        }
        for (int r = 0; r < n; ++r) {
            if (r == c) continue;
            const double f = A[r * n + c] / A[c * n + c];
            if (f == 0.0) continue;
            for (int k = c; k < n; ++k) A[r * n + k] -= f * A[c * n + k];
            x[r] -= f * x[c];
        }
    }
    if (ok)
        for (int c = 0; c < n; ++c) x[c] /= A[c * n + c];
    free(A);
    return ok;
}

/* The search of "Key designs" 2 (a pseudo-inverse start, then an auxiliary
 * vector that cuts the search from 2^D to 2^{D-d} patterns), read as:
 *   candidate 0:      y = sign(M^+ w), M^+ w = M^T (M M^T)^{-1} w;
 *   candidate 1 + p:  for p in [0, 2^{D-d}), the auxiliary vector z is the first
 *                     D - d coordinates (z_a = +1 iff bit a of p is set) and the
 *                     last d coordinates solve M_B y_B = w - M_A z, rounded:
 *                     y_B = sign(M_B^{-1} (w - M_A z)).
 * sign(0) = +1. Returns the candidate of smallest error, the earliest on ties;
 * *err is its error. Returns UINT64_MAX with *err = -1 if M M^T or M_B is singular. */
uint64_t lqo_encode_search(const double* M, int d, int D, const double* w, double* err) {
    const int na = D - d;
    double* G = (double*)malloc(sizeof(double) * (size_t)d * d);
    double* t = (double*)malloc(sizeof(double) * (size_t)(d > D ? d : D));
    double* rhs = (double*)malloc(sizeof(double) * (size_t)d);
    uint64_t best = UINT64_MAX;
    double best_e = -1.0;
    /* candidate 0: the pseudo-inverse start */
    for (int i = 0; i < d; ++i)
        for (int k = 0; k < d; ++k) {
            double acc = 0.0;
            for (int j = 0; j < D; ++j) acc += M[i * D + j] * M[k * D + j];
            G[i * d + k] = acc;
        }
    if (!lqo_solve(G, w, d, t)) goto done;
    {
        uint64_t y0 = 0;
        for (int j = 0; j < D; ++j) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i) acc += M[i * D + j] * t[i];
            if (acc >= 0.0) y0 |= 1ull << j;
        }
        best = y0;
        best_e = lqo_code_err(M, d, D, w, y0);
    }
    /* candidates 1 + p: M_B holds the last d columns of M */
    for (int i = 0; i < d; ++i)
        for (int k = 0; k < d; ++k) G[i * d + k] = M[i * D + na + k];
    for (uint64_t p = 0; p < (1ull << na); ++p) {
        for (int i = 0; i < d; ++i) {
            double acc = w[i];
            for (int a = 0; a < na; ++a) acc -= M[i * D + a] * (((p >> a) & 1u) ? 1.0 : -1.0);
            rhs[i] = acc;
        }
        if (!lqo_solve(G, rhs, d, t)) {
            best = UINT64_MAX;
            best_e = -1.0;
            goto done;
        }
        uint64_t y = p;
        for (int k = 0; k < d; ++k)
            if (t[k] >= 0.0) y |= 1ull << (na + k);
        const double e = lqo_code_err(M, d, D, w, y);
        if (e < best_e) {
            best_e = e;
            best = y;
        }
    }
done:
    free(G);
    free(t);
    free(rhs);
    *err = best_e;
    return best;
}

/* Blocks [nblocks][d] of w -> patterns and errors; brute != 0 selects the naive search. */
typedef struct {
    const double* M; int d, D; const double* w; int64_t b0, b1; int brute; uint64_t* y; double* err;
} lqo_encode_job;

static void* lqo_encode_worker(void* p) {
    lqo_encode_job* j = (lqo_encode_job*)p;
    for (int64_t b = j->b0; b < j->b1; ++b)
        j->y[b] = j->brute ? lqo_encode_brute(j->M, j->d, j->D, j->w + b * j->d, j->err + b)
                           : lqo_encode_search(j->M, j->d, j->D, j->w + b * j->d, j->err + b);
    return NULL;
}

void lqo_encode_blocks(const double* M, int d, int D, const double* w, int64_t nblocks, int brute, uint64_t* y,
                       double* err, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    lqo_encode_job jobs[256];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].M = M;
        jobs[t].d = d;
        jobs[t].D = D;
        jobs[t].w = w;
        jobs[t].b0 = nblocks * t / nthreads;
        jobs[t].b1 = nblocks * (t + 1) / nthreads;
        jobs[t].brute = brute;
        jobs[t].y = y;
        jobs[t].err = err;
        pthread_create(&th[t], NULL, lqo_encode_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
}
