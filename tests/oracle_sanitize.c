/* Drives every routine of oracle/lq_oracle.c on small inputs, with padded K,
 * ragged sizes and several threads, so that a build with AddressSanitizer and
 * UndefinedBehaviorSanitizer can check the oracle's memory accesses. Test
 * infrastructure: tests/test_oracle_sanitizers.py compiles and runs it. It also
 * checks a few results that must hold exactly (pack round trip, search never
 * below brute force), returning nonzero on a mismatch. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

int lqo_lifted_dim(int in, int d, int D);
void lqo_pack_signs(const int8_t* signs, int64_t out, int64_t K, uint32_t* packed);
void lqo_unpack_signs(const uint32_t* packed, int64_t out, int64_t K, int8_t* signs);
void lqo_whiten(const double* a, int64_t batch, int64_t in, const double* tinv, int64_t tblk, double* ap);
void lqo_whiten_kron(const double* a, int64_t batch, int64_t in, const double* r1, const double* q1, int64_t n1,
                     const double* q2, int64_t n2, const double* r2, int64_t d, double* ap);
void lqo_lift(const double* ap, int64_t batch, int64_t in, const double* M, int d, int D, int64_t K, double* u);
void lqo_contract(const uint32_t* packed, const double* s, int64_t out, int64_t K, const double* u, int64_t batch,
                  double* o, int nthreads);
void lqo_contract_rows(const uint32_t* packed, const double* s, int64_t out, int64_t K, const double* u,
                       int64_t batch, const int64_t* rows, int64_t nrows, double* o);
void lqo_dense_route(const uint32_t* packed, const double* s, int64_t out, int64_t K, const double* M, int d, int D,
                     const double* ap, int64_t batch, int64_t in, double* o);
int lqo_forward(const uint32_t* packed, const double* s, int64_t out, int64_t K, const double* a, int64_t batch,
                int64_t in, const double* tinv, int64_t tblk, const double* M, int d, int D, double* u_out, double* o,
                int nthreads);
void lqo_codebook_moments(const double* M, int d, int D, double* mean, double* second);
double lqo_block_identity_maxerr(const double* M, int d, int D, const double* ap_blk);
void lqo_encode_blocks(const double* M, int d, int D, const double* w, int64_t nblocks, int brute, uint64_t* y,
                       double* err, int nthreads);

static uint64_t state = 0x9E3779B97F4A7C15ull;
static double urand(void) { /* xorshift64*, uniform in [-1, 1) */
    state ^= state >> 12;
    state ^= state << 25;
    state ^= state >> 27;
    return (double)((state * 2685821657736338717ull) >> 11) / 9007199254740992.0 * 2.0 - 1.0;
}
static double* vec(size_t n) {
    double* v = (double*)malloc(sizeof(double) * n);
    for (size_t i = 0; i < n; ++i) v[i] = urand();
    return v;
}

int main(void) {
    /* a layer with in = 30, d = 5, D = 9: K = lifted_dim = 64 (10 padded lifted coordinates) */
    const int in = 30, d = 5, D = 9, batch = 3, out = 7, tblk = 6;
    const int K = lqo_lifted_dim(in, d, D);
    if (K != 64) return 10;
    int8_t* signs = (int8_t*)malloc((size_t)out * K);
    int8_t* back = (int8_t*)malloc((size_t)out * K);
    for (int i = 0; i < out * K; ++i) signs[i] = urand() >= 0 ? 1 : -1;
    uint32_t* packed = (uint32_t*)calloc((size_t)out * (K / 32), 4);
    lqo_pack_signs(signs, out, K, packed);
    lqo_unpack_signs(packed, out, K, back);
    if (memcmp(signs, back, (size_t)out * K) != 0) return 11;

    double* a = vec((size_t)batch * in);
    double* tinv = vec((size_t)(in / tblk) * tblk * tblk);
    double* M = vec((size_t)d * D);
    double* s = vec(out);
    double* ap = vec((size_t)batch * in);
    double* u = vec((size_t)batch * K);
    double* o = vec((size_t)batch * out);
    lqo_whiten(a, batch, in, tinv, tblk, ap);
    lqo_whiten(a, batch, in, NULL, 0, ap);
    double* r1 = vec(in);
    double* q1 = vec(25);
    double* q2 = vec(36);
    double* r2 = vec(in / d);
    lqo_whiten_kron(a, batch, in, r1, q1, 5, q2, 6, r2, d, ap);
    lqo_whiten_kron(a, batch, in, NULL, q1, 5, q2, 6, NULL, d, ap);
    lqo_lift(ap, batch, in, M, d, D, K, u);
    lqo_contract(packed, s, out, K, u, batch, o, 1);
    lqo_contract(packed, s, out, K, u, batch, o, 3);
    int64_t rows[3] = {0, 3, 6};
    double o3[9];
    lqo_contract_rows(packed, s, out, K, u, batch, rows, 3, o3);
    lqo_dense_route(packed, s, out, K, M, d, D, ap, batch, in, o);
    if (lqo_forward(packed, s, out, K, a, batch, in, tinv, tblk, M, d, D, u, o, 2) != 0) return 12;
    double mean[5], second[25];
    lqo_codebook_moments(M, d, D, mean, second);
    (void)lqo_block_identity_maxerr(M, d, D, ap);

    /* encoder: brute force and search, several threads, a square case (D = d) */
    const int nb = 9;
    double* w = vec((size_t)nb * d);
    uint64_t yb[9], ys[9];
    double eb[9], es[9];
    lqo_encode_blocks(M, d, D, w, nb, 1, yb, eb, 2);
    lqo_encode_blocks(M, d, D, w, nb, 0, ys, es, 3);
    for (int i = 0; i < nb; ++i)
        if (es[i] < eb[i] - 1e-12) return 13;
    double* Msq = vec((size_t)d * d);
    for (int i = 0; i < d; ++i) Msq[i * d + i] += 3.0;
    lqo_encode_blocks(Msq, d, d, w, nb, 0, ys, es, 1);

    free(signs); free(back); free(packed); free(a); free(tinv); free(M); free(s); free(ap); free(u); free(o);
    free(r1); free(q1); free(q2); free(r2); free(w); free(Msq);
    puts("oracle sanitize ok");
    return 0;
}
