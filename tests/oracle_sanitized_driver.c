/*
 * Test driver for the fp64 oracle built with AddressSanitizer,
 * UndefinedBehaviorSanitizer and LeakSanitizer (tests/test_oracle_sanitized.py).
 *
 * TEST INFRASTRUCTURE ONLY.  It links oracle/kda_oracle.c, calls every entry
 * point of it on the case a directory holds, and writes the results back as
 * raw fp64 files, so that the test can compare them with the normal build of
 * the oracle.  Every buffer is allocated at exactly its size, so any read or
 * write past an end, any use after free and any leak is reported by the
 * sanitizers and ends the program with a non-zero status.
 *
 * Directory layout (written by the test):
 *   case.txt   N T_tot H dk dv B, then cu_seqlens[0..N], then the unit mask
 *              (N * H values, 0 or 1)
 *   q k g      [T_tot, H, dk]    v dO  [T_tot, H, dv]    beta [T_tot, H]
 *   h0 dhT     [N, H, dk, dv]
 *   dec_q dec_k dec_g [B, H, dk]  dec_v [B, H, dv]  dec_beta [B, H]
 *   dec_S      [B, H, dk, dv]
 * Outputs: o_sig hT_sig (K3 gate, h0), o_soft hT_soft (softplus gate, no h0),
 * hT_mask (K3 gate, masked units only, no o), bwd_* (with h0, dO, dhT),
 * bwd0_* (no h0, dO only), dec_o dec_S_new, and rc.txt with the return codes
 * of the calls, including those given a malformed cu_seqlens.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

int kda_oracle_forward_gate(const double *q, const double *k, const double *v,
                            const double *g, const double *beta, const double *h0,
                            const int64_t *cu_seqlens, int N, int64_t T_tot, int H,
                            int dk, int dv, const uint8_t *unit_mask, double *o,
                            double *hT, int gate);
int kda_oracle_forward(const double *q, const double *k, const double *v,
                       const double *g, const double *beta, const double *h0,
                       const int64_t *cu_seqlens, int N, int64_t T_tot, int H,
                       int dk, int dv, const uint8_t *unit_mask, double *o, double *hT);
int kda_oracle_decode(const double *q, const double *k, const double *v,
                      const double *g, const double *beta, double *S, int B, int H,
                      int dk, int dv, double *o);
int kda_oracle_backward(const double *q, const double *k, const double *v,
                        const double *g, const double *beta, const double *h0,
                        const int64_t *cu_seqlens, int N, int64_t T_tot, int H,
                        int dk, int dv, const double *dO, const double *dhT, double *dq,
                        double *dk_, double *dv_, double *dg, double *dbeta, double *dh0);

static const char *g_dir;

static void die(const char *what) {
    fprintf(stderr, "driver: %s\n", what);
    exit(2);
}

static double *alloc_n(size_t n) {
    /* malloc(0) may return NULL; the oracle never touches a zero-size array */
    double *p = (double *)malloc(n ? n * sizeof(double) : 1);
    if (!p) die("out of memory");
    return p;
}

static double *read_f64(const char *name, size_t n) {
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", g_dir, name);
    FILE *f = fopen(path, "rb");
    if (!f) die(name);
    double *p = alloc_n(n);
    if (n && fread(p, sizeof(double), n, f) != n) die(name);
    fclose(f);
    return p;
}

static void write_f64(const char *name, const double *p, size_t n) {
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", g_dir, name);
    FILE *f = fopen(path, "wb");
    if (!f) die(name);
    if (n && fwrite(p, sizeof(double), n, f) != n) die(name);
    fclose(f);
}

static double *filled(size_t n, double x) {
    double *p = alloc_n(n);
    for (size_t i = 0; i < n; ++i) p[i] = x;
    return p;
}

int main(int argc, char **argv) {
    if (argc != 2) die("usage: driver <case directory>");
    g_dir = argv[1];
    char path[4096];
    snprintf(path, sizeof path, "%s/case.txt", g_dir);
    FILE *f = fopen(path, "r");
    if (!f) die("case.txt");
    long long N_, T_, H_, dk_, dv_, B_;
    if (fscanf(f, "%lld %lld %lld %lld %lld %lld", &N_, &T_, &H_, &dk_, &dv_, &B_) != 6)
        die("case.txt header");
    const int N = (int)N_, H = (int)H_, dk = (int)dk_, dv = (int)dv_, B = (int)B_;
    const int64_t T = (int64_t)T_;
    int64_t *cu = (int64_t *)malloc(sizeof(int64_t) * (size_t)(N + 1));
    uint8_t *mask = (uint8_t *)malloc((size_t)N * H ? (size_t)N * H : 1);
    if (!cu || !mask) die("out of memory");
    for (int i = 0; i <= N; ++i) {
        long long x;
        if (fscanf(f, "%lld", &x) != 1) die("cu_seqlens");
        cu[i] = (int64_t)x;
    }
    for (long i = 0; i < (long)N * H; ++i) {
        int x;
        if (fscanf(f, "%d", &x) != 1) die("mask");
        mask[i] = (uint8_t)x;
    }
    fclose(f);

    const size_t nk = (size_t)T * H * dk, nv = (size_t)T * H * dv, nb = (size_t)T * H;
    const size_t ns = (size_t)N * H * dk * dv;
    double *q = read_f64("q", nk), *k = read_f64("k", nk), *g = read_f64("g", nk);
    double *v = read_f64("v", nv), *dO = read_f64("dO", nv), *beta = read_f64("beta", nb);
    double *h0 = read_f64("h0", ns), *dhT = read_f64("dhT", ns);
    int rc[9];

    /* prefill, K3 gate, with h0 */
    double *o = filled(nv, 0.0), *hT = filled(ns, 0.0);
    rc[0] = kda_oracle_forward(q, k, v, g, beta, h0, cu, N, T, H, dk, dv, NULL, o, hT);
    write_f64("o_sig", o, nv);
    write_f64("hT_sig", hT, ns);
    /* prefill, softplus gate, no h0 */
    rc[1] = kda_oracle_forward_gate(q, k, v, g, beta, NULL, cu, N, T, H, dk, dv, NULL, o, hT, 1);
    write_f64("o_soft", o, nv);
    write_f64("hT_soft", hT, ns);
    /* masked units, final states only */
    double *hTm = filled(ns, 0.0);
    rc[2] = kda_oracle_forward(q, k, v, g, beta, h0, cu, N, T, H, dk, dv, mask, NULL, hTm);
    write_f64("hT_mask", hTm, ns);

    /* backward, twice: with every input, then without h0 and dhT */
    double *dq = filled(nk, 0.0), *dkk = filled(nk, 0.0), *dg = filled(nk, 0.0);
    double *dvv = filled(nv, 0.0), *db = filled(nb, 0.0), *dh0 = filled(ns, 0.0);
    rc[3] = kda_oracle_backward(q, k, v, g, beta, h0, cu, N, T, H, dk, dv, dO, dhT, dq, dkk,
                                dvv, dg, db, dh0);
    write_f64("bwd_dq", dq, nk);
    write_f64("bwd_dk", dkk, nk);
    write_f64("bwd_dv", dvv, nv);
    write_f64("bwd_dg", dg, nk);
    write_f64("bwd_dbeta", db, nb);
    write_f64("bwd_dh0", dh0, ns);
    rc[4] = kda_oracle_backward(q, k, v, g, beta, NULL, cu, N, T, H, dk, dv, dO, NULL, dq, dkk,
                                dvv, dg, db, dh0);
    write_f64("bwd0_dq", dq, nk);
    write_f64("bwd0_dk", dkk, nk);
    write_f64("bwd0_dv", dvv, nv);
    write_f64("bwd0_dg", dg, nk);
    write_f64("bwd0_dbeta", db, nb);
    write_f64("bwd0_dh0", dh0, ns);

    /* decode */
    const size_t dkn = (size_t)B * H * dk, dvn = (size_t)B * H * dv;
    double *eq = read_f64("dec_q", dkn), *ek = read_f64("dec_k", dkn),
           *eg = read_f64("dec_g", dkn), *ev = read_f64("dec_v", dvn),
           *eb = read_f64("dec_beta", (size_t)B * H),
           *eS = read_f64("dec_S", (size_t)B * H * dk * dv);
    double *eo = filled(dvn, 0.0);
    rc[5] = kda_oracle_decode(eq, ek, ev, eg, eb, eS, B, H, dk, dv, eo);
    write_f64("dec_o", eo, dvn);
    write_f64("dec_S_new", eS, (size_t)B * H * dk * dv);

    /* malformed cu_seqlens: refused before any access */
    const int64_t keep_last = cu[N];
    cu[N] = T + 1;                                           /* cu[N] != T_tot */
    rc[6] = kda_oracle_forward(q, k, v, g, beta, h0, cu, N, T, H, dk, dv, NULL, o, hT);
    rc[7] = kda_oracle_backward(q, k, v, g, beta, h0, cu, N, T, H, dk, dv, dO, dhT, dq, dkk,
                                dvv, dg, db, dh0);
    cu[N] = keep_last;
    rc[8] = 0;
    if (N >= 2) {                                            /* a decreasing boundary */
        const int64_t keep = cu[1];
        cu[1] = cu[2] + 1;
        rc[8] = kda_oracle_forward(q, k, v, g, beta, h0, cu, N, T, H, dk, dv, NULL, o, hT);
        cu[1] = keep;
    }

    snprintf(path, sizeof path, "%s/rc.txt", g_dir);
    f = fopen(path, "w");
    if (!f) die("rc.txt");
    for (int i = 0; i < 9; ++i) fprintf(f, "%d\n", rc[i]);
    fclose(f);

    free(q); free(k); free(g); free(v); free(dO); free(beta); free(h0); free(dhT);
    free(o); free(hT); free(hTm);
    free(dq); free(dkk); free(dg); free(dvv); free(db); free(dh0);
    free(eq); free(ek); free(eg); free(ev); free(eb); free(eS); free(eo);
    free(cu); free(mask);
    return 0;
}
