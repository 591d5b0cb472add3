/*
 * Gated linear attention (GLA) oracle: plain fp64 CPU reference.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
 * load this file; it exists so that the tests, the smoke check and the CPU
 * baseline leg of the benchmark have an obviously correct answer to compare
 * the CUDA path against. It shares no code with the CUDA library.
 *
 * What it computes (per batch b and head h, row-major, contiguous):
 *   q, k, log_a : [B,H,L,K]     v, o : [B,H,L,V]     h0, hT, S : [B,H,K,V]
 *
 *   S_{-1} = h0 (zero when h0 == NULL)
 *   S_t    = diag(a_t) S_{t-1} + k_t^T v_t,    a_t = exp(log_a_t) in (0,1]^K
 *   o_t    = q_t S_t                            (read after the update)
 *   hT     = S_{L-1}
 *
 * Source: "Gated Linear Attention Transformers with Hardware-Efficient
 * Training" (atlas.scime.ai summary of arXiv 2312.06635), section
 * "Approach": the gate is G_t = alpha_t^T 1, i.e. a matrix whose rows are
 * constant along the value dimension, so G_t (.) S = diag(alpha_t) S: a decay
 * of each key channel. The recurrent (one-step) reading of the same layer, a
 * gated memory updated once per token, is the summary paragraph of the
 * podcast.app episode page ("Gated Linear Attention for Efficient Long
 * Sequences").
 * Output-after-update (o_t uses S_t, not S_{t-1}) is the plain reading of
 * o_t = q_t S_t; there is no 1/sqrt(d) scale and no normaliser inside the
 * layer (the pages give none).
 *
 * Backward (gla_oracle_bwd): plain reverse-mode chain rule through the same
 * step recurrence, with G = dL/dS_t carried backwards. S_t is not inverted
 * (dividing by a_t is unstable); instead the forward is re-run from
 * checkpoints taken every `seg` steps. The gate gradient is produced two
 * ways that share no arithmetic:
 *   dlog_a  (direct)  : dL/dlog a_t[c] = a_t[c] * sum_v G_t[c,v] S_{t-1}[c,v]
 *   dlog_a_cf (closed): sum_{s>=t} (q_s*dq_s - k_s*dk_s) + sum_v dhT*hT
 * The closed form is the one named in the Approach section ("a closed-form
 * gradient for the gates that avoids materializing per-step states"); its
 * derivation is restated in the repository's design notes.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC gla_oracle.c -o libgla_oracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef int64_t i64;

int gla_oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void gla_oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* One recurrence step on one (b,h) state S[K][V]: S = diag(exp(la)) S + k^T v,
 * then o = q S. `o` may be NULL. */
static void step_one(i64 K, i64 V, const double* q, const double* k,
                     const double* v, const double* la, double* S, double* o) {
    for (i64 c = 0; c < K; ++c) {
        const double a = exp(la[c]);
        const double kc = k[c];
        double* row = S + c * V;
        for (i64 x = 0; x < V; ++x) row[x] = a * row[x] + kc * v[x];
    }
    if (o) {
        for (i64 x = 0; x < V; ++x) o[x] = 0.0;
        for (i64 c = 0; c < K; ++c) {
            const double qc = q[c];
            const double* row = S + c * V;
            for (i64 x = 0; x < V; ++x) o[x] += qc * row[x];
        }
    }
}

/* Forward: o[B,H,L,V]; hT[B,H,K,V] (may be NULL); h0 may be NULL (zero). */
void gla_oracle_fwd(i64 B, i64 H, i64 L, i64 K, i64 V,
                    const double* q, const double* k, const double* v,
                    const double* log_a, const double* h0,
                    double* o, double* hT) {
    const i64 BH = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (i64 bh = 0; bh < BH; ++bh) {
        double* S = (double*)malloc(sizeof(double) * (size_t)(K * V));
        if (h0) memcpy(S, h0 + bh * K * V, sizeof(double) * (size_t)(K * V));
        else memset(S, 0, sizeof(double) * (size_t)(K * V));
        for (i64 t = 0; t < L; ++t) {
            const i64 rk = (bh * L + t) * K, rv = (bh * L + t) * V;
            step_one(K, V, q + rk, k + rk, v + rv, log_a + rk, S, o + rv);
        }
        if (hT) memcpy(hT + bh * K * V, S, sizeof(double) * (size_t)(K * V));
        free(S);
    }
}

/* Single decode step on a batch of states: S[B,H,K,V] updated in place,
 * o[B,H,V]. q,k,log_a: [B,H,K]; v: [B,H,V]. */
void gla_oracle_step(i64 B, i64 H, i64 K, i64 V,
                     const double* q, const double* k, const double* v,
                     const double* log_a, double* S, double* o) {
    const i64 BH = B * H;
#pragma omp parallel for schedule(static)
    for (i64 bh = 0; bh < BH; ++bh)
        step_one(K, V, q + bh * K, k + bh * K, v + bh * V, log_a + bh * K,
                 S + bh * K * V, o + bh * V);
}

/* Backward. Inputs as in the forward plus dO[B,H,L,V] and dhT[B,H,K,V]
 * (NULL = zero). Outputs dq, dk [B,H,L,K], dv [B,H,L,V], dlog_a and
 * dlog_a_cf [B,H,L,K] (either may be NULL), dh0 [B,H,K,V] (may be NULL).
 * `seg` is the checkpoint spacing (<= 0 picks 64). */
void gla_oracle_bwd(i64 B, i64 H, i64 L, i64 K, i64 V,
                    const double* q, const double* k, const double* v,
                    const double* log_a, const double* h0,
                    const double* dO, const double* dhT,
                    double* dq, double* dk, double* dv,
                    double* dlog_a, double* dlog_a_cf, double* dh0, i64 seg) {
    if (seg <= 0) seg = 64;
    const i64 BH = B * H;
    const i64 KV = K * V;
    const i64 nseg = (L + seg - 1) / seg;
#pragma omp parallel for schedule(dynamic, 1)
    for (i64 bh = 0; bh < BH; ++bh) {
        /* ckpt[g] = state before segment g (S_{g*seg - 1}); ckpt[nseg] = hT */
        double* ckpt = (double*)malloc(sizeof(double) * (size_t)((nseg + 1) * KV));
        double* Sseg = (double*)malloc(sizeof(double) * (size_t)((seg + 1) * KV));
        double* G = (double*)malloc(sizeof(double) * (size_t)KV);
        double* S = ckpt;
        if (h0) memcpy(S, h0 + bh * KV, sizeof(double) * (size_t)KV);
        else memset(S, 0, sizeof(double) * (size_t)KV);
        for (i64 g = 0; g < nseg; ++g) {
            double* nxt = ckpt + (g + 1) * KV;
            memcpy(nxt, ckpt + g * KV, sizeof(double) * (size_t)KV);
            const i64 t1 = (g + 1) * seg < L ? (g + 1) * seg : L;
            for (i64 t = g * seg; t < t1; ++t) {
                const i64 rk = (bh * L + t) * K, rv = (bh * L + t) * V;
                step_one(K, V, q + rk, k + rk, v + rv, log_a + rk, nxt, NULL);
            }
        }
        const double* hTbh = ckpt + nseg * KV;

        if (dhT) memcpy(G, dhT + bh * KV, sizeof(double) * (size_t)KV);
        else memset(G, 0, sizeof(double) * (size_t)KV);

        for (i64 g = nseg - 1; g >= 0; --g) {
            const i64 t0 = g * seg;
            const i64 t1 = (g + 1) * seg < L ? (g + 1) * seg : L;
            /* Sseg[0] = S_{t0-1}; Sseg[j+1] = S_{t0+j} */
            memcpy(Sseg, ckpt + g * KV, sizeof(double) * (size_t)KV);
            for (i64 t = t0; t < t1; ++t) {
                const i64 rk = (bh * L + t) * K, rv = (bh * L + t) * V;
                double* cur = Sseg + (t - t0 + 1) * KV;
                memcpy(cur, cur - KV, sizeof(double) * (size_t)KV);
                step_one(K, V, q + rk, k + rk, v + rv, log_a + rk, cur, NULL);
            }
            for (i64 t = t1 - 1; t >= t0; --t) {
                const i64 rk = (bh * L + t) * K, rv = (bh * L + t) * V;
                const double* St = Sseg + (t - t0 + 1) * KV;  /* S_t */
                const double* Sp = Sseg + (t - t0) * KV;      /* S_{t-1} */
                const double* qt = q + rk;
                const double* kt = k + rk;
                const double* vt = v + rv;
                const double* dot = dO + rv;
                /* o_t = q_t S_t contributes q_t^T do_t to dL/dS_t */
                for (i64 c = 0; c < K; ++c)
                    for (i64 x = 0; x < V; ++x) G[c * V + x] += qt[c] * dot[x];
                for (i64 c = 0; c < K; ++c) {
                    double acc_q = 0.0, acc_k = 0.0, acc_a = 0.0;
                    const double* Gr = G + c * V;
                    const double* Sr = St + c * V;
                    const double* Pr = Sp + c * V;
                    for (i64 x = 0; x < V; ++x) {
                        acc_q += Sr[x] * dot[x];  /* dL/dq_t = S_t do_t   */
                        acc_k += Gr[x] * vt[x];   /* dL/dk_t = G_t v_t    */
                        acc_a += Gr[x] * Pr[x];
                    }
                    dq[rk + c] = acc_q;
                    dk[rk + c] = acc_k;
                    if (dlog_a) dlog_a[rk + c] = exp(log_a[rk + c]) * acc_a;
                }
                for (i64 x = 0; x < V; ++x) {
                    double acc = 0.0;
                    for (i64 c = 0; c < K; ++c) acc += kt[c] * G[c * V + x];
                    dv[rv + x] = acc;                 /* dL/dv_t = k_t G_t */
                }
                /* S_t = diag(a_t) S_{t-1} + ... : dL/dS_{t-1} = diag(a_t) G */
                for (i64 c = 0; c < K; ++c) {
                    const double a = exp(log_a[rk + c]);
                    for (i64 x = 0; x < V; ++x) G[c * V + x] *= a;
                }
            }
        }
        if (dh0) memcpy(dh0 + bh * KV, G, sizeof(double) * (size_t)KV);

        if (dlog_a_cf) {
            /* constant term sum_v dhT * hT per key channel */
            for (i64 c = 0; c < K; ++c) {
                double base = 0.0;
                if (dhT)
                    for (i64 x = 0; x < V; ++x)
                        base += dhT[bh * KV + c * V + x] * hTbh[c * V + x];
                double run = base;
                for (i64 t = L - 1; t >= 0; --t) {
                    const i64 idx = (bh * L + t) * K + c;
                    run += q[idx] * dq[idx] - k[idx] * dk[idx];
                    dlog_a_cf[idx] = run;
                }
            }
        }
        free(G);
        free(Sseg);
        free(ckpt);
    }
}
