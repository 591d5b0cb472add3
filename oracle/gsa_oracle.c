/*
 * Gated slot attention (GSA) oracle: plain fp64 CPU reference.
 *
 * TEST INFRASTRUCTURE ONLY, like gla_oracle.c beside it: only the tests, the
 * smoke check and the CPU legs of the benchmark may call it. It shares no
 * code with the CUDA library (nor with gla_oracle.c).
 *
 * Source: the mlsanity card for "Gated Slot Attention for Efficient
 * Linear-Time Sequence Modeling" (abstract). The method keeps a bounded memory
 * of m slots, forgets it with a GLA-style data-dependent gate, and reads it in
 * two GLA layers joined by a softmax over the slots. The card prints no
 * equations; the reading taken here (the plainest one the abstract supports)
 * is, per batch b and head h, with a_t = exp(log_a_t) in (0,1]^m and the
 * write weight 1 - a_t (a slot writes what it forgets):
 *
 *   Kmem_t = diag(a_t) Kmem_{t-1} + (1 - a_t)^T k_t        [m x K]
 *   Vmem_t = diag(a_t) Vmem_{t-1} + (1 - a_t)^T v_t        [m x V]
 *   s_t    = softmax_m(Kmem_t q_t^T)                       (read after the update)
 *   o_t    = s_t Vmem_t
 *
 * Layouts (row-major, contiguous): q, k [B,H,L,K]; v, o, dO [B,H,L,V];
 * log_a [B,H,L,m]; hk [B,H,m,K]; hv [B,H,m,V]. No scale inside the softmax.
 *
 * Backward (gsa_oracle_bwd): plain reverse-mode chain rule through the same
 * step recurrence with GK = dL/dKmem_t and GV = dL/dVmem_t carried backwards;
 * the memories are re-run from checkpoints every `seg` steps (never inverted).
 * The loss is <dO, o> + <dhk, Kmem_T> + <dhv, Vmem_T>.
 *
 * Build: compiled into libgla_oracle.so together with gla_oracle.c.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef int64_t i64;

/* Kmem, Vmem <- one step with key k, value v and log gate la (m entries). */
static void gsa_update(i64 m, i64 K, i64 V, const double* k, const double* v, const double* la, double* Km,
                       double* Vm) {
    for (i64 c = 0; c < m; ++c) {
        const double a = exp(la[c]), w = 1.0 - a;
        double* kr = Km + c * K;
        double* vr = Vm + c * V;
        for (i64 d = 0; d < K; ++d) kr[d] = a * kr[d] + w * k[d];
        for (i64 x = 0; x < V; ++x) vr[x] = a * vr[x] + w * v[x];
    }
}

/* s = softmax over the m slots of Kmem q^T (max-subtracted). */
static void gsa_read_weights(i64 m, i64 K, const double* Km, const double* q, double* s) {
    double mx = -INFINITY;
    for (i64 c = 0; c < m; ++c) {
        double z = 0.0;
        for (i64 d = 0; d < K; ++d) z += Km[c * K + d] * q[d];
        s[c] = z;
        if (z > mx) mx = z;
    }
    double sum = 0.0;
    for (i64 c = 0; c < m; ++c) {
        s[c] = exp(s[c] - mx);
        sum += s[c];
    }
    for (i64 c = 0; c < m; ++c) s[c] /= sum;
}

static void gsa_output(i64 m, i64 V, const double* s, const double* Vm, double* o) {
    for (i64 x = 0; x < V; ++x) o[x] = 0.0;
    for (i64 c = 0; c < m; ++c)
        for (i64 x = 0; x < V; ++x) o[x] += s[c] * Vm[c * V + x];
}

static void gsa_init(i64 bh, i64 m, i64 K, i64 V, const double* hk0, const double* hv0, double* Km, double* Vm) {
    if (hk0) memcpy(Km, hk0 + bh * m * K, sizeof(double) * (size_t)(m * K));
    else memset(Km, 0, sizeof(double) * (size_t)(m * K));
    if (hv0) memcpy(Vm, hv0 + bh * m * V, sizeof(double) * (size_t)(m * V));
    else memset(Vm, 0, sizeof(double) * (size_t)(m * V));
}

/* Forward: o[B,H,L,V]; s[B,H,L,m] (read weights, may be NULL); hkT, hvT (final memories, may be NULL);
 * hk0, hv0 may be NULL (zero). */
void gsa_oracle_fwd(i64 B, i64 H, i64 L, i64 K, i64 V, i64 m, const double* q, const double* k, const double* v,
                    const double* log_a, const double* hk0, const double* hv0, double* o, double* s_out,
                    double* hkT, double* hvT) {
    const i64 BH = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (i64 bh = 0; bh < BH; ++bh) {
        double* Km = (double*)malloc(sizeof(double) * (size_t)(m * K));
        double* Vm = (double*)malloc(sizeof(double) * (size_t)(m * V));
        double* s = (double*)malloc(sizeof(double) * (size_t)m);
        gsa_init(bh, m, K, V, hk0, hv0, Km, Vm);
        for (i64 t = 0; t < L; ++t) {
            const i64 rk = (bh * L + t) * K, rv = (bh * L + t) * V, rm = (bh * L + t) * m;
            gsa_update(m, K, V, k + rk, v + rv, log_a + rm, Km, Vm);
            gsa_read_weights(m, K, Km, q + rk, s);
            gsa_output(m, V, s, Vm, o + rv);
            if (s_out) memcpy(s_out + rm, s, sizeof(double) * (size_t)m);
        }
        if (hkT) memcpy(hkT + bh * m * K, Km, sizeof(double) * (size_t)(m * K));
        if (hvT) memcpy(hvT + bh * m * V, Vm, sizeof(double) * (size_t)(m * V));
        free(Km);
        free(Vm);
        free(s);
    }
}

/* Backward of <dO, o> + <dhkT, Kmem_T> + <dhvT, Vmem_T> (dhkT, dhvT may be NULL = 0).
 * Outputs dq, dk [B,H,L,K]; dv [B,H,L,V]; dlog_a [B,H,L,m]; dhk0 [B,H,m,K]; dhv0 [B,H,m,V]
 * (dhk0, dhv0 may be NULL). */
void gsa_oracle_bwd(i64 B, i64 H, i64 L, i64 K, i64 V, i64 m, const double* q, const double* k, const double* v,
                    const double* log_a, const double* hk0, const double* hv0, const double* dO,
                    const double* dhkT, const double* dhvT, double* dq, double* dk, double* dv, double* dlog_a,
                    double* dhk0, double* dhv0, i64 seg) {
    const i64 BH = B * H;
    if (seg < 1) seg = 1;
    const i64 nck = (L + seg - 1) / seg;
#pragma omp parallel for schedule(dynamic, 1)
    for (i64 bh = 0; bh < BH; ++bh) {
        const size_t nk = (size_t)(m * K), nv = (size_t)(m * V);
        /* checkpoints: the memories entering steps 0, seg, 2 seg, ... */
        double* ckK = (double*)malloc(sizeof(double) * nk * (size_t)(nck > 0 ? nck : 1));
        double* ckV = (double*)malloc(sizeof(double) * nv * (size_t)(nck > 0 ? nck : 1));
        /* the memories after each step of the current segment (slot 0 = entering the segment) */
        double* segK = (double*)malloc(sizeof(double) * nk * (size_t)(seg + 1));
        double* segV = (double*)malloc(sizeof(double) * nv * (size_t)(seg + 1));
        double* GK = (double*)malloc(sizeof(double) * nk);
        double* GV = (double*)malloc(sizeof(double) * nv);
        double* s = (double*)malloc(sizeof(double) * (size_t)m);
        double* ds = (double*)malloc(sizeof(double) * (size_t)m);
        double* dz = (double*)malloc(sizeof(double) * (size_t)m);

        double* Km = segK;
        double* Vm = segV;
        gsa_init(bh, m, K, V, hk0, hv0, Km, Vm);
        for (i64 t = 0; t < L; ++t) {
            if (t % seg == 0) {
                memcpy(ckK + (t / seg) * nk, Km, sizeof(double) * nk);
                memcpy(ckV + (t / seg) * nv, Vm, sizeof(double) * nv);
            }
            gsa_update(m, K, V, k + (bh * L + t) * K, v + (bh * L + t) * V, log_a + (bh * L + t) * m, Km, Vm);
        }
        if (dhkT) memcpy(GK, dhkT + bh * nk, sizeof(double) * nk);
        else memset(GK, 0, sizeof(double) * nk);
        if (dhvT) memcpy(GV, dhvT + bh * nv, sizeof(double) * nv);
        else memset(GV, 0, sizeof(double) * nv);

        for (i64 g = nck - 1; g >= 0; --g) {
            const i64 t0 = g * seg, t1 = (t0 + seg < L) ? t0 + seg : L;
            memcpy(segK, ckK + g * nk, sizeof(double) * nk);
            memcpy(segV, ckV + g * nv, sizeof(double) * nv);
            for (i64 t = t0; t < t1; ++t) {
                const i64 j = t - t0;
                memcpy(segK + (j + 1) * nk, segK + j * nk, sizeof(double) * nk);
                memcpy(segV + (j + 1) * nv, segV + j * nv, sizeof(double) * nv);
                gsa_update(m, K, V, k + (bh * L + t) * K, v + (bh * L + t) * V, log_a + (bh * L + t) * m,
                           segK + (j + 1) * nk, segV + (j + 1) * nv);
            }
            for (i64 t = t1 - 1; t >= t0; --t) {
                const i64 j = t - t0;
                const double* Kt = segK + (j + 1) * nk; /* Kmem_t */
                const double* Vt = segV + (j + 1) * nv;
                const double* Kp = segK + j * nk;       /* Kmem_{t-1} */
                const double* Vp = segV + j * nv;
                const i64 rk = (bh * L + t) * K, rv = (bh * L + t) * V, rm = (bh * L + t) * m;
                const double* qt = q + rk;
                const double* dot = dO + rv;
                gsa_read_weights(m, K, Kt, qt, s);
                /* o_t = s Vmem_t */
                for (i64 c = 0; c < m; ++c) {
                    double acc = 0.0;
                    for (i64 x = 0; x < V; ++x) {
                        GV[c * V + x] += s[c] * dot[x];
                        acc += dot[x] * Vt[c * V + x];
                    }
                    ds[c] = acc;
                }
                /* s = softmax(z): dz = s * (ds - <s, ds>) */
                double sd = 0.0;
                for (i64 c = 0; c < m; ++c) sd += s[c] * ds[c];
                for (i64 c = 0; c < m; ++c) dz[c] = s[c] * (ds[c] - sd);
                /* z = Kmem_t q^T */
                for (i64 d = 0; d < K; ++d) dq[rk + d] = 0.0;
                for (i64 c = 0; c < m; ++c)
                    for (i64 d = 0; d < K; ++d) {
                        dq[rk + d] += dz[c] * Kt[c * K + d];
                        GK[c * K + d] += dz[c] * qt[d];
                    }
                /* Kmem_t = diag(a) Kmem_{t-1} + (1 - a)^T k_t, the same for Vmem */
                const double* kt = k + rk;
                const double* vt = v + rv;
                for (i64 d = 0; d < K; ++d) dk[rk + d] = 0.0;
                for (i64 x = 0; x < V; ++x) dv[rv + x] = 0.0;
                for (i64 c = 0; c < m; ++c) {
                    const double a = exp(log_a[rm + c]), w = 1.0 - a;
                    double dw = 0.0, da = 0.0;
                    for (i64 d = 0; d < K; ++d) {
                        const double gk = GK[c * K + d];
                        dk[rk + d] += w * gk;
                        dw += gk * kt[d];
                        da += gk * Kp[c * K + d];
                        GK[c * K + d] = a * gk;
                    }
                    for (i64 x = 0; x < V; ++x) {
                        const double gv = GV[c * V + x];
                        dv[rv + x] += w * gv;
                        dw += gv * vt[x];
                        da += gv * Vp[c * V + x];
                        GV[c * V + x] = a * gv;
                    }
                    /* a = exp(la), w = 1 - a: d/dla = a * (dL/da - dL/dw) */
                    dlog_a[rm + c] = a * (da - dw);
                }
            }
        }
        if (dhk0) memcpy(dhk0 + bh * nk, GK, sizeof(double) * nk);
        if (dhv0) memcpy(dhv0 + bh * nv, GV, sizeof(double) * nv);
        free(ckK);
        free(ckV);
        free(segK);
        free(segV);
        free(GK);
        free(GV);
        free(s);
        free(ds);
        free(dz);
    }
}
