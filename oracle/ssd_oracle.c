/*
 * ssd_oracle.c -- CPU fp64 oracle for the SSD (Mamba-2 structured state space
 * duality) forward pass.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls
 * this file: only the tests, the package smoke check and the benchmark's CPU
 * baseline leg do. It shares no code, header or constant with the CUDA path.
 *
 * What it computes is the plain definition of the layer, step by step, in fp64:
 *
 *   H_t = a_t H_{t-1} + B_t x_t^T,   y_t = C_t^T H_t + D x_t,   a_t = exp(log a_t)
 *
 * with H in R^{N x P}, B_t, C_t in R^N, x_t in R^P and one scalar decay a_t per
 * head and step. Sources: "Mamba-2: writing the recurrent state as a structured
 * matrix" (wq-win.github.io/llm/088-mamba2.html), section 2.1 "unrolling the
 * history" (the recurrence and its unrolled sum), and "Mamba and state space
 * models" (wang-x-xia.github.io, learn-ai/foundations), section 2 "formal
 * definition" (the discrete form with the D x skip term).
 *
 * Readings taken where the pages are silent (each is listed with its reason in
 * the design notes):
 *  - init_states is H_{-1}: the first step's a_0 decays it, as in the pages'
 *    chunk-split example where the incoming state 5 is multiplied by 0.5.
 *  - seq_idx marks independent samples. When seq_idx[b,t] != seq_idx[b,t-1], the
 *    state of the finished sequence is stored as its final state and H restarts
 *    from that sequence's initial state (or zero). The pages require that only
 *    independent-sample boundaries block state propagation (section 2.3 and the
 *    testing advice in section 5 of the same page).
 *  - D is one scalar per head, added after the read-out, never fed into H.
 *  - Head h uses group g = h / (nheads / ngroups) of B and C (contiguous heads
 *    share a group). The pages only say B and C are shared across heads.
 *  - Sequence ids that never occur in a row keep their initial state (or zero)
 *    as their final state.
 *
 * Layouts (row-major, all fp64 except seq_idx):
 *   X [batch, seqlen, nheads, headdim]     log_a [batch, seqlen, nheads]
 *   B, C [batch, seqlen, ngroups, dstate]  D [nheads] or NULL
 *   init_states, final_states [batch, nseq, nheads, dstate, headdim] (may be NULL)
 *   seq_idx [batch, seqlen] int32 or NULL  Y [batch, seqlen, nheads, headdim]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int check_dims(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                      int64_t dstate, int64_t ngroups, int64_t nseq) {
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0) return 1;
    if (ngroups <= 0 || nheads % ngroups != 0 || nseq <= 0) return 1;
    return 0;
}

static int seq_of(const int32_t* seq_idx, int64_t b, int64_t seqlen, int64_t t, int64_t nseq) {
    if (!seq_idx) return 0;
    int32_t s = seq_idx[b * seqlen + t];
    if (s < 0) s = 0;
    if (s >= nseq) s = (int32_t)(nseq - 1);
    return s;
}

static void load_state(double* H, const double* init_states, int64_t b, int64_t s, int64_t h,
                       int64_t nseq, int64_t nheads, int64_t NP) {
    if (init_states)
        memcpy(H, init_states + ((b * nseq + s) * nheads + h) * NP, (size_t)NP * sizeof(double));
    else
        memset(H, 0, (size_t)NP * sizeof(double));
}

/* Step-by-step recurrence. Returns 0 on success, 1 on bad arguments, 2 on
 * allocation failure. nthreads <= 0 uses the OpenMP default. */
int ssd_oracle_fwd(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                   int64_t dstate, int64_t ngroups, int64_t nseq,
                   const double* X, const double* log_a, const double* B, const double* C,
                   const double* D, const double* init_states, const int32_t* seq_idx,
                   double* Y, double* final_states, int nthreads) {
    if (check_dims(batch, seqlen, nheads, headdim, dstate, ngroups, nseq)) return 1;
    if (!X || !log_a || !B || !C || !Y) return 1;
    if (!seq_idx && nseq != 1) return 1;
    const int64_t P = headdim, N = dstate, NP = dstate * headdim;
    const int64_t heads_per_group = nheads / ngroups;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : failed)
#endif
    for (int64_t bh = 0; bh < batch * nheads; ++bh) {
        const int64_t b = bh / nheads, h = bh % nheads, g = h / heads_per_group;
        double* H = (double*)malloc((size_t)NP * sizeof(double));
        if (!H) { failed |= 1; continue; }
        if (final_states)
            for (int64_t s = 0; s < nseq; ++s)
                load_state(final_states + ((b * nseq + s) * nheads + h) * NP, init_states, b, s, h,
                           nseq, nheads, NP);
        int64_t cur = seq_of(seq_idx, b, seqlen, 0, nseq);
        load_state(H, init_states, b, cur, h, nseq, nheads, NP);
        for (int64_t t = 0; t < seqlen; ++t) {
            const int64_t s = seq_of(seq_idx, b, seqlen, t, nseq);
            if (t > 0 && s != cur) {
                /* independent-sample boundary: keep the finished state, restart */
                if (final_states)
                    memcpy(final_states + ((b * nseq + cur) * nheads + h) * NP, H,
                           (size_t)NP * sizeof(double));
                cur = s;
                load_state(H, init_states, b, cur, h, nseq, nheads, NP);
            }
            const int64_t bt = b * seqlen + t;
            const double a = exp(log_a[bt * nheads + h]);
            const double* x = X + (bt * nheads + h) * P;
            const double* Bt = B + (bt * ngroups + g) * N;
            const double* Ct = C + (bt * ngroups + g) * N;
            double* y = Y + (bt * nheads + h) * P;
            /* H_t = a_t H_{t-1} + B_t x_t^T */
            for (int64_t n = 0; n < N; ++n)
                for (int64_t p = 0; p < P; ++p)
                    H[n * P + p] = a * H[n * P + p] + Bt[n] * x[p];
            /* y_t = C_t^T H_t + D x_t */
            for (int64_t p = 0; p < P; ++p) {
                double acc = D ? D[h] * x[p] : 0.0;
                for (int64_t n = 0; n < N; ++n) acc += Ct[n] * H[n * P + p];
                y[p] = acc;
            }
        }
        if (final_states && seqlen > 0)
            memcpy(final_states + ((b * nseq + cur) * nheads + h) * NP, H, (size_t)NP * sizeof(double));
        free(H);
    }
    return failed ? 2 : 0;
}

/* States at chunk boundaries, by the same recurrence (for localising errors in
 * the chunked path). For chunk c = [cQ, cQ+Q):
 *   incoming[b,c,h] = the state the recurrence holds just before token cQ for
 *       the sequence of token cQ: H after token cQ-1 when that token belongs to
 *       the same sequence, else that sequence's initial state (or zero);
 *   local[b,c,h]    = the state at the end of the chunk of a recurrence that
 *       starts from zero at the first token of the chunk's last sequence piece
 *       (max(cQ, start of that sequence)).
 * Both are [batch, nchunks, nheads, dstate, headdim], nchunks = ceil(seqlen /
 * chunk) (the last chunk may be shorter); either may be NULL. */
int ssd_oracle_chunk_states(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                            int64_t dstate, int64_t ngroups, int64_t nseq, int64_t chunk,
                            const double* X, const double* log_a, const double* B,
                            const double* init_states, const int32_t* seq_idx,
                            double* incoming, double* local, int nthreads) {
    if (check_dims(batch, seqlen, nheads, headdim, dstate, ngroups, nseq)) return 1;
    if (chunk <= 0 || !X || !log_a || !B) return 1;
    if (!seq_idx && nseq != 1) return 1;
    const int64_t P = headdim, N = dstate, NP = dstate * headdim, nchunks = (seqlen + chunk - 1) / chunk;
    const int64_t heads_per_group = nheads / ngroups;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : failed)
#endif
    for (int64_t bh = 0; bh < batch * nheads; ++bh) {
        const int64_t b = bh / nheads, h = bh % nheads, g = h / heads_per_group;
        double* H = (double*)malloc((size_t)NP * sizeof(double));
        double* L = (double*)malloc((size_t)NP * sizeof(double));
        if (!H || !L) { free(H); free(L); failed |= 1; continue; }
        int64_t cur = seq_of(seq_idx, b, seqlen, 0, nseq);
        load_state(H, init_states, b, cur, h, nseq, nheads, NP);
        for (int64_t c = 0; c < nchunks; ++c) {
            const int64_t t0 = c * chunk;
            const int64_t t1 = (t0 + chunk < seqlen) ? t0 + chunk : seqlen;
            const int64_t s_last = seq_of(seq_idx, b, seqlen, t1 - 1, nseq);
            memset(L, 0, (size_t)NP * sizeof(double));
            for (int64_t t = t0; t < t1; ++t) {
                const int64_t s = seq_of(seq_idx, b, seqlen, t, nseq);
                if (t > 0 && s != cur) {
                    cur = s;
                    load_state(H, init_states, b, cur, h, nseq, nheads, NP);
                }
                if (t == t0 && incoming)
                    memcpy(incoming + ((b * nchunks + c) * nheads + h) * NP, H,
                           (size_t)NP * sizeof(double));
                const int64_t bt = b * seqlen + t;
                const double a = exp(log_a[bt * nheads + h]);
                const double* x = X + (bt * nheads + h) * P;
                const double* Bt = B + (bt * ngroups + g) * N;
                for (int64_t n = 0; n < N; ++n)
                    for (int64_t p = 0; p < P; ++p)
                        H[n * P + p] = a * H[n * P + p] + Bt[n] * x[p];
                if (s == s_last)
                    for (int64_t n = 0; n < N; ++n)
                        for (int64_t p = 0; p < P; ++p)
                            L[n * P + p] = a * L[n * P + p] + Bt[n] * x[p];
            }
            if (local) memcpy(local + ((b * nchunks + c) * nheads + h) * NP, L, (size_t)NP * sizeof(double));
        }
        free(H);
        free(L);
    }
    return failed ? 2 : 0;
}

int ssd_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
