/*
 * fp64 sequential oracle of the Mamba-2 state-space-duality (SSD) recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * definition that the CUDA path is checked against.  Only the tests, the
 * package's smoke check and the benchmark's CPU-baseline leg may load it.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * Source: "Compiler-First State Space Duality and Portable O(1) Autoregressive
 * Caching for Inference" (gist.science summary of arXiv 2603.09555), section
 * "2. Metodologia": per-head diagonal state dynamics, a chunkable recurrence,
 * decay factors exponentiated in fp32 or wider, and an O(1) state cache that
 * one decode step advances.  The page does not print the equations.  The
 * recurrence used here is the standard Mamba-2 SSD layer, for every batch b and
 * head h, with group g = h / (nheads / ngroups):
 *
 *     a_t = exp(dt_t * A_h)
 *     H_t = a_t * H_{t-1} + dt_t * B_t x_t^T        (H is N x P, H_{-1} = init or 0)
 *     y_t = C_t^T H_t + D_h * x_t                    (y uses the updated state)
 *
 * H is stored transposed, as [P][N] (dstate innermost), which is the layout of
 * the state cache everywhere in this project.
 *
 * Inputs are fp32 arrays (bf16 inputs are passed after exact widening); all
 * arithmetic is fp64 and follows the recurrence token by token, without any
 * chunking, blocking or reordering.  Parallelism is over independent (b, h)
 * units only; each unit is computed in program order.
 *
 * Parity pins (tests/test_oracle_*.py): a chunked fp64 form and the quadratic
 * (masked-matrix) form written separately in numpy, closed forms (A = 0 gives a
 * cumulative sum; constant dt gives a geometric series), identities (C = 0,
 * B = 0, dt = 0, linearity, batch permutation), prefill/decode resume, and a
 * hand-computed tiny case under tests/golden/.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Unit u covers (b, h) = (units[u] / nheads, units[u] % nheads); NULL units
 * means all batch*nheads units in order. */
static int unit_index(const int* units, int u) { return units ? units[u] : u; }

/*
 * Prefill of `seqlen` tokens.
 *   x        [batch][seqlen][nheads][headdim]
 *   dt       [batch][seqlen][nheads]          (positive)
 *   A, D     [nheads]
 *   Bm, Cm   [batch][seqlen][ngroups][dstate]
 *   init     [n_units][headdim][dstate] or NULL (zeros)
 *   y        [n_units][seqlen][headdim]        (output)
 *   state    [n_units][headdim][dstate]        (output: H after the last token)
 * Returns 0, or -1 on an invalid shape.
 */
int ssd_oracle_prefill(const float* x, const float* dt, const float* A, const float* Bm,
                       const float* Cm, const float* D, const double* init, int batch,
                       int seqlen, int nheads, int headdim, int ngroups, int dstate,
                       const int* units, int n_units, double* y, double* state, int nthreads)
{
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || ngroups <= 0 ||
        dstate <= 0 || nheads % ngroups != 0)
        return -1;
    if (!units) n_units = batch * nheads;
    const int heads_per_group = nheads / ngroups;
    const size_t PN = (size_t)headdim * dstate;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < n_units; ++u) {
        const int bh = unit_index(units, u);
        const int b = bh / nheads, h = bh % nheads, g = h / heads_per_group;
        double* H = state + (size_t)u * PN;
        if (init)
            memcpy(H, init + (size_t)u * PN, PN * sizeof(double));
        else
            memset(H, 0, PN * sizeof(double));
        for (int t = 0; t < seqlen; ++t) {
            const size_t tok = (size_t)b * seqlen + t;
            const double dtv = dt[tok * nheads + h];
            const double a = exp(dtv * (double)A[h]);
            const float* xt = x + (tok * nheads + h) * headdim;
            const float* Bt = Bm + (tok * ngroups + g) * dstate;
            const float* Ct = Cm + (tok * ngroups + g) * dstate;
            double* yt = y + ((size_t)u * seqlen + t) * headdim;
            for (int p = 0; p < headdim; ++p) {
                double* Hp = H + (size_t)p * dstate;
                const double dx = dtv * (double)xt[p];
                double acc = 0.0;
                for (int n = 0; n < dstate; ++n) {
                    Hp[n] = a * Hp[n] + dx * (double)Bt[n];
                    acc += (double)Ct[n] * Hp[n];
                }
                yt[p] = acc + (double)D[h] * (double)xt[p];
            }
        }
    }
    return 0;
}

/*
 * One decode step: the same update for a single token, on a given state.
 *   state    [n_units][headdim][dstate]  (in/out)
 *   x_t      [batch][nheads][headdim]
 *   dt_t     [batch][nheads]
 *   B_t, C_t [batch][ngroups][dstate]
 *   y_t      [n_units][headdim]          (output)
 */
int ssd_oracle_decode_step(double* state, const float* x_t, const float* dt_t, const float* A,
                           const float* B_t, const float* C_t, const float* D, int batch,
                           int nheads, int headdim, int ngroups, int dstate, const int* units,
                           int n_units, double* y_t, int nthreads)
{
    if (batch < 0 || nheads <= 0 || headdim <= 0 || ngroups <= 0 || dstate <= 0 ||
        nheads % ngroups != 0)
        return -1;
    if (!units) n_units = batch * nheads;
    const int heads_per_group = nheads / ngroups;
    const size_t PN = (size_t)headdim * dstate;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(static)
    for (int u = 0; u < n_units; ++u) {
        const int bh = unit_index(units, u);
        const int b = bh / nheads, h = bh % nheads, g = h / heads_per_group;
        double* H = state + (size_t)u * PN;
        const double dtv = dt_t[(size_t)b * nheads + h];
        const double a = exp(dtv * (double)A[h]);
        const float* xt = x_t + ((size_t)b * nheads + h) * headdim;
        const float* Bt = B_t + ((size_t)b * ngroups + g) * dstate;
        const float* Ct = C_t + ((size_t)b * ngroups + g) * dstate;
        for (int p = 0; p < headdim; ++p) {
            double* Hp = H + (size_t)p * dstate;
            const double dx = dtv * (double)xt[p];
            double acc = 0.0;
            for (int n = 0; n < dstate; ++n) {
                Hp[n] = a * Hp[n] + dx * (double)Bt[n];
                acc += (double)Ct[n] * Hp[n];
            }
            y_t[(size_t)u * headdim + p] = acc + (double)D[h] * (double)xt[p];
        }
    }
    return 0;
}

/* Number of threads an OpenMP parallel region would use with this request. */
int ssd_oracle_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) return nthreads;
    return omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}
