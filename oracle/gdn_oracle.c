/*
 * fp64 CPU oracle for the Gated DeltaNet decode step -- TEST INFRASTRUCTURE.
 *
 * Only tests/ and the benchmark's CPU-baseline leg may use this file.  The CUDA library
 * never calls it and shares no code with it.
 *
 * "Persistent-State Dataflow Accelerator for Memory-Bound Linear Attention Decode on
 * FPGA", section 2.B: each value head keeps a dk x dv state S and a token updates it as
 *     S_t = g S_{t-1} + k dv^T,       output o_t = S_t^T q,
 * with g the head's gate.  The page writes dv (the delta-rule correction) without
 * defining it; the reading used here is the gated delta rule,
 *     dv = beta (v - g S_{t-1}^T k),
 * i.e. S_t = g (I - beta k k^T) S_{t-1} + beta k v^T.  Section 2.C: value heads come in
 * groups that share one query/key head (two per query/key head in the page's model);
 * value head h reads query/key head h / (hv / hqk).
 *
 * The step below is the definition written out in the order above: the retrieval
 * S_{t-1}^T k, the correction dv, the update of every state element, then the output
 * from the updated state.
 */
#include <math.h>
#include <stddef.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/*
 * state [batch][hv][dk][dv] fp64, updated in place; q, k [batch][hqk][dk]; v [batch][hv][dv];
 * gate, beta [batch][hv]; out [batch][hv][dv] fp64.  Returns 0, or 1 on bad sizes.
 */
int gdn_oracle_decode_step(double* state, const float* q, const float* k, const float* v,
                           const float* gate, const float* beta, int batch, int hqk, int hv, int dk,
                           int dv, double* out, int nthreads)
{
    if (batch < 0 || hqk <= 0 || hv <= 0 || hv % hqk != 0 || dk <= 0 || dv <= 0) return 1;
    const int group = hv / hqk;
    const int units = batch * hv;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int u = 0; u < units; ++u) {
        const int b = u / hv, h = u % hv, hk = h / group;
        const float* qh = q + ((size_t)b * hqk + hk) * dk;
        const float* kh = k + ((size_t)b * hqk + hk) * dk;
        const float* vh = v + (size_t)u * dv;
        const double g = (double)gate[u], bt = (double)beta[u];
        double* S = state + (size_t)u * dk * dv;
        double* o = out + (size_t)u * dv;
        for (int j = 0; j < dv; ++j) {
            double r = 0.0;                                  /* (S_{t-1}^T k)_j */
            for (int i = 0; i < dk; ++i) r += S[(size_t)i * dv + j] * (double)kh[i];
            const double corr = bt * ((double)vh[j] - g * r);
            for (int i = 0; i < dk; ++i)
                S[(size_t)i * dv + j] = g * S[(size_t)i * dv + j] + (double)kh[i] * corr;
            double acc = 0.0;                                /* (S_t^T q)_j */
            for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * (double)qh[i];
            o[j] = acc;
        }
    }
    return 0;
}
