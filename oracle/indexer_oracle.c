/*
 * fp64 CPU oracle for the DeepSeek-Sparse-Attention lightning indexer.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this library. It shares no code with the
 * CUDA path and must never be linked into it.
 *
 * Everything here works on fp64 copies of the already-rounded inputs (bf16
 * widened exactly, FP8 bytes decoded exactly and multiplied by their fp32
 * scales, both exact in fp64), with plain sequential summation.
 *
 * Sources for the arithmetic:
 *  - Lightning-indexer score of DeepSeek Sparse Attention: every prefix token
 *    is scored by H_I indexer heads ("MISA: Mixture of Indexer Sparse
 *    Attention for Long-Context LLM Inference", section "Problem statement");
 *    head weights are signed and per-head terms non-negative ("DoSA: Dots
 *    Sparse Attention" review, section 3, "Nonnegative Head Projection" and
 *    "Signed Indexer Score"):
 *        I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,:])
 *    "cond" is the condition scale sum_h |w[t,h]| * ReLU(q[t,h,:] . k[s,:]),
 *    used by the tests to bound rounding error of a signed sum.
 *  - MISA router (MISA page, section "Methodology", step 1): per-head
 *    affinity over mean-pooled block keys, aggregated per head,
 *        a[t,h] = |w[t,h]| * sum_{visible blocks m} ReLU(q[t,h,:] . kbar[m,:])
 */
#include <stdint.h>
#include <stddef.h>

/* Score explicit (query row, key row) pairs.
 *   q     [nq, H, d]  fp64
 *   k     [nk, d]     fp64
 *   w     [nq, H]     fp64 (signed)
 *   hmask [nq, H]     optional; when non-NULL only heads with hmask != 0 count
 *                     (MISA routed scoring on the selected heads)
 *   pq[i], pk[i]      query row and key row of pair i
 *   out[i]            score of pair i;  cond[i] (optional) its condition scale
 */
void or_score_pairs(const double* q, const double* k, const double* w,
                    const unsigned char* hmask, int H, int d, long long npairs,
                    const long long* pq, const long long* pk,
                    double* out, double* cond)
{
    long long i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < npairs; ++i) {
        const long long t = pq[i];
        const double* ks = k + (size_t)pk[i] * d;
        double s = 0.0, c = 0.0;
        for (int h = 0; h < H; ++h) {
            if (hmask && !hmask[(size_t)t * H + h]) continue;
            const double* qh = q + ((size_t)t * H + h) * d;
            double dot = 0.0;
            for (int j = 0; j < d; ++j) dot += qh[j] * ks[j];
            const double relu = dot > 0.0 ? dot : 0.0;
            const double wh = w[(size_t)t * H + h];
            s += wh * relu;
            c += (wh < 0.0 ? -wh : wh) * relu;
        }
        out[i] = s;
        if (cond) cond[i] = c;
    }
}

/* MISA router affinity.
 *   q    [nq, H, d] fp64, kbar [M, d] fp64, w [nq, H] fp64
 *   nvis[t]  number of visible pooled blocks of query t (blocks 0..nvis-1)
 *   a    [nq, H] output
 */
void or_router(const double* q, const double* kbar, const double* w,
               long long nq, int H, int d, long long M, const long long* nvis,
               double* a)
{
    long long th;
#pragma omp parallel for schedule(static)
    for (th = 0; th < nq * H; ++th) {
        const long long t = th / H;
        const double* qh = q + (size_t)th * d;
        long long nv = nvis[t] < M ? nvis[t] : M;
        double acc = 0.0;
        for (long long m = 0; m < nv; ++m) {
            const double* km = kbar + (size_t)m * d;
            double dot = 0.0;
            for (int j = 0; j < d; ++j) dot += qh[j] * km[j];
            acc += dot > 0.0 ? dot : 0.0;
        }
        const double wh = w[th];
        a[th] = (wh < 0.0 ? -wh : wh) * acc;
    }
}

int or_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
