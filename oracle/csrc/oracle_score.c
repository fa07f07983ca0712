/* Fixed-order fp32 block score for the sparse mode's block ranking.
 *
 * TEST INFRASTRUCTURE ONLY (CPU oracle); never linked into the product path.
 *
 * The pages (fluxbbs.com, section on single-GPU kernels) fix only that, after
 * the first two denoising steps, 25 % of the candidate video blocks are kept.
 * The ranking rule is this project's own definition:
 *     score(qblock, kblock) = sum over c of qmean[c] * kmean[c]
 * evaluated as a chain of fused multiply-adds in channel order, starting from
 * +0.0f:  acc = fmaf(qmean[c], kmean[c], acc).  C99 fmaf rounds once, which is
 * what makes the chain exactly defined.  Build with -ffp-contract=off.
 */
#include <math.h>
#include <stdint.h>

void oracle_scores_fmaf(int64_t n_q, int64_t n_k, int64_t d,
                        const float *qmean, /* [n_q][d] */
                        const float *kmean, /* [n_k][d] */
                        float *out)         /* [n_q][n_k] */
{
    for (int64_t i = 0; i < n_q; ++i) {
        for (int64_t j = 0; j < n_k; ++j) {
            float acc = 0.0f;
            for (int64_t c = 0; c < d; ++c)
                acc = fmaf(qmean[i * d + c], kmean[j * d + c], acc);
            out[i * n_k + j] = acc;
        }
    }
}
