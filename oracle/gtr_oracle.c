/*
 * Oracle for the key-only gated linear attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code with the CUDA path.
 *
 * What it computes (GTR: Gated Token Recurrence for Efficient Dense
 * Prediction; digest page "paper.rainbus.top/paper/2609.26590", prerequisite
 * "Gated linear attention (GLA)" and section "Core method"; page
 * "0539edu.com", section 3.1 "Key-only gated recurrence"):
 *
 *     S_t = Diag(gamma_t) S_{t-1} + k_t^T v_t ,   S_{-1} = 0
 *     o_t = d_k^{-1/2} q_t S_t
 *
 * with S_t a d_k x d_v matrix per (batch, head), gamma_t in (0,1] a per-key-
 * channel gate (the value side is not decayed) and a zero initial state (the
 * operator specialisation in step 5 of "Method details" on the first page).
 * The tokens are visited in one of four scan orders over the H x W patch grid
 * (section "Core method": left->right, right->left, top->bottom,
 * bottom->top).  The pages do not spell the orders out; the reading used is:
 *
 *   0 left->right : rows top to bottom, each row x = 0 .. W-1
 *   1 right->left : rows top to bottom, each row x = W-1 .. 0
 *   2 top->bottom : columns left to right, each column y = 0 .. H-1
 *   3 bottom->top : columns left to right, each column y = H-1 .. 0
 *
 * and one sequence of L = H*W tokens: the state carries across line ends.
 *
 * Data layout: every tensor is [B, L, heads, d] row-major, token index
 * m = y*W + x.  log_gamma holds log(gamma), shape [B, L, heads, d_k].
 * All arithmetic is IEEE double.  This is the plain sequential definition:
 * no chunking, blocking or reordering of the recurrence.  The only
 * parallelism is over independent (batch, head, value-column block)
 * problems; each state entry sees the same operations in the same order
 * whatever the split, so the result does not depend on the thread count.
 */
#include <math.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Scan position s (0 .. L-1) -> token index m = y*W + x, per the orders above. */
static long gtr_oracle_token_at(long s, int direction, long H, long W)
{
    long x, y;
    switch (direction) {
    case 0: y = s / W; x = s % W; break;
    case 1: y = s / W; x = W - 1 - (s % W); break;
    case 2: x = s / H; y = s % H; break;
    case 3: x = s / H; y = H - 1 - (s % H); break;
    default: return -1;
    }
    return y * W + x;
}

long gtr_oracle_scan_token(long s, int direction, int H, int W)
{
    if (H <= 0 || W <= 0 || s < 0 || s >= (long)H * (long)W) return -1;
    return gtr_oracle_token_at(s, direction, H, W);
}

/*
 * Returns 0 on success, -1 on a bad argument.  `nthreads` <= 0 lets OpenMP
 * choose; it is ignored when built without OpenMP.
 */
int gtr_oracle_fwd(const double *q, const double *k, const double *v,
                   const double *log_gamma, double *out,
                   int B, int heads, int H, int W, int d_k, int d_v,
                   int direction, int nthreads)
{
    const int CB = 8; /* value columns per independent task */
    if (!q || !k || !v || !log_gamma || !out) return -1;
    if (B <= 0 || heads <= 0 || H <= 0 || W <= 0 || d_k <= 0 || d_v <= 0) return -1;
    if (direction < 0 || direction > 3) return -1;

    const long L = (long)H * (long)W;
    const int nblk = (d_v + CB - 1) / CB;
    const long ntask = (long)B * heads * nblk;
    const double scale = 1.0 / sqrt((double)d_k);
    int failed = 0;

#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : omp_get_max_threads()) reduction(| : failed)
#endif
    for (long task = 0; task < ntask; ++task) {
        const int jb = (int)(task % nblk);
        const int h = (int)((task / nblk) % heads);
        const int b = (int)(task / ((long)nblk * heads));
        const int j0 = jb * CB;
        const int nj = (d_v - j0) < CB ? (d_v - j0) : CB;

        double *S = (double *)calloc((size_t)d_k * CB, sizeof(double));
        if (!S) { failed |= 1; continue; }

        for (long s = 0; s < L; ++s) {
            const long m = gtr_oracle_token_at(s, direction, H, W);
            const long row = ((long)b * L + m) * heads + h;
            const double *qt = q + row * d_k;
            const double *kt = k + row * d_k;
            const double *gt = log_gamma + row * d_k;
            const double *vt = v + row * d_v + j0;
            double *ot = out + row * d_v + j0;

            /* S_t = Diag(gamma_t) S_{t-1} + k_t^T v_t */
            for (int kk = 0; kk < d_k; ++kk) {
                const double g = exp(gt[kk]);
                double *Srow = S + (long)kk * CB;
                for (int j = 0; j < nj; ++j)
                    Srow[j] = g * Srow[j] + kt[kk] * vt[j];
            }
            /* o_t = d_k^{-1/2} q_t S_t */
            for (int j = 0; j < nj; ++j) {
                double acc = 0.0;
                for (int kk = 0; kk < d_k; ++kk)
                    acc += qt[kk] * S[(long)kk * CB + j];
                ot[j] = acc * scale;
            }
        }
        free(S);
    }
    return failed ? -1 : 0;
}

int gtr_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
