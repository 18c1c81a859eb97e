/*
 * Plain C brute force of block-causal ReLU-kernel linear attention, in double precision.
 *
 * TEST INFRASTRUCTURE ONLY: used to pin the numpy oracle; never linked into the CUDA library.
 *
 * It evaluates the quadratic definition directly, with no state and no blocking:
 *   A_ij = sum_d max(q_id, 0) * max(k_jd, 0)
 *   M_ij = 1 if floor(j / L) <= floor(i / L), else 0   (L >= N: all ones, the bidirectional form)
 *   o_ie = sum_j M_ij A_ij v_je / (sum_j M_ij A_ij + eps)
 * for each of BH independent (batch, head) slices. Layout: q, k [BH][N][D], v, o [BH][N][E].
 * The block structure (a block sees itself and every earlier block) is the block-causal linear
 * attention of the SANA-Video talk (block KV cache passage) written as a mask.
 */
#include <stddef.h>

static double relu(double x) { return x > 0.0 ? x : 0.0; }

void oracle_bruteforce(const double *q, const double *k, const double *v, double *o,
                       int BH, int N, int D, int E, int block_len, double eps)
{
    for (int bh = 0; bh < BH; ++bh) {
        const double *Q = q + (size_t)bh * N * D;
        const double *K = k + (size_t)bh * N * D;
        const double *V = v + (size_t)bh * N * E;
        double *O = o + (size_t)bh * N * E;
        for (int i = 0; i < N; ++i) {
            int bi = i / block_len;
            double den = 0.0;
            for (int e = 0; e < E; ++e) O[(size_t)i * E + e] = 0.0;
            for (int j = 0; j < N; ++j) {
                if (j / block_len > bi) continue;
                double a = 0.0;
                for (int d = 0; d < D; ++d)
                    a += relu(Q[(size_t)i * D + d]) * relu(K[(size_t)j * D + d]);
                den += a;
                for (int e = 0; e < E; ++e) O[(size_t)i * E + e] += a * V[(size_t)j * E + e];
            }
            for (int e = 0; e < E; ++e) O[(size_t)i * E + e] /= (den + eps);
        }
    }
}
