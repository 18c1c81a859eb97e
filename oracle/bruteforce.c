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
#include <math.h>
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

/*
 * The same brute force for the rotary form (3D RoPE on the numerator; the normaliser unturned),
 * written through relative angles instead of turned vectors: for a feature pair p with
 * (a, c) = (relu(q_i,2p), relu(q_i,2p+1)) and (b, d) = (relu(k_j,2p), relu(k_j,2p+1)),
 *   (R_i (a, c)) . (R_j (b, d)) = (a b + c d) cos(t_jp - t_ip) + (c b - a d) sin(t_jp - t_ip),
 * with t_np = ang[n][p] the angle of pair p at token n (ang [N][D/2], the same for every slice):
 *   num_ie = sum_j M_ij (sum_p that score) v_je,   den_i = sum_j M_ij (sum_d relu(q_id) relu(k_jd)),
 *   o_ie = num_ie / (den_i + eps).
 * D must be even.
 */
void oracle_bruteforce_rope(const double *q, const double *k, const double *v, const double *ang, double *o,
                            int BH, int N, int D, int E, int block_len, double eps)
{
    const int P = D / 2;
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
                double s = 0.0, a_den = 0.0;
                for (int p = 0; p < P; ++p) {
                    double a = relu(Q[(size_t)i * D + 2 * p]), c = relu(Q[(size_t)i * D + 2 * p + 1]);
                    double b = relu(K[(size_t)j * D + 2 * p]), d = relu(K[(size_t)j * D + 2 * p + 1]);
                    double dt = ang[(size_t)j * P + p] - ang[(size_t)i * P + p];
                    s += (a * b + c * d) * cos(dt) + (c * b - a * d) * sin(dt);
                    a_den += a * b + c * d;
                }
                den += a_den;
                for (int e = 0; e < E; ++e) O[(size_t)i * E + e] += s * V[(size_t)j * E + e];
            }
            for (int e = 0; e < E; ++e) O[(size_t)i * E + e] /= (den + eps);
        }
    }
}
