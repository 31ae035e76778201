/*
 * Plain fp64 CPU oracle for exact softmax attention, forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg use it. It shares no code, header or constant with the CUDA library.
 *
 * What it computes is the textbook definition, with every N x N matrix
 * materialised in fp64, in the order the definition states it:
 *
 *   S = scale * Q K^T                         (page "PyTorch-CUDA-v2.9镜像中使用FlashAttention
 *                                              提升训练速度", the Attention(Q,K,V) formula;
 *                                              page "告别OOM和训练慢…(含A100环境配置)" §1, the
 *                                              three-line PyTorch implementation)
 *   S_ij += -m_h |i - j|  when per-head ALiBi slopes m_h are given (the linear bias
 *          `alibi_slopes` of `flash_attn_fn`, page "告别OOM和训练慢…" §4.2)
 *   S_ij = -inf where key j is not visible from query i (causal: "mask future
 *          positions", page "Flash Attention 3.7 核心原理与实战" §3.2; sliding window
 *          `window_size=(left,right)`, page "告别OOM和训练慢…" §4.2), and where key j of
 *          the batch entry is padding (`key_padding_mask`, True = padded: the attention
 *          layer of page "PyTorch-CUDA-v2.9镜像…" accepts it, and the reference layer of page
 *          "Flash Attention 3.7 核心原理与实战" §4.2 applies it with masked_fill(-inf),
 *          broadcast over every head and query)
 *   P = row-softmax(S), with the row maximum subtracted first (`safe_softmax`,
 *       page "告别OOM和训练慢…" §2.2)
 *   O = P V
 *   LSE_i = m_i + ln sum_j exp(S_ij - m_i)    (the per-row normalisation factor the
 *                                              forward keeps for the backward, same page §2.2)
 *
 * The pages print no backward; the backward here is the chain rule of the above
 * for the scalar L = <O, dO> (the "recompute P" backward of page
 * "告别OOM和训练慢…" §2.2 and the recomputation paragraph of page
 * "PyTorch-CUDA-v2.9镜像…", restated from the definition):
 *   dV = P^T dO;  dP = dO V^T;  D_i = sum_j P_ij dP_ij;  dS = P o (dP - D);
 *   dQ = scale * dS K;  dK = scale * dS^T Q.
 *
 * Variable-length batches (`lengths`: each sample's real length, the dynamic batching of
 * page "告别OOM和训练慢…" §6, which groups sequences by length to avoid computing on
 * padding): batch entry b holds L_b real tokens; query i and key j of that entry interact
 * only if i < L_b and j < L_b (on top of the mask). Rows i >= L_b see no key (O = 0,
 * LSE = -inf, no gradient) and keys j >= L_b get none.
 *
 * Dropout on the attention weights (`dropout_p` of `flash_attn_fn`, page "告别OOM和训练慢…"
 * §4.2; the reference layer of page "Flash Attention 3.7 核心原理与实战" §4.2 applies
 * F.dropout to the softmax weights and then multiplies by V): with keep flags Z_ij,
 *   O = (P o Z / (1 - p)) V, and LSE is that of P (dropout comes after the softmax).
 * Backward (chain rule): dV = (P o Z / (1-p))^T dO; dP~ = (dO V^T) o Z / (1-p);
 *   D_i = sum_j P_ij dP~_ij (= rowsum(dO o O)); dS = P o (dP~ - D); dQ, dK as above.
 * The pages do not say how the keep flags are drawn; they are drawn here, as in the GPU
 * kernels, from the counter-based generator Philox4x32-10 (Salmon, Moraes, Dror and Shaw,
 * "Parallel random numbers: as easy as 1, 2, 3", SC 2011), written out below from that
 * paper's definition:
 *   - key (k0, k1) = the low and high 32 bits of the seed;
 *   - counter (c0, c1, c2, c3) = (floor(j / 16), i, b*H + h, offset) for query i, key j;
 *   - key j uses byte (j mod 4) (least significant first) of output word (j mod 16) / 4;
 *   - with t = floor(256 p + 1/2), the weight is dropped iff that byte < t, and kept
 *     weights are scaled by 256 / (256 - t), i.e. by 1 / (1 - p') with p' = t / 256 the
 *     probability the generator really drops with (p is rounded to a multiple of 1/256).
 *
 * Readings where the pages are silent:
 *   - visible(i, j) <=> (left < 0 or j >= i - left) and (right < 0 or j <= i + right);
 *     -1 means unbounded; causal forces right = min(right, 0) (right = 0 when unbounded).
 *   - a row with no visible key has P_i = 0, O_i = 0, LSE_i = -inf, and adds nothing
 *     to any gradient.
 *   - ALiBi (the page names the parameter and calls it a linear bias, nothing more): a
 *     slope m_h per head, the bias -m_h |i - j| added to the scaled score; it is a
 *     constant of the scores, so the backward formulas are unchanged.
 *
 * Layout: every tensor is (B, H, N, d) row-major fp64; lse is (B, H, N).
 * Loops over rows are shared out with OpenMP; each output element is still
 * summed in plain index order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int resolve_right(int causal, long right)
{
    if (causal) {
        if (right < 0 || right > 0) return 0;
    }
    return (int)right;
}

static int visible(long i, long j, long left, long right)
{
    if (left >= 0 && j < i - left) return 0;
    if (right >= 0 && j > i + right) return 0;
    return 1;
}

/* The ALiBi slope of head bh (of B*H, heads fastest): 0 without slopes. */
static double head_slope(const double *alibi_slopes, long bh, long H)
{
    return alibi_slopes ? alibi_slopes[bh % H] : 0.0;
}

/* P (N x N) := softmax rows of the masked, scaled (and biased, when slope != 0) scores of
 * one head; lse (N). kpad: N flags of the head's batch entry (nonzero = padded key), or
 * NULL; len: the entry's real length (N when the batch is not variable-length). */
static void head_probabilities(const double *q, const double *k, long N, long d,
                               double scale, double slope, long left, long right,
                               const unsigned char *kpad, long len, double *P, double *lse)
{
    long i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < N; ++i) {
        double *Pi = P + i * N;
        double m = -INFINITY;
        long j, c;
        for (j = 0; j < N; ++j) {
            double s = 0.0;
            for (c = 0; c < d; ++c) s += q[i * d + c] * k[j * d + c];
            s *= scale;
            s += -slope * fabs((double)(i - j));
            if (!visible(i, j, left, right)) s = -INFINITY;
            if (kpad && kpad[j]) s = -INFINITY;
            if (i >= len || j >= len) s = -INFINITY;
            Pi[j] = s;
            if (s > m) m = s;
        }
        if (m == -INFINITY) {
            for (j = 0; j < N; ++j) Pi[j] = 0.0;
            lse[i] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (j = 0; j < N; ++j) {
            Pi[j] = exp(Pi[j] - m);
            sum += Pi[j];
        }
        for (j = 0; j < N; ++j) Pi[j] /= sum;
        lse[i] = m + log(sum);
    }
}

/* Philox4x32-10 (Salmon et al., SC 2011): ten rounds of the Philox S-box on the 4-word
 * counter, the 2-word key bumped by the Weyl constants between rounds. One round maps
 * (c0, c1, c2, c3) to (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2), hi(M0*c0) ^ c3 ^ k1, lo(M0*c0)). */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    int r;
    for (r = 0; r < 10; ++r) {
        uint64_t p0, p1;
        uint32_t n0, n1, n2, n3;
        if (r > 0) {
            k0 += W0;
            k1 += W1;
        }
        p0 = (uint64_t)M0 * c0;
        p1 = (uint64_t)M1 * c2;
        n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        n1 = (uint32_t)p1;
        n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        n3 = (uint32_t)p0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Drop threshold on a byte: t = floor(256 p + 1/2). */
static int dropout_threshold(double p)
{
    return (int)floor(256.0 * p + 0.5);
}

/* 1 if the weight of query i on key j of head bh is kept, 0 if dropped. */
static int dropout_keep(unsigned long long seed, unsigned long long offset, long bh, long i,
                        long j, int t)
{
    uint32_t ctr[4], key[2], out[4];
    unsigned byte;
    if (t <= 0) return 1;
    ctr[0] = (uint32_t)(j / 16);
    ctr[1] = (uint32_t)i;
    ctr[2] = (uint32_t)bh;
    ctr[3] = (uint32_t)offset;
    key[0] = (uint32_t)seed;
    key[1] = (uint32_t)(seed >> 32);
    oracle_philox4x32_10(ctr, key, out);
    byte = (out[(j % 16) / 4] >> (8 * (j % 4))) & 0xFFu;
    return (int)byte >= t ? 1 : 0;
}

/* The keep flags of head bh (N x N, row = query), for tests. */
int oracle_dropout_mask(unsigned long long seed, unsigned long long offset, long bh, long N,
                        double dropout_p, unsigned char *mask)
{
    long i, j;
    const int t = dropout_threshold(dropout_p);
    if (t < 0 || t > 255) return 1;
    for (i = 0; i < N; ++i)
        for (j = 0; j < N; ++j) mask[i * N + j] = (unsigned char)dropout_keep(seed, offset, bh, i, j, t);
    return 0;
}

/* P := P o Z / (1 - p') in place (one head): the weights the forward multiplies V by. */
static void apply_dropout(double *P, long N, long bh, double dropout_p, unsigned long long seed,
                          unsigned long long offset)
{
    const int t = dropout_threshold(dropout_p);
    const double keep_scale = 256.0 / (256.0 - t);
    long i;
    if (t <= 0) return;
#pragma omp parallel for schedule(static)
    for (i = 0; i < N; ++i) {
        long j;
        for (j = 0; j < N; ++j)
            P[i * N + j] = dropout_keep(seed, offset, bh, i, j, t) ? P[i * N + j] * keep_scale : 0.0;
    }
}

/* The real length of head bh's batch entry: lengths[b], or N without lengths. */
static long head_length(const long *lengths, long bh, long H, long N)
{
    return lengths ? lengths[bh / H] : N;
}

/* The key-padding flags of head bh's batch entry (B*H heads, heads fastest), or NULL. */
static const unsigned char *head_padding(const unsigned char *key_padding, long bh, long H,
                                         long N)
{
    return key_padding ? key_padding + (bh / H) * N : NULL;
}

/* alibi_slopes: H slopes, or NULL for no bias; key_padding: B x N flags (nonzero = padded
 * key), or NULL for none; lengths: B real lengths in [0, N], or NULL; dropout_p in [0, 1),
 * 0 for none, with its seed and offset. */
int oracle_attention_fwd(const double *q, const double *k, const double *v,
                         long B, long H, long N, long d, double scale,
                         int causal, long left, long right, const double *alibi_slopes,
                         const unsigned char *key_padding, const long *lengths,
                         double dropout_p, unsigned long long seed, unsigned long long offset,
                         double *o, double *lse)
{
    long bh;
    if (B < 0 || H < 0 || N < 0 || d < 1) return 1;
    if (dropout_threshold(dropout_p) < 0 || dropout_threshold(dropout_p) > 255) return 1;
    right = resolve_right(causal, right);
    double *P = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1) * (size_t)(N > 0 ? N : 1));
    if (!P) return 2;
    for (bh = 0; bh < B * H; ++bh) {
        const double *qh = q + bh * N * d, *kh = k + bh * N * d, *vh = v + bh * N * d;
        double *oh = o + bh * N * d;
        long i;
        head_probabilities(qh, kh, N, d, scale, head_slope(alibi_slopes, bh, H), left, right,
                           head_padding(key_padding, bh, H, N),
                           head_length(lengths, bh, H, N), P, lse + bh * N);
        apply_dropout(P, N, bh, dropout_p, seed, offset);
        /* O = P V (P with dropout applied) */
#pragma omp parallel for schedule(static)
        for (i = 0; i < N; ++i) {
            long j, c;
            for (c = 0; c < d; ++c) oh[i * d + c] = 0.0;
            for (j = 0; j < N; ++j) {
                double p = P[i * N + j];
                for (c = 0; c < d; ++c) oh[i * d + c] += p * vh[j * d + c];
            }
        }
    }
    free(P);
    return 0;
}

int oracle_attention_bwd(const double *q, const double *k, const double *v,
                         const double *dout,
                         long B, long H, long N, long d, double scale,
                         int causal, long left, long right, const double *alibi_slopes,
                         const unsigned char *key_padding, const long *lengths,
                         double dropout_p, unsigned long long seed, unsigned long long offset,
                         double *dq, double *dk, double *dv)
{
    long bh;
    if (B < 0 || H < 0 || N < 0 || d < 1) return 1;
    if (dropout_threshold(dropout_p) < 0 || dropout_threshold(dropout_p) > 255) return 1;
    const int t = dropout_threshold(dropout_p);
    const double keep_scale = t > 0 ? 256.0 / (256.0 - t) : 1.0;
    right = resolve_right(causal, right);
    size_t nn = (size_t)(N > 0 ? N : 1) * (size_t)(N > 0 ? N : 1);
    double *P = (double *)malloc(sizeof(double) * nn);
    double *Pd = (double *)malloc(sizeof(double) * nn);
    double *dP = (double *)malloc(sizeof(double) * nn);
    double *lse = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    double *D = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    if (!P || !Pd || !dP || !lse || !D) {
        free(P); free(Pd); free(dP); free(lse); free(D);
        return 2;
    }
    for (bh = 0; bh < B * H; ++bh) {
        const double *qh = q + bh * N * d, *kh = k + bh * N * d, *vh = v + bh * N * d;
        const double *doh = dout + bh * N * d;
        double *dqh = dq + bh * N * d, *dkh = dk + bh * N * d, *dvh = dv + bh * N * d;
        long i, j;
        head_probabilities(qh, kh, N, d, scale, head_slope(alibi_slopes, bh, H), left, right,
                           head_padding(key_padding, bh, H, N),
                           head_length(lengths, bh, H, N), P, lse);
        /* Pd = P o Z / (1 - p'): the weights that multiplied V (Pd = P without dropout) */
        memcpy(Pd, P, sizeof(double) * (size_t)N * (size_t)N);
        apply_dropout(Pd, N, bh, dropout_p, seed, offset);
        /* dV = Pd^T dO */
#pragma omp parallel for schedule(static)
        for (j = 0; j < N; ++j) {
            long ii, c;
            for (c = 0; c < d; ++c) dvh[j * d + c] = 0.0;
            for (ii = 0; ii < N; ++ii) {
                double p = Pd[ii * N + j];
                for (c = 0; c < d; ++c) dvh[j * d + c] += p * doh[ii * d + c];
            }
        }
        /* dP~ = (dO V^T) o Z / (1 - p') ; D_i = sum_j P_ij dP~_ij ; dS = P o (dP~ - D),
         * stored over dP */
#pragma omp parallel for schedule(static)
        for (i = 0; i < N; ++i) {
            long jj, c;
            double acc = 0.0;
            for (jj = 0; jj < N; ++jj) {
                double s = 0.0, zs;
                for (c = 0; c < d; ++c) s += doh[i * d + c] * vh[jj * d + c];
                zs = dropout_keep(seed, offset, bh, i, jj, t) ? keep_scale : 0.0;
                dP[i * N + jj] = s * zs;
                acc += P[i * N + jj] * dP[i * N + jj];
            }
            D[i] = acc;
            for (jj = 0; jj < N; ++jj) dP[i * N + jj] = P[i * N + jj] * (dP[i * N + jj] - D[i]);
        }
        /* dQ = scale * dS K */
#pragma omp parallel for schedule(static)
        for (i = 0; i < N; ++i) {
            long jj, c;
            for (c = 0; c < d; ++c) dqh[i * d + c] = 0.0;
            for (jj = 0; jj < N; ++jj) {
                double s = dP[i * N + jj];
                for (c = 0; c < d; ++c) dqh[i * d + c] += s * kh[jj * d + c];
            }
            for (c = 0; c < d; ++c) dqh[i * d + c] *= scale;
        }
        /* dK = scale * dS^T Q */
#pragma omp parallel for schedule(static)
        for (j = 0; j < N; ++j) {
            long ii, c;
            for (c = 0; c < d; ++c) dkh[j * d + c] = 0.0;
            for (ii = 0; ii < N; ++ii) {
                double s = dP[ii * N + j];
                for (c = 0; c < d; ++c) dkh[j * d + c] += s * qh[ii * d + c];
            }
            for (c = 0; c < d; ++c) dkh[j * d + c] *= scale;
        }
    }
    free(P); free(Pd); free(dP); free(lse); free(D);
    return 0;
}

/* Number of OpenMP threads the loops above use (for reporting the CPU baseline). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
