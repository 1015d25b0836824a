/*
 * attn_oracle.c -- plain, slow, fp64 CPU oracle for exact scaled-dot-product
 * attention and its gradient.
 *
 * THIS IS TEST INFRASTRUCTURE.  Only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load it.  It shares no code, header,
 * table or helper with the CUDA library; it computes every result from the
 * definitions below, in IEEE double precision, with no tiling, no online
 * softmax and no reordering beyond what the definitions state.
 *
 * Sources (the web pages this method is described on):
 *   [STD]   unite.ai, "Flash Attention: Revolutionizing Transformer
 *           Efficiency" -- the standard-attention definition
 *           softmax(Q K^T / sqrt(d_k)) V, with the (batch, seq, seq) score
 *           tensor materialised.
 *   [SAFE]  same page, "The math behind Flash Attention", item 1: the softmax
 *           of x is exp(x - m) / sum exp(x - m), m = max(x).
 *   [MERGE] same page, same section, item 2: two partial softmaxes are
 *           combined by rescaling each with exp(m_x - m), exp(m_y - m),
 *           m = max(m_x, m_y).  The printed formula is garbled; the reading
 *           implemented in oracle_softmax_merge is stated there.
 *   [RECOMP] same page, "Enter Flash Attention", idea 2: the backward pass
 *           recomputes attention instead of storing it.  The pages print no
 *           backward formulas; oracle_attention_backward is the exact
 *           gradient of [STD].
 *   [CAUSAL] downcodes.com, "triton transformer", usage section: the
 *           `causal = True` (autoregressive) flag.  Reading: square,
 *           top-left aligned -- query i sees keys j <= i.
 *
 * Readings where the pages are silent:
 *   - scale is an explicit argument (the pages fix 1/sqrt(d));
 *   - LSE_i = ln sum_j exp(s_ij) in natural-log units of the SCALED scores;
 *   - masked scores are -inf and contribute exp(-inf) = 0.
 *
 * Inputs are either IEEE doubles (dtype ORACLE_F64) or bfloat16 bit patterns
 * (dtype ORACLE_BF16, widened exactly to double on load).  Layout of every
 * tensor: contiguous [B, H, N, d] (d fastest); LSE is [B, H, N].
 *
 *   [GQA]   same unite.ai page, "FlashAttention-2" item 3: grouped-query and
 *           multi-query attention.  Reading: H query heads share H_kv key/
 *           value heads (H_kv divides H); query head h of a batch attends
 *           with key/value head h / (H / H_kv).  The *_gqa functions take
 *           K, V as [B, H_kv, N, d]; with H_kv = H they are [STD] per head.
 *   [PAD]   downcodes.com "triton transformer", BERT example: a padding
 *           mask over the tokens of each sequence.  Reading: seqlens[b] (0 ..
 *           N) tokens of batch b are real, the rest padding.  Padding keys are
 *           masked for every query; a padding query row has O = 0, LSE = 0
 *           and contributes nothing to any gradient.  Equivalently: batch b is
 *           [STD] on its first seqlens[b] tokens.  seqlens = NULL: all N.
 *
 *   [DROP]  downcodes.com "triton transformer", usage section: the
 *           `attn_dropout = 0.1` option (attention dropout).  The page gives
 *           no formula; reading: inverted dropout on the normalised
 *           probabilities, O_i = sum_j P_ij z_ij / (1 - p) v_j with z_ij in
 *           {0, 1} kept with probability 1 - p; LSE is that of the undropped
 *           scores.  The page gives no random-number convention either:
 *           z_ij comes from the counter-based generator Philox-4x32 (Salmon,
 *           Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3",
 *           SC'11) with 7 rounds (the paper reports Philox-4x32 passing
 *           TestU01's Crush batteries from 7 rounds on; its default of 10
 *           adds a safety margin), called with
 *             counter = (j / 16, i, b * H + h, offset), key = (seed mod 2^32,
 *                       seed / 2^32)
 *           for query i, key j of query head h of batch b (positions counted
 *           from the start of the sequence).  One call gives the 8-bit
 *           numbers of 16 consecutive keys: key j takes word (j mod 16) / 4,
 *           byte 2 (j mod 2) + (j mod 4) / 2 of it (keys 4w, 4w+1, 4w+2,
 *           4w+3 in bytes 0, 2, 1, 3 of word w), and is kept iff
 *           u < t = floor((1 - p) 2^8 + 1/2).  The keep probability is then
 *           q = t / 2^8 (the nearest multiple of 2^-8 to 1 - p) and kept
 *           weights are scaled by 1 / q, so the dropout stays unbiased:
 *             O_i = sum_j P_ij z_ij / q v_j.
 *           t = 2^8 (p < 2^-9) keeps everything; p > 1 - 2^-9 (t = 0) is
 *           rejected.
 *
 * Every function returns 0 on success, -1 on a bad argument, -2 if memory
 * could not be allocated.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_F64 0
#define ORACLE_BF16 1

/* Load element i of an input tensor as a double (bf16 widening is exact). */
static double ld(const void *p, int64_t i, int dtype)
{
    if (dtype == ORACLE_F64)
        return ((const double *)p)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static int bad_shape(int64_t B, int64_t H, int64_t N, int64_t d, int dtype)
{
    return B < 1 || H < 1 || N < 1 || d < 1 ||
           (dtype != ORACLE_F64 && dtype != ORACLE_BF16);
}

/* [PAD]: real tokens of batch b. */
static int64_t seq_len(const int32_t *seqlens, int64_t b, int64_t N)
{
    return seqlens ? seqlens[b] : N;
}

static int bad_seqlens(const int32_t *seqlens, int64_t B, int64_t N)
{
    if (!seqlens)
        return 0;
    for (int64_t b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > N)
            return 1;
    return 0;
}

/*
 * [DROP] Philox-4x32 with R rounds, as the SC'11 paper defines it: each
 * round multiplies counter words 0 and 2 by the constants M0, M1 into 64-bit
 * products (hi, lo), and the new counter is
 *     (hi(M1 c2) ^ c1 ^ k0,  lo(M1 c2),  hi(M0 c0) ^ c3 ^ k1,  lo(M0 c0));
 * between rounds the key is bumped by the Weyl constants W0, W1.
 */
static void philox4x32(const uint32_t ctr[4], const uint32_t key[2], int rounds, uint32_t out[4])
{
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < rounds; ++r) {
        const uint64_t p0 = (uint64_t)M0 * c0, p1 = (uint64_t)M1 * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        c1 = (uint32_t)p1;
        c3 = (uint32_t)p0;
        c0 = n0;
        c2 = n2;
        k0 += W0;
        k1 += W1;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

/* The paper's default, 10 rounds (the form its known-answer vectors cover). */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    philox4x32(ctr, key, 10, out);
}

/* The [DROP] generator: 7 rounds. */
#define DROP_ROUNDS 7
void oracle_philox4x32_7(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    philox4x32(ctr, key, DROP_ROUNDS, out);
}

/* [DROP] parameters; NULL or p == 0 means no dropout. */
struct dropout {
    double p;            /* requested probability of dropping, [0, 1) */
    uint32_t key[2];     /* the seed */
    uint32_t offset;     /* counter word 3 */
    uint32_t threshold;  /* t = floor((1 - p) 2^8 + 1/2): keep iff u < t */
    double keep_scale;   /* 2^8 / t = 1 / (keep probability) */
};

static int make_dropout(struct dropout *dr, double p, uint64_t seed, uint32_t offset)
{
    if (!(p >= 0.0 && p < 1.0))
        return -1;
    const double t = floor((1.0 - p) * 256.0 + 0.5);
    if (t < 1.0)
        return -1;
    dr->p = p;
    dr->key[0] = (uint32_t)seed;
    dr->key[1] = (uint32_t)(seed >> 32);
    dr->offset = offset;
    dr->threshold = (uint32_t)t;
    dr->keep_scale = 256.0 / t;
    return 0;
}

/* z_ij of [DROP] for query i, key j of query head bh = b * H + h. */
static int dropout_keep(const struct dropout *dr, int64_t bh, int64_t i, int64_t j)
{
    const uint32_t ctr[4] = {(uint32_t)(j / 16), (uint32_t)i, (uint32_t)bh, dr->offset};
    uint32_t w[4];
    philox4x32(ctr, dr->key, DROP_ROUNDS, w);
    const uint32_t u = (w[(j % 16) / 4] >> (8 * (2 * (j % 2) + (j % 4) / 2))) & 0xFFu;
    return u < dr->threshold;
}

/* The [DROP] keep mask z as bytes [B, H, N, N] (row = query, column = key). */
int oracle_dropout_keep_mask(int64_t B, int64_t H, int64_t N, double p, uint64_t seed,
                             uint32_t offset, uint8_t *mask)
{
    struct dropout dr;
    if (!mask || B < 1 || H < 1 || N < 1 || make_dropout(&dr, p, seed, offset))
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < B * H * N; ++r)
        for (int64_t j = 0; j < N; ++j)
            mask[r * N + j] = (uint8_t)dropout_keep(&dr, r / N, r % N, j);
    return 0;
}

/* [GQA]: key/value head of query head bh = b * H + h. */
static int64_t kv_head(int64_t bh, int64_t H, int64_t Hkv)
{
    return (bh / H) * Hkv + (bh % H) / (H / Hkv);
}

/*
 * One output row of [STD] for query i over keys j < n_keys (queries of this
 * head start at element q_base, its keys and values at kv_base):
 *   s_j   = scale * <q_i, k_j>           (s_j = -inf if causal and j > i)
 *   m     = max_j s_j                    ([SAFE])
 *   LSE_i = m + ln sum_j exp(s_j - m)
 *   P_j   = exp(s_j - m) / sum_j exp(s_j - m)
 *   O_i   = sum_j P_j v_j                (sum_j P_j z_ij / (1 - p) v_j with [DROP])
 * s is caller-provided scratch of N doubles; bh names the query head for
 * [DROP] (dr = NULL: no dropout).
 */
static void attention_row(const void *Q, const void *K, const void *V, int dtype,
                          int64_t n_keys, int64_t d, int64_t q_base, int64_t kv_base, int64_t i,
                          double scale, int causal, const struct dropout *dr, int64_t bh,
                          double *s, double *o_row, double *lse)
{
    const int64_t N = n_keys;
    for (int64_t j = 0; j < N; ++j) {
        if (causal && j > i) {
            s[j] = -INFINITY;
            continue;
        }
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c)
            acc += ld(Q, q_base + i * d + c, dtype) * ld(K, kv_base + j * d + c, dtype);
        s[j] = scale * acc;
    }
    double m = -INFINITY;
    for (int64_t j = 0; j < N; ++j)
        m = fmax(m, s[j]);
    double sum = 0.0;
    for (int64_t j = 0; j < N; ++j) {
        s[j] = exp(s[j] - m); /* exp(-inf) = 0 for masked keys */
        sum += s[j];
    }
    *lse = m + log(sum);
    for (int64_t c = 0; c < d; ++c)
        o_row[c] = 0.0;
    for (int64_t j = 0; j < N; ++j) {
        double p = s[j] / sum;
        if (dr)
            p = dropout_keep(dr, bh, i, j) ? p * dr->keep_scale : 0.0;
        if (p == 0.0)
            continue;
        for (int64_t c = 0; c < d; ++c)
            o_row[c] += p * ld(V, kv_base + j * d + c, dtype);
    }
}

/* Full forward with [GQA] heads, [PAD] lengths and [DROP] dropout: O
 * [B,H,N,d] and LSE [B,H,N], both double; K, V are [B,Hkv,N,d]; seqlens [B]
 * or NULL; p_drop = 0: no dropout. */
int oracle_attention_forward_dropout(const void *Q, const void *K, const void *V, int dtype,
                                     const int32_t *seqlens, int64_t B, int64_t H, int64_t Hkv,
                                     int64_t N, int64_t d, double scale, int causal,
                                     double p_drop, uint64_t seed, uint32_t offset,
                                     double *O, double *LSE)
{
    struct dropout drop;
    if (!Q || !K || !V || !O || !LSE || bad_shape(B, H, N, d, dtype) ||
        Hkv < 1 || Hkv > H || H % Hkv != 0 || bad_seqlens(seqlens, B, N) ||
        make_dropout(&drop, p_drop, seed, offset))
        return -1;
    const struct dropout *dr = p_drop > 0.0 ? &drop : NULL;
    const int64_t rows = B * H * N;
    int failed = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc((size_t)N * sizeof(double));
        if (!s) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < rows; ++r) {
            if (!s)
                continue;
            const int64_t bh = r / N, i = r % N;
            const int64_t len = seq_len(seqlens, bh / H, N);
            if (i >= len) { /* padding query row */
                for (int64_t c = 0; c < d; ++c)
                    O[r * d + c] = 0.0;
                LSE[r] = 0.0;
                continue;
            }
            attention_row(Q, K, V, dtype, len, d, bh * N * d, kv_head(bh, H, Hkv) * N * d, i,
                          scale, causal, dr, bh, s, O + r * d, LSE + r);
        }
        free(s);
    }
    return failed ? -2 : 0;
}

/* Full forward with [GQA] heads and [PAD] lengths, no dropout. */
int oracle_attention_forward_varlen(const void *Q, const void *K, const void *V, int dtype,
                                    const int32_t *seqlens, int64_t B, int64_t H, int64_t Hkv,
                                    int64_t N, int64_t d, double scale, int causal,
                                    double *O, double *LSE)
{
    return oracle_attention_forward_dropout(Q, K, V, dtype, seqlens, B, H, Hkv, N, d, scale,
                                            causal, 0.0, 0, 0, O, LSE);
}

/* Full forward with [GQA] heads, no padding. */
int oracle_attention_forward_gqa(const void *Q, const void *K, const void *V, int dtype,
                                 int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t d,
                                 double scale, int causal, double *O, double *LSE)
{
    return oracle_attention_forward_varlen(Q, K, V, dtype, NULL, B, H, Hkv, N, d, scale, causal,
                                           O, LSE);
}

/* Full forward, one key/value head per query head. */
int oracle_attention_forward(const void *Q, const void *K, const void *V, int dtype,
                             int64_t B, int64_t H, int64_t N, int64_t d,
                             double scale, int causal, double *O, double *LSE)
{
    return oracle_attention_forward_gqa(Q, K, V, dtype, B, H, H, N, d, scale, causal, O, LSE);
}

/*
 * Forward for a sample of rows only.  rows[k] = bh * N + i names query i of
 * head bh; O_rows is [n_rows, d], LSE_rows is [n_rows].  Each output row of
 * [STD] depends only on its own query and on all keys/values of its head, so
 * a sampled row equals the same row of the full forward.
 */
int oracle_attention_forward_rows(const void *Q, const void *K, const void *V, int dtype,
                                  int64_t B, int64_t H, int64_t N, int64_t d,
                                  double scale, int causal,
                                  const int64_t *rows, int64_t n_rows,
                                  double *O_rows, double *LSE_rows)
{
    if (!Q || !K || !V || !rows || !O_rows || !LSE_rows || n_rows < 0 ||
        bad_shape(B, H, N, d, dtype))
        return -1;
    for (int64_t k = 0; k < n_rows; ++k)
        if (rows[k] < 0 || rows[k] >= B * H * N)
            return -1;
    int failed = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc((size_t)N * sizeof(double));
        if (!s) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t k = 0; k < n_rows; ++k) {
            if (!s)
                continue;
            const int64_t bh = rows[k] / N, i = rows[k] % N;
            attention_row(Q, K, V, dtype, N, d, bh * N * d, bh * N * d, i, scale, causal, NULL,
                          bh, s, O_rows + k * d, LSE_rows + k);
        }
        free(s);
    }
    return failed ? -2 : 0;
}

/*
 * Forward rows with [GQA] heads and [DROP] (no padding): rows[k] = bh * N + i
 * names query i of query head bh.  As oracle_attention_forward_rows, each
 * sampled row equals the same row of oracle_attention_forward_dropout.
 */
int oracle_attention_forward_dropout_rows(const void *Q, const void *K, const void *V, int dtype,
                                          int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t d,
                                          double scale, int causal, double p_drop, uint64_t seed,
                                          uint32_t offset, const int64_t *rows, int64_t n_rows,
                                          double *O_rows, double *LSE_rows)
{
    struct dropout drop;
    if (!Q || !K || !V || !rows || !O_rows || !LSE_rows || n_rows < 0 ||
        bad_shape(B, H, N, d, dtype) || Hkv < 1 || Hkv > H || H % Hkv != 0 ||
        make_dropout(&drop, p_drop, seed, offset))
        return -1;
    for (int64_t k = 0; k < n_rows; ++k)
        if (rows[k] < 0 || rows[k] >= B * H * N)
            return -1;
    const struct dropout *dr = p_drop > 0.0 ? &drop : NULL;
    int failed = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc((size_t)N * sizeof(double));
        if (!s) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t k = 0; k < n_rows; ++k) {
            if (!s)
                continue;
            const int64_t bh = rows[k] / N, i = rows[k] % N;
            attention_row(Q, K, V, dtype, N, d, bh * N * d, kv_head(bh, H, Hkv) * N * d, i, scale,
                          causal, dr, bh, s, O_rows + k * d, LSE_rows + k);
        }
        free(s);
    }
    return failed ? -2 : 0;
}

/*
 * Exact gradient of [STD] (with [GQA] heads) for upstream gradient dO, one
 * query head at a time,
 * with the full N x N matrices P, dP and dS materialised ([RECOMP] says only
 * that the fast path recomputes instead of storing; the oracle stores).
 *   P_ij  = softmax_j(s_ij)                  (row i, masked keys give 0)
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = <dO_i, v_j>
 *   D_i   = sum_j P_ij dP_ij
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale sum_j dS_ij k_j
 *   dK_j  = scale sum_i dS_ij q_i
 * With [GQA] heads the key/value gradients of a key/value head are the sums
 * of these over the query heads that share it.  With [PAD] lengths each
 * (batch, head) is the same on its first len tokens (P = 0 outside) and all
 * gradients of padding tokens are 0.  With [DROP] the output is
 * O_i = sum_j Pd_ij v_j, Pd_ij = P_ij z_ij / q, and by the chain rule
 *   dV_j  = sum_i Pd_ij dO_i
 *   dP_ij = <dO_i, v_j> z_ij / q             (gradient with respect to P)
 * with D, dS, dQ, dK as above (D_i = sum_j P_ij dP_ij still equals
 * <dO_i, O_i>).  dQ is double [B,H,N,d]; dK, dV are double [B,Hkv,N,d].
 */
static int backward_impl(const void *Q, const void *K, const void *V, const void *dO, int dtype,
                         const int32_t *seqlens, int64_t B, int64_t H, int64_t Hkv, int64_t N,
                         int64_t d, double scale, int causal, double p_drop, uint64_t seed,
                         uint32_t offset, const int64_t *heads, int64_t n_heads,
                         double *dQ, double *dK, double *dV)
{
    struct dropout drop;
    if (!Q || !K || !V || !dO || !dQ || !dK || !dV || bad_shape(B, H, N, d, dtype) ||
        Hkv < 1 || Hkv > H || H % Hkv != 0 || bad_seqlens(seqlens, B, N) ||
        make_dropout(&drop, p_drop, seed, offset))
        return -1;
    if (heads) { /* distinct query heads in range */
        if (n_heads < 0)
            return -1;
        for (int64_t a = 0; a < n_heads; ++a) {
            if (heads[a] < 0 || heads[a] >= B * H)
                return -1;
            for (int64_t b = 0; b < a; ++b)
                if (heads[b] == heads[a])
                    return -1;
        }
    }
    const struct dropout *dr = p_drop > 0.0 ? &drop : NULL;
    double *P = (double *)malloc((size_t)N * (size_t)N * sizeof(double));
    double *dS = (double *)malloc((size_t)N * (size_t)N * sizeof(double));
    /* z_ij / q of the current head (only with dropout) */
    double *Z = dr ? (double *)malloc((size_t)N * (size_t)N * sizeof(double)) : NULL;
    if (!P || !dS || (dr && !Z)) {
        free(P);
        free(dS);
        free(Z);
        return -2;
    }
    for (int64_t e = 0; e < B * Hkv * N * d; ++e) {
        dK[e] = 0.0;
        dV[e] = 0.0;
    }
    for (int64_t e = 0; e < B * H * N * d; ++e)
        dQ[e] = 0.0;
    for (int64_t hi = 0; hi < (heads ? n_heads : B * H); ++hi) {
        const int64_t bh = heads ? heads[hi] : hi;
        const int64_t base = bh * N * d;                        /* Q, dO, dQ */
        const int64_t kv_base = kv_head(bh, H, Hkv) * N * d;    /* K, V, dK, dV */
        const int64_t N_full = N;
        const int64_t N = seq_len(seqlens, bh / H, N_full);     /* real tokens */
        /* P row by row, exactly as the forward defines it. */
#pragma omp parallel for schedule(dynamic, 8)
        for (int64_t i = 0; i < N; ++i) {
            double *s = P + i * N;
            for (int64_t j = 0; j < N; ++j) {
                if (causal && j > i) {
                    s[j] = -INFINITY;
                    continue;
                }
                double acc = 0.0;
                for (int64_t c = 0; c < d; ++c)
                    acc += ld(Q, base + i * d + c, dtype) * ld(K, kv_base + j * d + c, dtype);
                s[j] = scale * acc;
            }
            double m = -INFINITY;
            for (int64_t j = 0; j < N; ++j)
                m = fmax(m, s[j]);
            double sum = 0.0;
            for (int64_t j = 0; j < N; ++j) {
                s[j] = exp(s[j] - m);
                sum += s[j];
            }
            for (int64_t j = 0; j < N; ++j)
                s[j] /= sum;
            if (dr)
                for (int64_t j = 0; j < N; ++j)
                    Z[i * N + j] = dropout_keep(dr, bh, i, j) ? dr->keep_scale : 0.0;
        }
        /* dP, D and dS. */
#pragma omp parallel for schedule(dynamic, 8)
        for (int64_t i = 0; i < N; ++i) {
            double *ds = dS + i * N;
            for (int64_t j = 0; j < N; ++j) {
                double acc = 0.0;
                for (int64_t c = 0; c < d; ++c)
                    acc += ld(dO, base + i * d + c, dtype) * ld(V, kv_base + j * d + c, dtype);
                ds[j] = dr ? acc * Z[i * N + j] : acc; /* dP_ij */
            }
            double D = 0.0;
            for (int64_t j = 0; j < N; ++j)
                D += P[i * N + j] * ds[j];
            for (int64_t j = 0; j < N; ++j)
                ds[j] = P[i * N + j] * (ds[j] - D);
        }
        /* dQ_i = scale sum_j dS_ij k_j */
#pragma omp parallel for schedule(dynamic, 8)
        for (int64_t i = 0; i < N; ++i) {
            for (int64_t c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int64_t j = 0; j < N; ++j)
                    acc += dS[i * N + j] * ld(K, kv_base + j * d + c, dtype);
                dQ[base + i * d + c] = scale * acc;
            }
        }
        /* dK_j = scale sum_i dS_ij q_i ;  dV_j = sum_i P_ij dO_i */
#pragma omp parallel for schedule(dynamic, 8)
        for (int64_t j = 0; j < N; ++j) {
            for (int64_t c = 0; c < d; ++c) {
                double acc_k = 0.0, acc_v = 0.0;
                for (int64_t i = 0; i < N; ++i) {
                    const double pd = dr ? P[i * N + j] * Z[i * N + j] : P[i * N + j];
                    acc_k += dS[i * N + j] * ld(Q, base + i * d + c, dtype);
                    acc_v += pd * ld(dO, base + i * d + c, dtype);
                }
                dK[kv_base + j * d + c] += scale * acc_k;
                dV[kv_base + j * d + c] += acc_v;
            }
        }
    }
    free(P);
    free(dS);
    free(Z);
    return 0;
}

/* The backward of [STD] with [GQA], [PAD] and [DROP]: see backward_impl. */
int oracle_attention_backward_dropout(const void *Q, const void *K, const void *V,
                                      const void *dO, int dtype, const int32_t *seqlens,
                                      int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t d,
                                      double scale, int causal, double p_drop, uint64_t seed,
                                      uint32_t offset, double *dQ, double *dK, double *dV)
{
    return backward_impl(Q, K, V, dO, dtype, seqlens, B, H, Hkv, N, d, scale, causal, p_drop,
                         seed, offset, NULL, 0, dQ, dK, dV);
}

/*
 * The same for the listed query heads only (distinct, each bh = b * H + h):
 * dQ rows of those heads; dK, dV of a K/V head summed over the listed query
 * heads of its group; everything else 0.  Each head's gradient depends only
 * on that head, so with one query head per K/V head this equals the full
 * backward on the listed heads.  For checking large shapes a head at a time.
 */
int oracle_attention_backward_dropout_heads(const void *Q, const void *K, const void *V,
                                            const void *dO, int dtype, int64_t B, int64_t H,
                                            int64_t Hkv, int64_t N, int64_t d, double scale,
                                            int causal, double p_drop, uint64_t seed,
                                            uint32_t offset, const int64_t *heads,
                                            int64_t n_heads, double *dQ, double *dK, double *dV)
{
    if (!heads)
        return -1;
    return backward_impl(Q, K, V, dO, dtype, NULL, B, H, Hkv, N, d, scale, causal, p_drop, seed,
                         offset, heads, n_heads, dQ, dK, dV);
}

/* Backward with [GQA] heads and [PAD] lengths, no dropout. */
int oracle_attention_backward_varlen(const void *Q, const void *K, const void *V,
                                     const void *dO, int dtype, const int32_t *seqlens,
                                     int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t d,
                                     double scale, int causal,
                                     double *dQ, double *dK, double *dV)
{
    return oracle_attention_backward_dropout(Q, K, V, dO, dtype, seqlens, B, H, Hkv, N, d, scale,
                                             causal, 0.0, 0, 0, dQ, dK, dV);
}

/* Backward with [GQA] heads, no padding. */
int oracle_attention_backward_gqa(const void *Q, const void *K, const void *V, const void *dO,
                                  int dtype, int64_t B, int64_t H, int64_t Hkv, int64_t N,
                                  int64_t d, double scale, int causal,
                                  double *dQ, double *dK, double *dV)
{
    return oracle_attention_backward_varlen(Q, K, V, dO, dtype, NULL, B, H, Hkv, N, d, scale,
                                            causal, dQ, dK, dV);
}

/* Backward with one key/value head per query head. */
int oracle_attention_backward(const void *Q, const void *K, const void *V, const void *dO,
                              int dtype, int64_t B, int64_t H, int64_t N, int64_t d,
                              double scale, int causal, double *dQ, double *dK, double *dV)
{
    return oracle_attention_backward_gqa(Q, K, V, dO, dtype, B, H, H, N, d, scale, causal,
                                         dQ, dK, dV);
}

/*
 * [SAFE] applied to one block of scores: for scores s[0..n) and value rows
 * Vblk [n, d] (double), returns the block's max m, its sum
 * l = sum exp(s - m), and the block-normalised output
 * o = sum_j exp(s_j - m) v_j / l.  Used only to test [MERGE].
 */
int oracle_softmax_partial(const double *s, int64_t n, const double *Vblk, int64_t d,
                           double *m, double *l, double *o)
{
    if (!s || !Vblk || !m || !l || !o || n < 1 || d < 1)
        return -1;
    double mx = -INFINITY;
    for (int64_t j = 0; j < n; ++j)
        mx = fmax(mx, s[j]);
    double sum = 0.0;
    for (int64_t j = 0; j < n; ++j)
        sum += exp(s[j] - mx);
    for (int64_t c = 0; c < d; ++c)
        o[c] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        const double w = exp(s[j] - mx) / sum;
        for (int64_t c = 0; c < d; ++c)
            o[c] += w * Vblk[j * d + c];
    }
    *m = mx;
    *l = sum;
    return 0;
}

/*
 * [MERGE], read as: with m = max(m_x, m_y),
 *   l = exp(m_x - m) l_x + exp(m_y - m) l_y
 *   o = (exp(m_x - m) l_x o_x + exp(m_y - m) l_y o_y) / l
 * where o_x, o_y are the block-normalised partial outputs.  The result is the
 * softmax-weighted output over the union of both blocks.
 */
int oracle_softmax_merge(double m_x, double l_x, const double *o_x,
                         double m_y, double l_y, const double *o_y, int64_t d,
                         double *m, double *l, double *o)
{
    if (!o_x || !o_y || !m || !l || !o || d < 1)
        return -1;
    const double mm = fmax(m_x, m_y);
    const double a = exp(m_x - mm) * l_x;
    const double b = exp(m_y - mm) * l_y;
    const double ll = a + b;
    for (int64_t c = 0; c < d; ++c)
        o[c] = (a * o_x[c] + b * o_y[c]) / ll;
    *m = mm;
    *l = ll;
    return 0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}
