/*
 * CPU oracle for split-KV (replicated prefix + suffix) tail-padded attention
 * and for the fused Q/K RMSNorm + RoPE prologue.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA path, and it never calls it.
 *
 * Plain C, fp64 arithmetic, OpenMP over independent (batch, query row, head)
 * items.  No blocking, no online softmax, no reordering: every output is the
 * textbook definition written out.  Build: gcc -O2 -fopenmp -ffp-contract=off
 * (no -ffast-math) so the summation order below is the order executed.
 *
 * Sources (the pages the method comes from):
 *  - "sglang PR 26973" (Cosmos3 split K/V prefix), layer.py listing of
 *    forward_with_replicated_kv_prefix: the non-sequence-parallel branch
 *    concatenates the K/V prefix and suffix along the sequence axis (prefix
 *    first) and runs ordinary attention over the result.  That is what
 *    oracle_attn_split_kv computes, with the concatenation done by indexing.
 *  - "sglang PR 30107" (unified SP shard utils), sp_shard_utils.py listing:
 *    padding is one contiguous block at the global tail; tail_attn_meta's
 *    valid_len says how many leading tokens are real.  Keys at positions
 *    >= real_len[b] are excluded from the softmax.
 *  - "vLLM-Omni performance patterns", shared Attention wiring: BSND layout,
 *    softmax_scale = head_dim ** -0.5, causal=False, GQA with
 *    num_heads % num_kv_heads == 0.
 *  - "vLLM-Omni performance patterns", Q/K RMSNorm + RoPE section and the
 *    materialisation rule (round to bf16 wherever the unfused path stores
 *    bf16): oracle_qk_rmsnorm_rope.
 *
 * Readings where the pages are silent:
 *  - GQA: query head hq reads KV head hq / (Hq / Hkv) (contiguous groups).
 *  - Query rows i >= q_valid[b] are pad; their output is exactly 0.
 *  - A row with no valid key (real_len[b] == 0) outputs exactly 0.
 *  - Softmax uses the natural exponential of scale * <q, k>.
 *
 * All tensors are contiguous, row-major, bf16 passed as raw uint16 bits:
 *   q        [B, Sq, Hq, D]
 *   k/v pref [B, Sp, Hkv, D]
 *   k/v suff [B, Ss, Hkv, D]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Planted mistakes for the pin tests (0 = the definition). */
enum {
    MUT_NONE = 0,
    MUT_GQA_MODULO = 1,         /* hkv = hq % Hkv instead of hq / g          */
    MUT_ONE_PAD_KEY = 2,        /* includes key real_len[b] (one pad key)    */
    MUT_V_FROM_K = 3,           /* value rows read from the K tensors        */
    MUT_DROP_LAST_IN_SUM = 4,   /* normaliser l omits the last key's term    */
    MUT_NEGATED_SCORES = 5,     /* s_j = -scale * <q, k_j>                   */
    MUT_SCALE_IGNORED = 6,      /* scale treated as 1                        */
    MUT_DROP_LAST_DIM = 7,      /* dot product over d < D - 1                */
    MUT_Q_FROM_KV_HEAD = 8      /* query row read from head hkv, not hq      */
};

static double bf16_bits_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Key row j of the virtual concatenation cat(prefix, suffix) for (b, hkv). */
static const uint16_t *kv_row(const uint16_t *pre, const uint16_t *suf,
                              int b, int j, int hkv,
                              int Sp, int Ss, int Hkv, int D)
{
    if (j < Sp)
        return pre + (((int64_t)b * Sp + j) * Hkv + hkv) * D;
    return suf + (((int64_t)b * Ss + (j - Sp)) * Hkv + hkv) * D;
}

/*
 * out[b, r, hq, :] for every batch row b, every requested query row
 * i = rows[r] (or i = r when rows == NULL), every query head hq.
 *   n    = real_len[b]                      (valid keys, prefix first)
 *   s_j  = scale * sum_d q[b,i,hq,d] * K*[j,d]          j = 0 .. n-1
 *   m    = max_j s_j
 *   e_j  = exp(s_j - m)
 *   l    = sum_j e_j                        (j ascending)
 *   out  = (sum_j e_j * V*[j,:]) / l        (j ascending)
 * Returns 0, or -1 on bad arguments / allocation failure.
 */
int oracle_attn_split_kv(const uint16_t *q, const uint16_t *k_prefix,
                         const uint16_t *v_prefix, const uint16_t *k_suffix,
                         const uint16_t *v_suffix, int B, int Sq, int Sp,
                         int Ss, int Hq, int Hkv, int D,
                         const int32_t *real_len, const int32_t *q_valid,
                         double softmax_scale, const int32_t *rows, int nrows,
                         double *out, int mutate)
{
    if (B < 0 || Sq < 0 || Sp < 0 || Ss < 0 || Hq <= 0 || Hkv <= 0 || D <= 0)
        return -1;
    if (Hq % Hkv != 0)
        return -1;
    const int g = Hq / Hkv;
    const int Skv = Sp + Ss;
    const int nr = rows ? nrows : Sq;
    for (int b = 0; b < B; ++b)
        if (real_len[b] < 0 || real_len[b] > Skv || q_valid[b] < 0 || q_valid[b] > Sq)
            return -1;
    if (rows)
        for (int r = 0; r < nr; ++r)
            if (rows[r] < 0 || rows[r] >= Sq)
                return -1;

    const int64_t items = (int64_t)B * nr * Hq;
    int failed = 0;

#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
        double *acc = (double *)malloc(sizeof(double) * (size_t)D);
        if (!s || !acc) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t it = 0; it < items; ++it) {
            if (!s || !acc)
                continue;
            const int hq = (int)(it % Hq);
            const int r = (int)((it / Hq) % nr);
            const int b = (int)(it / ((int64_t)Hq * nr));
            const int i = rows ? rows[r] : r;
            double *o = out + (((int64_t)b * nr + r) * Hq + hq) * D;

            int n = real_len[b];
            if (mutate == MUT_ONE_PAD_KEY && n < Skv)
                n += 1;
            if (i >= q_valid[b] || n == 0) {
                for (int d = 0; d < D; ++d)
                    o[d] = 0.0;
                continue;
            }
            const int hkv = (mutate == MUT_GQA_MODULO) ? (hq % Hkv) : (hq / g);
            const int qh = (mutate == MUT_Q_FROM_KV_HEAD) ? hkv : hq;
            const uint16_t *qrow = q + (((int64_t)b * Sq + i) * Hq + qh) * D;
            const double scale = (mutate == MUT_SCALE_IGNORED) ? 1.0 : softmax_scale;
            const int Dd = (mutate == MUT_DROP_LAST_DIM) ? D - 1 : D;

            /* scores */
            for (int j = 0; j < n; ++j) {
                const uint16_t *krow = kv_row(k_prefix, k_suffix, b, j, hkv, Sp, Ss, Hkv, D);
                double dot = 0.0;
                for (int d = 0; d < Dd; ++d)
                    dot += bf16_bits_to_f64(qrow[d]) * bf16_bits_to_f64(krow[d]);
                s[j] = scale * dot;
                if (mutate == MUT_NEGATED_SCORES)
                    s[j] = -s[j];
            }
            /* softmax: max, exponentials, normaliser */
            double m = s[0];
            for (int j = 1; j < n; ++j)
                if (s[j] > m)
                    m = s[j];
            double l = 0.0;
            for (int j = 0; j < n; ++j) {
                s[j] = exp(s[j] - m);
                if (!(mutate == MUT_DROP_LAST_IN_SUM && j == n - 1))
                    l += s[j];
            }
            /* weighted sum of value rows */
            for (int d = 0; d < D; ++d)
                acc[d] = 0.0;
            for (int j = 0; j < n; ++j) {
                const uint16_t *vrow = (mutate == MUT_V_FROM_K)
                    ? kv_row(k_prefix, k_suffix, b, j, hkv, Sp, Ss, Hkv, D)
                    : kv_row(v_prefix, v_suffix, b, j, hkv, Sp, Ss, Hkv, D);
                for (int d = 0; d < D; ++d)
                    acc[d] += s[j] * bf16_bits_to_f64(vrow[d]);
            }
            for (int d = 0; d < D; ++d)
                o[d] = acc[d] / l;
        }
        free(s);
        free(acc);
    }
    return failed ? -1 : 0;
}

/* Round a double to the nearest bf16 (ties to even), directly (no double
 * rounding through fp32 on the tie case). */
static uint16_t f64_to_bf16_rne(double x)
{
    if (isnan(x))
        return 0x7FC0;
    float f = (float)x; /* nearest fp32; every bf16 midpoint is an fp32 value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7F800000u) == 0x7F800000u) /* +-inf after the fp32 step */
        return (uint16_t)(u >> 16);
    uint32_t up = u >> 16;
    const uint32_t low = u & 0xFFFFu;
    if (low > 0x8000u) {
        up += 1;
    } else if (low == 0x8000u) {
        const double fd = (double)f;
        if (fd == x)
            up += (up & 1u);           /* exact tie: to even */
        else if (fabs(x) > fabs(fd))
            up += 1;                   /* true value beyond the midpoint */
    }
    return (uint16_t)up;
}

uint16_t oracle_round_bf16(double x) { return f64_to_bf16_rne(x); }

/*
 * Fused Q/K RMSNorm + RoPE, one (token, head) row of D at a time, for one
 * tensor x [T, H, D] (call it once for q and once for k).
 *   r      = 1 / sqrt(mean_d x_d^2 + eps)
 *   y_d    = bf16( x_d * r * w_d )                    (RMSNorm output, stored bf16)
 *   rotary part, d < rot_dim, with c_i = table[pos, i], s_i = table[pos, rot_dim/2 + i]:
 *     half-split (rotate_half):  pair (i, i + rot_dim/2)
 *       z_i          = y_i * c_i - y_{i+h} * s_i
 *       z_{i+h}      = y_{i+h} * c_i + y_i * s_i
 *     interleaved:               pair (2i, 2i + 1)
 *       z_{2i}       = y_{2i} * c_i - y_{2i+1} * s_i
 *       z_{2i+1}     = y_{2i+1} * c_i + y_{2i} * s_i
 *   pass-through, d >= rot_dim: z_d = y_d
 *   out_d  = bf16(z_d)
 * pos[t] selects the table row of token t.  Returns 0 or -1.
 */
int oracle_qk_rmsnorm_rope(const uint16_t *x, int T, int H, int D,
                           const int32_t *pos, int table_rows,
                           const uint16_t *w, const float *table, int rot_dim,
                           int interleaved, double eps, uint16_t *y_out)
{
    if (T < 0 || H <= 0 || D <= 0 || rot_dim < 0 || rot_dim > D || (rot_dim & 1))
        return -1;
    for (int t = 0; t < T; ++t)
        if (pos[t] < 0 || pos[t] >= table_rows)
            return -1;
    const int h2 = rot_dim / 2;
    const int64_t items = (int64_t)T * H;
    int failed = 0;
#pragma omp parallel
    {
        double *y = (double *)malloc(sizeof(double) * (size_t)D);
        if (!y) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(static)
        for (int64_t it = 0; it < items; ++it) {
            if (!y)
                continue;
            const int t = (int)(it / H);
            const uint16_t *xr = x + it * D;
            uint16_t *outr = y_out + it * D;
            double ss = 0.0;
            for (int d = 0; d < D; ++d) {
                const double v = bf16_bits_to_f64(xr[d]);
                ss += v * v;
            }
            const double r = 1.0 / sqrt(ss / (double)D + eps);
            for (int d = 0; d < D; ++d)
                y[d] = bf16_bits_to_f64(
                    f64_to_bf16_rne(bf16_bits_to_f64(xr[d]) * r * bf16_bits_to_f64(w[d])));
            const float *row = table + (int64_t)pos[t] * rot_dim;
            for (int i = 0; i < h2; ++i) {
                const double c = (double)row[i];
                const double sn = (double)row[h2 + i];
                int a, bb;
                if (interleaved) {
                    a = 2 * i;
                    bb = 2 * i + 1;
                } else {
                    a = i;
                    bb = i + h2;
                }
                outr[a] = f64_to_bf16_rne(y[a] * c - y[bb] * sn);
                outr[bb] = f64_to_bf16_rne(y[bb] * c + y[a] * sn);
            }
            for (int d = rot_dim; d < D; ++d)
                outr[d] = f64_to_bf16_rne(y[d]);
        }
        free(y);
    }
    return failed ? -1 : 0;
}
