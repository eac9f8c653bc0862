/*
 * attention_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of the multi-head softmax attention that
 * the LTX-2 joint audio-video DiT runs in every block: video self-attention,
 * audio self-attention with a key-padding mask on the zero-padded audio tail,
 * v2a (audio queries over video keys/values) and a2v (video queries over audio
 * keys/values).  Sources for what is computed:
 *
 *   - "LTX-2: replicate audio stream across Ulysses ranks by default"
 *     (TensorRT-LLM pull request 16228), Description: the two streams (15360
 *     video tokens, 126 audio tokens), v2a = audio-Q x video-KV, the a2v
 *     all-gather of audio keys/values, and the padding of the audio sequence.
 *   - "feat(ltx2): tile-parallel video VAE and the two-stage pipeline"
 *     (TensorRT-Model-Connect pull request 1586), commit "Onboard Lightricks
 *     LTX-2.5": video self-attention over normed and rotated keys/values, and
 *     v2a split over key ranges whose per-part softmax statistics are merged
 *     in fp32 -- the merge rule is oracle_merge_partials below.
 *
 * The pages give no formula for attention itself; this file writes out the
 * textbook definition
 *     s_j = scale * <q_i, k_j>            for keys j < kv_valid_len
 *     p_j = exp(s_j - max_j s_j),  l = sum_j p_j
 *     o_i = sum_j p_j v_j / l
 * per (batch b, head h, query row i), in double precision, with plain loops.
 * Only tests, the smoke check and the CPU-baseline leg of the benchmark may
 * load this file.  It shares no code with the CUDA library.
 *
 * Data layout (a reading; the pages print no tensor layout): BSHD contiguous,
 * element (b, s, h, d) at ((b*len + s)*heads + h)*head_dim + d, bf16 stored as
 * raw 16-bit patterns and widened exactly to double here.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 bit pattern -> double, exactly (bf16 is the upper half of an IEEE binary32). */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static size_t bshd(int b, int s, int h, int d, int len, int heads, int head_dim) {
    return (((size_t)b * (size_t)len + (size_t)s) * (size_t)heads + (size_t)h) * (size_t)head_dim + (size_t)d;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Attention of one query row (b, i, h) over keys j in [j0, j1), j1 <= kv_valid_len.
 * Writes the normalised output o[head_dim] and the row statistics m (max score)
 * and l (sum of exp(s_j - m)).  Returns 0, or -1 for an empty key range.
 */
static int attend_row(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      int b, int i, int h, int q_len, int kv_len, int heads, int head_dim,
                      double scale, int j0, int j1, double* s_buf, double* o, double* m_out,
                      double* l_out) {
    if (j1 <= j0) return -1;
    /* scores */
    double m = -INFINITY;
    for (int j = j0; j < j1; ++j) {
        double acc = 0.0;
        for (int d = 0; d < head_dim; ++d) {
            acc += bf16_to_double(q[bshd(b, i, h, d, q_len, heads, head_dim)]) *
                   bf16_to_double(k[bshd(b, j, h, d, kv_len, heads, head_dim)]);
        }
        double s = scale * acc;
        s_buf[j - j0] = s;
        if (s > m) m = s;
    }
    /* probabilities and their sum */
    double l = 0.0;
    for (int j = j0; j < j1; ++j) {
        double p = exp(s_buf[j - j0] - m);
        s_buf[j - j0] = p;
        l += p;
    }
    /* weighted sum of values */
    for (int d = 0; d < head_dim; ++d) o[d] = 0.0;
    for (int j = j0; j < j1; ++j) {
        double p = s_buf[j - j0];
        for (int d = 0; d < head_dim; ++d)
            o[d] += p * bf16_to_double(v[bshd(b, j, h, d, kv_len, heads, head_dim)]);
    }
    for (int d = 0; d < head_dim; ++d) o[d] /= l;
    *m_out = m;
    *l_out = l;
    return 0;
}

static int check_args(int batch, int q_len, int kv_len, int kv_valid_len, int heads, int head_dim) {
    if (batch < 1 || q_len < 1 || kv_len < 1 || heads < 1 || head_dim < 1) return -1;
    if (kv_valid_len < 1 || kv_valid_len > kv_len) return -1;
    return 0;
}

/*
 * Full or row-sampled attention.
 *   rows == NULL : every (b, i, h); out is BSHD [batch, q_len, heads, head_dim].
 *   rows != NULL : n_rows flat indices r = (b*q_len + i)*heads + h; out is [n_rows, head_dim].
 * lse (optional, may be NULL): natural-log log-sum-exp m + log(l) per output row.
 * Keys j >= kv_valid_len are excluded (the key-padding mask).
 * Returns 0 on success, -1 on a bad argument.
 */
int oracle_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, double* out,
                     double* lse, int batch, int q_len, int kv_len, int kv_valid_len, int heads,
                     int head_dim, double scale, const int64_t* rows, int64_t n_rows) {
    if (check_args(batch, q_len, kv_len, kv_valid_len, heads, head_dim)) return -1;
    int64_t total = (int64_t)batch * q_len * heads;
    int64_t n = rows ? n_rows : total;
    if (rows) {
        for (int64_t r = 0; r < n; ++r)
            if (rows[r] < 0 || rows[r] >= total) return -1;
    }
    int bad = 0;
#pragma omp parallel
    {
        double* s_buf = (double*)malloc(sizeof(double) * (size_t)kv_valid_len);
        if (!s_buf) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t r = 0; r < n; ++r) {
                int64_t flat = rows ? rows[r] : r;
                int h = (int)(flat % heads);
                int64_t bi = flat / heads;
                int i = (int)(bi % q_len);
                int b = (int)(bi / q_len);
                double m, l;
                attend_row(q, k, v, b, i, h, q_len, kv_len, heads, head_dim, scale, 0, kv_valid_len,
                           s_buf, out + (size_t)r * (size_t)head_dim, &m, &l);
                if (lse) lse[r] = m + log(l);
            }
            free(s_buf);
        }
    }
    return bad ? -1 : 0;
}

/*
 * Attention restricted to the key range [j0, j1) (j1 <= kv_valid_len), for every
 * (b, i, h): the per-part result of a key-range split.  o_part is BSHD
 * [batch, q_len, heads, head_dim] (normalised within the part), m_part and l_part
 * are [batch, q_len, heads]: the part's max score and its sum of exp(s - m).
 */
int oracle_attention_part(const uint16_t* q, const uint16_t* k, const uint16_t* v, double* o_part,
                          double* m_part, double* l_part, int batch, int q_len, int kv_len,
                          int kv_valid_len, int heads, int head_dim, double scale, int j0, int j1) {
    if (check_args(batch, q_len, kv_len, kv_valid_len, heads, head_dim)) return -1;
    if (j0 < 0 || j1 > kv_valid_len || j1 <= j0) return -1;
    int64_t total = (int64_t)batch * q_len * heads;
    int bad = 0;
#pragma omp parallel
    {
        double* s_buf = (double*)malloc(sizeof(double) * (size_t)(j1 - j0));
        if (!s_buf) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t r = 0; r < total; ++r) {
                int h = (int)(r % heads);
                int64_t bi = r / heads;
                int i = (int)(bi % q_len);
                int b = (int)(bi / q_len);
                attend_row(q, k, v, b, i, h, q_len, kv_len, heads, head_dim, scale, j0, j1, s_buf,
                           o_part + (size_t)r * (size_t)head_dim, &m_part[r], &l_part[r]);
            }
            free(s_buf);
        }
    }
    return bad ? -1 : 0;
}

/*
 * Merge of per-part softmax statistics (the key-range split of v2a in
 * "feat(ltx2): tile-parallel video VAE and the two-stage pipeline", commit
 * "Onboard Lightricks LTX-2.5"):
 *     m = max_p m_p,   l = sum_p exp(m_p - m) l_p,
 *     o = sum_p exp(m_p - m) l_p o_p / l.
 * o_parts [n_parts][n_rows][head_dim], m_parts/l_parts [n_parts][n_rows];
 * out [n_rows][head_dim]; lse (optional) [n_rows] = m + log(l).
 */
int oracle_merge_partials(int n_parts, int64_t n_rows, int head_dim, const double* o_parts,
                          const double* m_parts, const double* l_parts, double* out, double* lse) {
    if (n_parts < 1 || n_rows < 0 || head_dim < 1) return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        double m = -INFINITY;
        for (int p = 0; p < n_parts; ++p) {
            double mp = m_parts[(size_t)p * (size_t)n_rows + (size_t)r];
            if (mp > m) m = mp;
        }
        double l = 0.0;
        for (int p = 0; p < n_parts; ++p) {
            size_t pr = (size_t)p * (size_t)n_rows + (size_t)r;
            l += exp(m_parts[pr] - m) * l_parts[pr];
        }
        for (int d = 0; d < head_dim; ++d) {
            double acc = 0.0;
            for (int p = 0; p < n_parts; ++p) {
                size_t pr = (size_t)p * (size_t)n_rows + (size_t)r;
                acc += exp(m_parts[pr] - m) * l_parts[pr] *
                       o_parts[pr * (size_t)head_dim + (size_t)d];
            }
            out[(size_t)r * (size_t)head_dim + (size_t)d] = acc / l;
        }
        if (lse) lse[r] = m + log(l);
    }
    return 0;
}

/*
 * The softmax weights themselves, P[b, h, i, j] = p_j / l (zero for masked keys
 * j >= kv_valid_len), for small cases: [batch, heads, q_len, kv_len].
 */
int oracle_softmax_weights(const uint16_t* q, const uint16_t* k, double* p_out, int batch,
                           int q_len, int kv_len, int kv_valid_len, int heads, int head_dim,
                           double scale) {
    if (check_args(batch, q_len, kv_len, kv_valid_len, heads, head_dim)) return -1;
    for (int b = 0; b < batch; ++b)
        for (int h = 0; h < heads; ++h)
            for (int i = 0; i < q_len; ++i) {
                double* row = p_out + (((size_t)b * heads + h) * q_len + i) * (size_t)kv_len;
                double m = -INFINITY;
                for (int j = 0; j < kv_valid_len; ++j) {
                    double acc = 0.0;
                    for (int d = 0; d < head_dim; ++d)
                        acc += bf16_to_double(q[bshd(b, i, h, d, q_len, heads, head_dim)]) *
                               bf16_to_double(k[bshd(b, j, h, d, kv_len, heads, head_dim)]);
                    row[j] = scale * acc;
                    if (row[j] > m) m = row[j];
                }
                double l = 0.0;
                for (int j = 0; j < kv_valid_len; ++j) {
                    row[j] = exp(row[j] - m);
                    l += row[j];
                }
                for (int j = 0; j < kv_valid_len; ++j) row[j] /= l;
                for (int j = kv_valid_len; j < kv_len; ++j) row[j] = 0.0;
            }
    return 0;
}
