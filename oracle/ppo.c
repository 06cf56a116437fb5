/*
 * Oracle for Parallel Prompting attention: TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
 * load this library.  It shares no code, header, table or helper with the
 * CUDA path under shared_context_decode_b200/csrc, and it never reads any
 * value the CUDA path produced.
 *
 * What it computes (project page "Read Once, Answer Many", section
 * "How it works", item 1 "A stream mask" and item 2 "Shared positions"; the
 * arXiv abstract of the same paper):
 *   Every KV slot carries a stream id and a position.  Stream id 0 is the
 *   shared document; answer streams are 1..P.  A query of stream s at
 *   position p sees key j iff
 *       sid_j == 0                      (a document key), or
 *       sid_j == s  and  pos_j <= p     (an earlier-or-same token of its own
 *                                        stream).
 *   For a document query (s == 0) the document keys are visible only when
 *   pos_j <= p, i.e. ordinary causal attention over the document.
 *   A query with s < 0 (an inactive row) sees nothing.
 *   Over the visible set V:  x_j = scale * <q, k_j>,  M = max x_j,
 *   Z = sum exp(x_j - M),  o = sum exp(x_j - M) v_j / Z,  lse = M + ln Z.
 *   An empty visible set gives o = 0 and lse = -inf.
 *
 * Everything is evaluated in double precision from the exact bf16 inputs,
 * with a two-pass softmax (max first, then the sums), one (query, head) at a
 * time, in slot order.  No blocking, no online rescaling, no reordering.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 -> double.  A bf16 value is the top 16 bits of an IEEE binary32. */
static double bf16_to_double(uint16_t h)
{
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* The stream-mask rule (project page, "How it works", item 1). */
static int key_visible(int32_t q_sid, int32_t q_pos, int32_t k_sid, int32_t k_pos)
{
    if (q_sid < 0 || k_sid < 0) return 0;
    if (k_sid == 0) return (q_sid != 0) || (k_pos <= q_pos);
    return (k_sid == q_sid) && (k_pos <= q_pos);
}

/*
 * ppo_attention: masked softmax attention over a flat list of tagged slots.
 *   q      [nq][H][d] bf16 bits         q_sid, q_pos [nq]
 *   k, v   [nk][H][d] bf16 bits         k_sid, k_pos [nk]
 *   o      [nq][H][d] double (out)      lse [nq][H] double (out, may be NULL)
 *   nvis   [nq] int32 (out, may be NULL): size of the visible set.
 * Returns 0, or -1 on bad sizes.
 */
int ppo_attention(int32_t nq, int32_t nk, int32_t H, int32_t d,
                  const uint16_t *q, const int32_t *q_sid, const int32_t *q_pos,
                  const uint16_t *k, const uint16_t *v,
                  const int32_t *k_sid, const int32_t *k_pos,
                  double scale, double *o, double *lse, int32_t *nvis)
{
    if (nq < 0 || nk < 0 || H <= 0 || d <= 0) return -1;
    if (nvis) {
        for (int32_t i = 0; i < nq; ++i) {
            int32_t c = 0;
            for (int32_t j = 0; j < nk; ++j)
                c += key_visible(q_sid[i], q_pos[i], k_sid[j], k_pos[j]);
            nvis[i] = c;
        }
    }
    int64_t work = (int64_t)nq * H;
#pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * (nk > 0 ? nk : 1));
        char *vis = (char *)malloc(nk > 0 ? nk : 1);
#pragma omp for schedule(dynamic, 1)
        for (int64_t w = 0; w < work; ++w) {
            int32_t i = (int32_t)(w / H), h = (int32_t)(w % H);
            const uint16_t *qi = q + ((int64_t)i * H + h) * d;
            double *oi = o + ((int64_t)i * H + h) * d;
            for (int32_t c = 0; c < d; ++c) oi[c] = 0.0;
            /* pass 1: scores of the visible keys and their maximum */
            double M = -INFINITY;
            int32_t count = 0;
            for (int32_t j = 0; j < nk; ++j) {
                vis[j] = (char)key_visible(q_sid[i], q_pos[i], k_sid[j], k_pos[j]);
                if (!vis[j]) continue;
                const uint16_t *kj = k + ((int64_t)j * H + h) * d;
                double s = 0.0;
                for (int32_t c = 0; c < d; ++c) s += bf16_to_double(qi[c]) * bf16_to_double(kj[c]);
                x[j] = scale * s;
                if (x[j] > M) M = x[j];
                ++count;
            }
            if (count == 0) {
                if (lse) lse[(int64_t)i * H + h] = -INFINITY;
                continue;
            }
            /* pass 2: normaliser and weighted sum of values */
            double Z = 0.0;
            for (int32_t j = 0; j < nk; ++j) {
                if (!vis[j]) continue;
                double wgt = exp(x[j] - M);
                Z += wgt;
                const uint16_t *vj = v + ((int64_t)j * H + h) * d;
                for (int32_t c = 0; c < d; ++c) oi[c] += wgt * bf16_to_double(vj[c]);
            }
            for (int32_t c = 0; c < d; ++c) oi[c] /= Z;
            if (lse) lse[(int64_t)i * H + h] = M + log(Z);
        }
        free(x);
        free(vis);
    }
    return 0;
}

/* Visibility matrix of the same rule: mask[i][j] = 1 iff query i sees key j. */
int ppo_visibility(int32_t nq, int32_t nk,
                   const int32_t *q_sid, const int32_t *q_pos,
                   const int32_t *k_sid, const int32_t *k_pos, uint8_t *mask)
{
    if (nq < 0 || nk < 0) return -1;
    for (int32_t i = 0; i < nq; ++i)
        for (int32_t j = 0; j < nk; ++j)
            mask[(int64_t)i * nk + j] = (uint8_t)key_visible(q_sid[i], q_pos[i], k_sid[j], k_pos[j]);
    return 0;
}

/* Number of host threads OpenMP will use (reported beside CPU timings). */
int ppo_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
