/*
 * bsa_oracle.c -- the CPU oracle for dynamic block-sparse attention.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only tests/, __graft_entry__.smoke()
 * and the cpu_baseline / reference legs of bench.py may load this library.
 * The CUDA library shares no code, header, table or helper with this file.
 *
 * It is deliberately plain and slow: fp64 arithmetic throughout, the steps
 * taken in the order the pages state them, no blocking, no fusion, no
 * reordering.  OpenMP only spreads independent rows over host cores; it never
 * changes the order of any sum.
 *
 * Sources restated here (pages by title, with section):
 *  [p1] "Attention matrix view: make only frame-0 query rows dense"
 *       s1 token packing, s2 dense vs sparse rows, s4 block-level mask
 *       override (frame-0 query-block range), s6 before/after masks,
 *       s7 "always keep text/global blocks".
 *  [p3] "Competition Domains Matter: Selective Head Globalization for
 *       Training-Free Sparse Attention in Video Diffusion Transformers"
 *       s3 setup: centroids with cluster sizes n_i, n_j and the
 *       cluster-size-weighted softmax P' (Eq. 1, rows sum to one);
 *       per-head entropy H_h (Eq. 3) and its normalisation by log C_k;
 *       domain 1 "per-row local" top-p (Eq. 2); domain 3 "grouped
 *       cross-head" with the median split on H_h and the safeguard; s4 the
 *       value-aware score of the cross-head pool (EG-Sparse).
 *  [p2] "Efficient Autoregressive Video Diffusion with Dummy Head"
 *       Step 0 frame attention score [alpha_sink, alpha_neighbor,
 *       alpha_current] per head; Step 1 Dynamic Head Programming (the greedy
 *       labelling into sink / neighbor / dummy heads).
 *  [p5] "AB-Attention: accurate block-sparse attention for video diffusion"
 *       TL;DR: exact attention computed only on the selected K/V blocks;
 *       fix (2): blocks sampled in proportion to importance and reweighted
 *       by the inverse inclusion probability (an unbiased one-pass estimate
 *       of dense attention); fix (1): the Intra-Block Clustering Selector
 *       clusters queries only within each query block (no token permutation)
 *       so the block importance estimate is faithful.
 *
 * Readings taken where the pages are silent or garbled (the equations of
 * [p3] are lost in the extracted text):
 *  - a cluster is one contiguous fixed-size block, centroid = mean over the
 *    block's valid tokens, n = its valid-token count;
 *  - P'[i,j] = n_j exp(s_ij) / sum_j' n_j' exp(s_ij'), s_ij = qc_i.kc_j/sqrt(D);
 *  - natural log; entropy mean over all C_q rows;
 *  - top-p = smallest prefix of the row in (P' desc, j asc) order whose
 *    fp64 running sum of the fp32 values reaches p, the cut entry included;
 *    every block if the row never reaches p;
 *  - text keep sets key columns j < ceil(text_len / k_block);
 *  - the frame-0 override sets every column of query blocks
 *    text_len / q_block .. (text_len + tokens_per_frame - 1) / q_block;
 *  - keys at positions >= seq_len are excluded; padded query rows give 0
 *    output and -inf log-sum-exp.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t batch, heads, seq_len, seq_pad, head_dim, q_block, k_block;
    int32_t text_len, tokens_per_frame, num_frames;
} ora_layout;

enum { ORA_TEXT_KEEP = 1u, ORA_FRAME0_DENSE = 2u };

/* bf16 bit pattern -> exact double (a bf16 is the top half of an fp32). */
static double bf16_val(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Number of tokens of block `idx` that lie before seq_len ([p3] s3: n_i, n_j). */
int ora_block_count(int seq_len, int block, int idx)
{
    long v = (long)seq_len - (long)idx * block;
    if (v < 0) return 0;
    return v > block ? block : (int)v;
}

/* [p1] s4: first and last query block that overlaps frame 0. */
void ora_frame0_qblocks(const ora_layout *L, int *first, int *last)
{
    int start = L->text_len;
    int end = L->text_len + L->tokens_per_frame;   /* exclusive */
    *first = start / L->q_block;
    *last = (end - 1) / L->q_block;
}

/* [p1] s7: number of key blocks that hold text tokens. */
int ora_text_kblocks(const ora_layout *L)
{
    return (L->text_len + L->k_block - 1) / L->k_block;
}

/*
 * Centroid of every block ([p3] s3 centroids q_{h,i}, k_{h,j}):
 * mean over the block's valid tokens, summed in fp64 in ascending token
 * order, stored as fp32.  x is bf16 [B,H,seq_pad,D]; out is fp32 [B,H,C,D].
 */
void ora_pool(const ora_layout *L, const uint16_t *x, int block, float *out)
{
    const int D = L->head_dim, C = L->seq_pad / block;
    const long BH = (long)L->batch * L->heads;
    #pragma omp parallel for schedule(static)
    for (long r = 0; r < BH * C; ++r) {
        long bh = r / C;
        int i = (int)(r % C);
        int n = ora_block_count(L->seq_len, block, i);
        const uint16_t *base = x + (bh * L->seq_pad + (long)i * block) * D;
        for (int d = 0; d < D; ++d) {
            double s = 0.0;
            for (int t = 0; t < n; ++t) s += bf16_val(base[(long)t * D + d]);
            out[r * D + d] = (float)(n > 0 ? s / n : 0.0);
        }
    }
}

/*
 * Cluster-size-weighted softmax ([p3] s3, Eq. 1):
 *   s_ij  = (qc_i . kc_j) / sqrt(D)
 *   P'_ij = n_j exp(s_ij) / sum_j' n_j' exp(s_ij')
 * evaluated in fp64 with the max of (s_ij + ln n_j) subtracted first, stored
 * as fp32 [B,H,C_q,C_k].
 */
void ora_scores(const ora_layout *L, const float *qc, const float *kc, float *probs)
{
    const int D = L->head_dim;
    const int Cq = L->seq_pad / L->q_block, Ck = L->seq_pad / L->k_block;
    const long BH = (long)L->batch * L->heads;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    #pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * Ck);
        #pragma omp for schedule(static)
        for (long r = 0; r < BH * Cq; ++r) {
            long bh = r / Cq;
            const float *qi = qc + r * D;
            double m = -INFINITY;
            for (int j = 0; j < Ck; ++j) {
                const float *kj = kc + (bh * Ck + j) * D;
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += (double)qi[d] * (double)kj[d];
                int nj = ora_block_count(L->seq_len, L->k_block, j);
                logit[j] = nj > 0 ? dot * inv_sqrt_d + log((double)nj) : -INFINITY;
                if (logit[j] > m) m = logit[j];
            }
            double z = 0.0;
            for (int j = 0; j < Ck; ++j) z += exp(logit[j] - m);
            for (int j = 0; j < Ck; ++j) probs[r * Ck + j] = (float)(exp(logit[j] - m) / z);
        }
        free(logit);
    }
}

/*
 * Per-head entropy ([p3] s3, Eq. 3): H_h = (1/C_q) sum_i ( -sum_j P' ln(P' + eps) ),
 * in fp64 over the fp32 P'.  Also H_h / ln C_k.  Outputs fp64 [B,H].
 */
void ora_entropy(const ora_layout *L, const float *probs, double eps, double *H, double *H_norm)
{
    const int Cq = L->seq_pad / L->q_block, Ck = L->seq_pad / L->k_block;
    const long BH = (long)L->batch * L->heads;
    for (long bh = 0; bh < BH; ++bh) {
        double acc = 0.0;
        for (int i = 0; i < Cq; ++i) {
            const float *row = probs + (bh * Cq + i) * (long)Ck;
            double h = 0.0;
            for (int j = 0; j < Ck; ++j) h -= (double)row[j] * log((double)row[j] + eps);
            acc += h;
        }
        H[bh] = acc / Cq;
        if (H_norm) H_norm[bh] = H[bh] / log((double)Ck);
    }
}

/* Order used by the top-p rule: larger P' first, then the lower block index. */
typedef struct { float p; int j; } ora_entry;

static int ora_entry_cmp(const void *a, const void *b)
{
    const ora_entry *x = (const ora_entry *)a, *y = (const ora_entry *)b;
    if (x->p > y->p) return -1;
    if (x->p < y->p) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

/*
 * Per-row local top-p ([p3] domain 1 "Per-row local", Eq. 2): row (b,h,i)
 * keeps the first k* entries of its (P' desc, j asc) order, with
 * k* = min{k : c_k >= p_h}, c_k the fp64 running sum of the first k fp32
 * values, or every entry when no k qualifies.  Writes mask u8 [B,H,C_q,C_k]
 * (0/1) and, when kstar is not NULL, k* per row (int32 [B,H,C_q]).
 */
void ora_topp(const ora_layout *L, const float *probs, const float *top_p,
              uint8_t *mask, int32_t *kstar)
{
    const int Cq = L->seq_pad / L->q_block, Ck = L->seq_pad / L->k_block;
    const long BH = (long)L->batch * L->heads;
    if (Ck <= 0 || Cq <= 0) return;
    #pragma omp parallel
    {
        ora_entry *e = (ora_entry *)malloc(sizeof(ora_entry) * Ck);
        #pragma omp for schedule(static)
        for (long r = 0; r < BH * Cq; ++r) {
            int h = (int)((r / Cq) % L->heads);
            const float *row = probs + r * Ck;
            for (int j = 0; j < Ck; ++j) { e[j].p = row[j]; e[j].j = j; }
            qsort(e, (size_t)Ck, sizeof(ora_entry), ora_entry_cmp);
            double p = (double)top_p[h], c = 0.0;
            int k = Ck;
            for (int t = 0; t < Ck; ++t) {
                c += (double)e[t].p;
                if (c >= p) { k = t + 1; break; }
            }
            uint8_t *m = mask + r * Ck;
            memset(m, 0, (size_t)Ck);
            for (int t = 0; t < k; ++t) m[e[t].j] = 1;
            if (kstar) kstar[r] = k;
        }
        free(e);
    }
}

/*
 * Overrides on the block mask:
 *  - text keep ([p1] s7 "always keep text/global blocks"): every query row
 *    keeps every key block that holds a text token;
 *  - frame-0 dense ([p1] s4 and s6 "After"): every key block of the query
 *    blocks that overlap frame 0.
 */
void ora_overrides(const ora_layout *L, uint32_t flags, uint8_t *mask)
{
    const int Cq = L->seq_pad / L->q_block, Ck = L->seq_pad / L->k_block;
    const long BH = (long)L->batch * L->heads;
    int tk = ora_text_kblocks(L);
    if (tk > Ck) tk = Ck;
    int f0 = 0, f1 = -1;
    if (L->tokens_per_frame > 0 && L->num_frames > 0) ora_frame0_qblocks(L, &f0, &f1);
    if (f1 > Cq - 1) f1 = Cq - 1;
    for (long bh = 0; bh < BH; ++bh) {
        for (int i = 0; i < Cq; ++i) {
            uint8_t *m = mask + (bh * Cq + i) * (long)Ck;
            if (flags & ORA_TEXT_KEEP)
                for (int j = 0; j < tk; ++j) m[j] = 1;
            if ((flags & ORA_FRAME0_DENSE) && i >= f0 && i <= f1)
                for (int j = 0; j < Ck; ++j) m[j] = 1;
        }
    }
}

/* Compacted lists: ascending selected key blocks per query block, and their count. */
void ora_lists(const ora_layout *L, const uint8_t *mask, int32_t *kv_index, int32_t *kv_count)
{
    const int Cq = L->seq_pad / L->q_block, Ck = L->seq_pad / L->k_block;
    const long rows = (long)L->batch * L->heads * Cq;
    for (long r = 0; r < rows; ++r) {
        int c = 0;
        for (int j = 0; j < Ck; ++j)
            if (mask[r * Ck + j]) kv_index[r * Ck + c++] = j;
        for (int t = c; t < Ck; ++t) kv_index[r * Ck + t] = -1;
        kv_count[r] = c;
    }
}

/*
 * Exact softmax attention over the selected key blocks only
 * ([p1] s2: dense rows attend to all K/V, sparse rows to the selected K/V;
 *  [p5] TL;DR: exact attention on the selected blocks).
 * For each valid query t of query block i:
 *   U = { u : u in key block j, mask[i][j] = 1, u < seq_len }
 *   s_u = scale * (Q_t . K_u), two-pass softmax with the exact max,
 *   O_t = sum_u softmax_u V_u, lse_t = m + ln sum_u exp(s_u - m),
 * all in fp64, stored as fp32.  mask == NULL means every block (dense).
 * weight (fp32 [B,H,C_q,C_k], or NULL for 1) multiplies every exp term of a
 * key of block j by weight[row, j], in the sum z and in the numerator alike
 * ([p5] fix (2): inverse-inclusion-probability reweighting).
 * Only the query blocks listed in `qrows` (flat b*H*C_q + h*C_q + i) are
 * computed; qrows == NULL means all of them.  out is fp32 [nrows, q_block, D]
 * and lse fp32 [nrows, q_block] (indexed by position in the row list).
 */
void ora_attention(const ora_layout *L, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                   const uint8_t *mask, const float *weight, double scale, long nrows,
                   const int64_t *qrows, float *out, float *lse)
{
    const int D = L->head_dim, bq = L->q_block, bk = L->k_block;
    const int Cq = L->seq_pad / bq, Ck = L->seq_pad / bk;
    const long total = qrows ? nrows : (long)L->batch * L->heads * Cq;
    #pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * L->seq_pad);
        int *u_of = (int *)malloc(sizeof(int) * L->seq_pad);
        double *acc = (double *)malloc(sizeof(double) * D);
        #pragma omp for schedule(dynamic, 1)
        for (long n = 0; n < total; ++n) {
            long r = qrows ? (long)qrows[n] : n;
            long bh = r / Cq;
            int i = (int)(r % Cq);
            const uint16_t *Kb = k + bh * L->seq_pad * (long)D;
            const uint16_t *Vb = v + bh * L->seq_pad * (long)D;
            /* the selected keys, ascending */
            int nu = 0;
            for (int j = 0; j < Ck; ++j) {
                if (mask && !mask[r * Ck + j]) continue;
                int cnt = ora_block_count(L->seq_len, bk, j);
                for (int t = 0; t < cnt; ++t) u_of[nu++] = j * bk + t;
            }
            for (int tq = 0; tq < bq; ++tq) {
                long t = (long)i * bq + tq;
                float *o = out + (n * bq + tq) * (long)D;
                const uint16_t *Qt = q + (bh * L->seq_pad + t) * D;
                if (t >= L->seq_len || nu == 0) {
                    for (int d = 0; d < D; ++d) o[d] = 0.0f;
                    if (lse) lse[n * bq + tq] = -INFINITY;
                    continue;
                }
                double m = -INFINITY;
                for (int a = 0; a < nu; ++a) {
                    const uint16_t *Ku = Kb + (long)u_of[a] * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += bf16_val(Qt[d]) * bf16_val(Ku[d]);
                    s[a] = dot * scale;
                    if (s[a] > m) m = s[a];
                }
                double z = 0.0;
                for (int d = 0; d < D; ++d) acc[d] = 0.0;
                for (int a = 0; a < nu; ++a) {
                    double e = exp(s[a] - m);
                    if (weight) e *= (double)weight[r * Ck + u_of[a] / bk];
                    const uint16_t *Vu = Vb + (long)u_of[a] * D;
                    z += e;
                    for (int d = 0; d < D; ++d) acc[d] += e * bf16_val(Vu[d]);
                }
                for (int d = 0; d < D; ++d) o[d] = (float)(acc[d] / z);
                if (lse) lse[n * bq + tq] = (float)(m + log(z));
            }
        }
        free(s);
        free(u_of);
        free(acc);
    }
}

/*
 * ---------------------------------------------------------------------------
 * Entropy-guided competition domains ([p3] s3.3 domain 3 "Grouped
 * cross-head", the minimum one-key-per-row safeguard; s4 the value-aware
 * importance score in the cross-head pool).  Readings where the page is
 * silent (its equations are lost in the extracted text):
 *  - the value centroid c^V_{h,j} is the mean of V over key block j's valid
 *    tokens (like the key centroid), and the score of a pool pair is
 *    I_{h,i,j} = P'_{h,i,j} * ||c^V_{h,j}||_2, the product of the two fp32
 *    values rounded to fp32;
 *  - "split by the median of H_h": per batch entry, heads ordered by
 *    (H_h ascending, h ascending); the first floor(H/2) are the low-entropy
 *    heads (an odd middle head stays with the high-entropy, per-row heads);
 *  - a pool's top-p keeps the shortest prefix of its (I desc, h, i, j asc)
 *    order whose fp64 running sum reaches pool_p times the pool's total
 *    (rows of a pool are not normalised to one as a single row is);
 *  - the safeguard gives an empty pool row its highest-scoring key block
 *    (lowest j on ties), by the pool's score.
 * ---------------------------------------------------------------------------
 */

/* ||c^V_{h,j}||_2 with the centroid a fp64 mean over the block's valid tokens
 * in ascending token order; fp32 [B,H,C_k]. */
void ora_value_norms(const ora_layout *L, const uint16_t *v, float *out)
{
    const int D = L->head_dim, Ck = L->seq_pad / L->k_block;
    const long BH = (long)L->batch * L->heads;
    #pragma omp parallel for schedule(static)
    for (long r = 0; r < BH * Ck; ++r) {
        long bh = r / Ck;
        int j = (int)(r % Ck);
        int n = ora_block_count(L->seq_len, L->k_block, j);
        const uint16_t *base = v + (bh * L->seq_pad + (long)j * L->k_block) * D;
        double ss = 0.0;
        for (int d = 0; d < D; ++d) {
            double s = 0.0;
            for (int t = 0; t < n; ++t) s += bf16_val(base[(long)t * D + d]);
            double c = n > 0 ? s / n : 0.0;
            ss += c * c;
        }
        out[r] = (float)sqrt(ss);
    }
}

/* Centroid-output distortion ([p3] s3, the controlled diagnostic of the
 * competition domains): per head the dense centroid output O_i = sum_j P'_ij
 * c^V_j, the masked one renormalised per row, Om_i = sum_j M_ij P'_ij c^V_j /
 * sum_j M_ij P'_ij (0 for an empty row), and the relative Frobenius error
 * ||Om - O||_F / ||O||_F, fp64 [B,H].  vcent fp32 [B,H,C_k,D] (the value
 * centroids, block means of V). */
void ora_centroid_distortion(const ora_layout *L, const float *probs, const float *vcent,
                             const uint8_t *mask, double *out)
{
    const int D = L->head_dim, Cq = L->seq_pad / L->q_block, Ck = L->seq_pad / L->k_block;
    const long BH = (long)L->batch * L->heads;
    #pragma omp parallel for schedule(static)
    for (long bh = 0; bh < BH; ++bh) {
        double num = 0.0, den = 0.0;
        for (int i = 0; i < Cq; ++i) {
            const float *p = probs + (bh * Cq + i) * (long)Ck;
            const uint8_t *m = mask + (bh * Cq + i) * (long)Ck;
            double z = 0.0;
            for (int j = 0; j < Ck; ++j)
                if (m[j]) z += (double)p[j];
            for (int d = 0; d < D; ++d) {
                double o = 0.0, om = 0.0;
                for (int j = 0; j < Ck; ++j) {
                    double c = (double)vcent[(bh * Ck + j) * D + d];
                    o += (double)p[j] * c;
                    if (m[j]) om += (double)p[j] * c;
                }
                om = z > 0.0 ? om / z : 0.0;
                num += (om - o) * (om - o);
                den += o * o;
            }
        }
        out[bh] = den > 0.0 ? sqrt(num / den) : 0.0;
    }
}

typedef struct { double H; int h; } ora_head;

static int ora_head_cmp(const void *a, const void *b)
{
    const ora_head *x = (const ora_head *)a, *y = (const ora_head *)b;
    if (x->H < y->H) return -1;
    if (x->H > y->H) return 1;
    return (x->h > y->h) - (x->h < y->h);
}

/* Median split of the heads of every batch entry: low[b,h] = 1 for the
 * floor(H/2) heads first in (H_h asc, h asc) order, else 0.  H is [B,H]. */
void ora_eg_route(const ora_layout *L, const double *H, uint8_t *low)
{
    const int nh = L->heads;
    ora_head *o = (ora_head *)malloc(sizeof(ora_head) * nh);
    for (int b = 0; b < L->batch; ++b) {
        for (int h = 0; h < nh; ++h) {
            o[h].H = H[(long)b * nh + h];
            o[h].h = h;
        }
        qsort(o, (size_t)nh, sizeof(ora_head), ora_head_cmp);
        for (int h = 0; h < nh; ++h) low[(long)b * nh + h] = 0;
        for (int k = 0; k < nh / 2; ++k) low[(long)b * nh + o[k].h] = 1;
    }
    free(o);
}

typedef struct { float I; int h, i, j; } ora_pair;

static int ora_pair_cmp(const void *a, const void *b)
{
    const ora_pair *x = (const ora_pair *)a, *y = (const ora_pair *)b;
    if (x->I > y->I) return -1;
    if (x->I < y->I) return 1;
    if (x->h != y->h) return (x->h > y->h) - (x->h < y->h);
    if (x->i != y->i) return (x->i > y->i) - (x->i < y->i);
    if (x->j != y->j) return x->j < y->j ? -1 : 1;
    return 0;
}

/* Score of pair (bh, i, j) in the cross-head pool: P' * ||c^V||, rounded to
 * fp32, or P' itself when there are no value norms. */
static float ora_pool_score(const float *probs, const float *vnorm, long bh, int Cq, int Ck,
                            int i, int j)
{
    float p = probs[(bh * Cq + i) * (long)Ck + j];
    if (!vnorm) return p;
    float v = vnorm[bh * Ck + j];
    return p * v;
}

/*
 * Entropy-guided selection.  Heads with low[b,h] == 0 keep the per-row local
 * top-p of ora_topp with p = top_p[h].  For every batch entry, all pairs
 * (h,i,j) of its low heads form one pool ranked by I in (I desc, h, i, j asc)
 * order; the pool keeps its first k* pairs, k* = min{k >= 1 : c_k >= pool_p * T}
 * with c_k the fp64 running sum of the first k fp32 scores and T = c_N, or
 * every pair when no k qualifies.  Then every pool row (h,i) left without a
 * kept pair keeps its highest-scoring key block.  mask is u8 [B,H,C_q,C_k].
 */
/* Pooled top-p over competition domains: heads with pool_of[b,h] = g >= 0 form
 * pool g of batch entry b (G pools per entry); the pairs (h, i, j) of one pool
 * compete in (I desc, h, i, j asc) order for the shortest prefix reaching
 * pool_p of the pool's total, then the safeguard; heads with pool_of = -1 keep
 * the per-row rule with their top_p[h] ([p3] s3 the four domains). */
void ora_pool_select(const ora_layout *L, const float *probs, const float *vnorm,
                     const float *top_p, float pool_p, const int8_t *pool_of, int G, uint8_t *mask)
{
    const int Cq = L->seq_pad / L->q_block, Ck = L->seq_pad / L->k_block;
    const int nh = L->heads;
    /* per-row heads: the domain-1 rule, whole layout at once */
    ora_topp(L, probs, top_p, mask, NULL);
    if (Cq <= 0 || Ck <= 0) return;
    for (int b = 0; b < L->batch; ++b)
      for (int g = 0; g < G; ++g) {
        long n = 0;
        for (int h = 0; h < nh; ++h)
            if (pool_of[(long)b * nh + h] == g) n += (long)Cq * Ck;
        if (n == 0) continue;
        ora_pair *e = (ora_pair *)malloc(sizeof(ora_pair) * (size_t)n);
        long k = 0;
        for (int h = 0; h < nh; ++h) {
            if (pool_of[(long)b * nh + h] != g) continue;
            long bh = (long)b * nh + h;
            for (int i = 0; i < Cq; ++i) {
                memset(mask + (bh * Cq + i) * (long)Ck, 0, (size_t)Ck);
                for (int j = 0; j < Ck; ++j) {
                    e[k].I = ora_pool_score(probs, vnorm, bh, Cq, Ck, i, j);
                    e[k].h = h;
                    e[k].i = i;
                    e[k].j = j;
                    ++k;
                }
            }
        }
        qsort(e, (size_t)n, sizeof(ora_pair), ora_pair_cmp);
        double T = 0.0;
        for (long t = 0; t < n; ++t) T += (double)e[t].I;
        const double target = (double)pool_p * T;
        long kstar = n;
        double c = 0.0;
        for (long t = 0; t < n; ++t) {
            c += (double)e[t].I;
            if (c >= target) { kstar = t + 1; break; }
        }
        for (long t = 0; t < kstar; ++t) {
            long bh = (long)b * nh + e[t].h;
            mask[(bh * Cq + e[t].i) * (long)Ck + e[t].j] = 1;
        }
        free(e);
        /* safeguard: an empty pool row keeps its best key block */
        for (int h = 0; h < nh; ++h) {
            if (pool_of[(long)b * nh + h] != g) continue;
            long bh = (long)b * nh + h;
            for (int i = 0; i < Cq; ++i) {
                uint8_t *m = mask + (bh * Cq + i) * (long)Ck;
                int any = 0;
                for (int j = 0; j < Ck; ++j) any |= m[j];
                if (any) continue;
                int best = 0;
                float bv = ora_pool_score(probs, vnorm, bh, Cq, Ck, i, 0);
                for (int j = 1; j < Ck; ++j) {
                    float x = ora_pool_score(probs, vnorm, bh, Cq, Ck, i, j);
                    if (x > bv) { bv = x; best = j; }
                }
                m[best] = 1;
            }
        }
      }
}

/* EG-Sparse: the low-entropy heads of every batch entry form one pool, the
 * other heads stay per-row. */
void ora_eg_select(const ora_layout *L, const float *probs, const float *vnorm,
                   const float *top_p, float pool_p, const uint8_t *low, uint8_t *mask)
{
    const long BH = (long)L->batch * L->heads;
    int8_t *pool_of = (int8_t *)malloc((size_t)BH);
    for (long r = 0; r < BH; ++r) pool_of[r] = low[r] ? 0 : -1;
    ora_pool_select(L, probs, vnorm, top_p, pool_p, pool_of, 1, mask);
    free(pool_of);
}

/* The competition domains of [p3] s3 as pools: 0 per-row local (no pools),
 * 1 per-head global (pool h = head h), 2 grouped cross-head (the low-entropy
 * heads pool 0, the rest pool 1), 3 all-head global (one pool), 4 EG-Sparse
 * (the low-entropy heads pool 0, the rest per-row).  pool_of int8 [B,H];
 * returns G, the pools per batch entry. */
int ora_domain_route(const ora_layout *L, const double *H, int domain, int8_t *pool_of)
{
    const long BH = (long)L->batch * L->heads;
    uint8_t *low = (uint8_t *)malloc((size_t)BH);
    ora_eg_route(L, H, low);
    int G = 0;
    for (long r = 0; r < BH; ++r) {
        const int h = (int)(r % L->heads);
        switch (domain) {
            case 1: pool_of[r] = (int8_t)h; G = L->heads; break;
            case 2: pool_of[r] = low[r] ? 0 : 1; G = 2; break;
            case 3: pool_of[r] = 0; G = 1; break;
            case 4: pool_of[r] = low[r] ? 0 : -1; G = 1; break;
            default: pool_of[r] = -1; G = 0; break;
        }
    }
    free(low);
    return G;
}
/*
 * ---------------------------------------------------------------------------
 * Importance sampling with inverse-inclusion-probability weights ([p5] TL;DR
 * fix (2)).  The page gives no sampling law; the readings taken:
 *  - importance is P'; every pair (b, h, i, j) is included independently of
 *    the others (Poisson sampling) with probability
 *    pi = min(1, fp32(K * P')), K the per-row budget: a row of P' sums to one,
 *    so the expected number of blocks per row is at most K; a negative or NaN
 *    P' counts as 0;
 *  - the draw of pair idx = ((b*H + h)*C_q + i)*C_k + j is
 *    u = (z >> 40) * 2^-24 with z the idx-th output (from 0) of SplitMix64
 *    seeded with `seed`; the pair is included iff u < pi;
 *  - an included pair carries w = fp32(1 / pi); the overrides (text columns,
 *    frame-0 rows) are included with pi = 1 and w = 1;
 *  - attention multiplies each included key's exp term by its block's w in
 *    the numerator and in the sum alike (Horvitz-Thompson for both).
 * ---------------------------------------------------------------------------
 */

/* The idx-th output (idx = 0 first) of SplitMix64 started from state `seed`
 * (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
 * OOPSLA 2014): the state advances by the golden-ratio increment, the output
 * is the state passed through the two xor-shift-multiply rounds. */
uint64_t ora_splitmix64(uint64_t seed, uint64_t idx)
{
    uint64_t z = seed + (idx + 1u) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* Inclusion probability and weight of every pair: pi fp32 and w = fp32(1/pi)
 * (0 where pi = 0), both [B,H,C_q,C_k]; the overrides get pi = w = 1. */
void ora_inclusion(const ora_layout *L, const float *probs, float budget, uint32_t flags,
                   float *pi, float *w)
{
    const long n = (long)L->batch * L->heads * (L->seq_pad / L->q_block) * (L->seq_pad / L->k_block);
    uint8_t *forced = (uint8_t *)calloc((size_t)n, 1);
    ora_overrides(L, flags, forced);                     /* the pairs kept regardless */
    for (long e = 0; e < n; ++e) {
        float x = probs[e];
        if (!(x > 0.0f)) x = 0.0f;
        float prod = budget * x;                         /* fp32 product */
        float p = prod < 1.0f ? prod : 1.0f;
        if (!(p >= 0.0f)) p = 0.0f;
        if (forced[e]) p = 1.0f;
        pi[e] = p;
        w[e] = p > 0.0f ? 1.0f / p : 0.0f;               /* fp32 division */
    }
    free(forced);
}

/* One draw of the sampler: mask u8 and weight fp32 (w of included pairs, 0
 * elsewhere), [B,H,C_q,C_k]. */
void ora_sample_select(const ora_layout *L, const float *probs, float budget, uint64_t seed,
                       uint32_t flags, uint8_t *mask, float *weight)
{
    const long n = (long)L->batch * L->heads * (L->seq_pad / L->q_block) * (L->seq_pad / L->k_block);
    float *pi = (float *)malloc(sizeof(float) * (size_t)n);
    float *w = (float *)malloc(sizeof(float) * (size_t)n);
    ora_inclusion(L, probs, budget, flags, pi, w);
    for (long e = 0; e < n; ++e) {
        double u = (double)(ora_splitmix64(seed, (uint64_t)e) >> 40) * (1.0 / 16777216.0);
        int keep = u < (double)pi[e];
        mask[e] = (uint8_t)keep;
        weight[e] = keep ? w[e] : 0.0f;
    }
    free(pi);
    free(w);
}

/*
 * ---------------------------------------------------------------------------
 * Intra-block query clustering ([p5] TL;DR fix (1)).  The page names the idea
 * (cluster the queries of each query block among themselves, tokens stay in
 * place) but no procedure; the readings taken:
 *  - k-means (Lloyd's iterations) on the block's valid query tokens, k = nsub
 *    clusters, seeded with the tokens at positions floor(c * n / nsub),
 *    c = 0 .. nsub-1 (n = valid tokens of the block); squared Euclidean
 *    distance, ties to the lower cluster index; `iters` >= 1 rounds of
 *    (assign every token, move every non-empty cluster to the mean of its
 *    tokens); an empty cluster keeps its centroid and has size 0;
 *  - the block's score row is the size-weighted mixture of its
 *    sub-centroids' cluster-size-weighted softmax rows ([p3] Eq. 1 with the
 *    sub-centroid in place of q_i):
 *      P'_ij = sum_c (n_c / n_i) n_j exp(s_cj) / sum_j' n_j' exp(s_cj'),
 *    s_cj = q_c . k_j / sqrt(D); rows still sum to one, and nsub = 1 is the
 *    plain block centroid.
 * ---------------------------------------------------------------------------
 */

/* Sub-cluster centroids fp32 [B,H,C_q,nsub,D] and sizes int32 [B,H,C_q,nsub]
 * of every query block, in fp64 (sums in ascending token / dimension order). */
void ora_subclusters(const ora_layout *L, const uint16_t *q, int nsub, int iters, float *cent,
                     int32_t *size)
{
    const int D = L->head_dim, bq = L->q_block, Cq = L->seq_pad / bq;
    const long BH = (long)L->batch * L->heads;
    #pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * (size_t)bq * D);
        double *c = (double *)malloc(sizeof(double) * (size_t)nsub * D);
        double *acc = (double *)malloc(sizeof(double) * (size_t)nsub * D);
        int *cnt = (int *)malloc(sizeof(int) * (size_t)nsub);
        #pragma omp for schedule(static)
        for (long r = 0; r < BH * Cq; ++r) {
            long bh = r / Cq;
            int i = (int)(r % Cq);
            int n = ora_block_count(L->seq_len, bq, i);
            const uint16_t *base = q + (bh * L->seq_pad + (long)i * bq) * D;
            for (int t = 0; t < n; ++t)
                for (int d = 0; d < D; ++d) x[(long)t * D + d] = bf16_val(base[(long)t * D + d]);
            for (int k = 0; k < nsub; ++k) {
                int t0 = n > 0 ? (int)(((long)k * n) / nsub) : 0;
                for (int d = 0; d < D; ++d) c[(long)k * D + d] = n > 0 ? x[(long)t0 * D + d] : 0.0;
                cnt[k] = 0;
            }
            for (int it = 0; it < iters; ++it) {
                for (int k = 0; k < nsub; ++k) {
                    cnt[k] = 0;
                    for (int d = 0; d < D; ++d) acc[(long)k * D + d] = 0.0;
                }
                for (int t = 0; t < n; ++t) {
                    int best = 0;
                    double bd = INFINITY;
                    for (int k = 0; k < nsub; ++k) {
                        double dist = 0.0;
                        for (int d = 0; d < D; ++d) {
                            double e = x[(long)t * D + d] - c[(long)k * D + d];
                            dist += e * e;
                        }
                        if (dist < bd) { bd = dist; best = k; }
                    }
                    cnt[best] += 1;
                    for (int d = 0; d < D; ++d) acc[(long)best * D + d] += x[(long)t * D + d];
                }
                for (int k = 0; k < nsub; ++k)
                    if (cnt[k] > 0)
                        for (int d = 0; d < D; ++d) c[(long)k * D + d] = acc[(long)k * D + d] / cnt[k];
            }
            for (int k = 0; k < nsub; ++k) {
                for (int d = 0; d < D; ++d) cent[(r * nsub + k) * D + d] = (float)c[(long)k * D + d];
                size[r * nsub + k] = cnt[k];
            }
        }
        free(x);
        free(c);
        free(acc);
        free(cnt);
    }
}

/* Block scores from sub-clusters: the size-weighted mixture of the
 * sub-centroid rows, fp64, stored fp32 [B,H,C_q,C_k]. */
void ora_scores_clustered(const ora_layout *L, const float *cent, const int32_t *size, int nsub,
                          const float *kc, float *probs)
{
    const int D = L->head_dim;
    const int Cq = L->seq_pad / L->q_block, Ck = L->seq_pad / L->k_block;
    const long BH = (long)L->batch * L->heads;
    const double inv_sqrt_d = 1.0 / sqrt((double)L->head_dim);
    #pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * Ck);
        double *row = (double *)malloc(sizeof(double) * Ck);
        #pragma omp for schedule(static)
        for (long r = 0; r < BH * Cq; ++r) {
            long bh = r / Cq;
            long ntot = 0;
            for (int k = 0; k < nsub; ++k) ntot += size[r * nsub + k];
            for (int j = 0; j < Ck; ++j) row[j] = 0.0;
            for (int k = 0; k < nsub; ++k) {
                int nk = size[r * nsub + k];
                if (nk <= 0) continue;
                const float *qk = cent + (r * nsub + k) * D;
                double m = -INFINITY;
                for (int j = 0; j < Ck; ++j) {
                    const float *kj = kc + (bh * Ck + j) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += (double)qk[d] * (double)kj[d];
                    int nj = ora_block_count(L->seq_len, L->k_block, j);
                    logit[j] = nj > 0 ? log((double)nj) + dot * inv_sqrt_d : -INFINITY;
                    if (logit[j] > m) m = logit[j];
                }
                double z = 0.0;
                for (int j = 0; j < Ck; ++j) z += exp(logit[j] - m);
                const double wk = (double)nk / (double)ntot;
                for (int j = 0; j < Ck; ++j) row[j] += wk * (exp(logit[j] - m) / z);
            }
            for (int j = 0; j < Ck; ++j) probs[r * Ck + j] = (float)row[j];
        }
        free(logit);
        free(row);
    }
}

/*
 * ---------------------------------------------------------------------------
 * Head profiling for autoregressive generation ([p2] Step 0 and Step 1).
 * Readings where the page is informal:
 *  - the key window is num_frames frames of tokens_per_frame tokens (no text):
 *    frame 0 the sink, frames 1 .. F-2 the neighbor window, frame F-1 the
 *    current frame (the group of a key is its frame's);
 *  - the queries are the current frame's tokens, every query_stride-th one
 *    from the frame's first token ("a subset of queries for speed");
 *  - a query's attention is the softmax of scale * q . k over the whole
 *    window; alpha_g = the mean over the queries of the mass on group g
 *    (so the three values sum to one: "normalize so they add up to 1");
 *  - DHP: l_h = max(alpha_sink, alpha_neighbor); the n_dummy heads with the
 *    smallest l_h (lower h on ties) are dummy; every other head is sink if
 *    alpha_sink > alpha_neighbor, else neighbor.
 * ---------------------------------------------------------------------------
 */

/* alpha fp64 [B,H,3] in the order sink, neighbor, current. */
void ora_frame_scores(const ora_layout *L, const uint16_t *q, const uint16_t *k, double scale,
                      int query_stride, double *alpha)
{
    const int D = L->head_dim, T = L->tokens_per_frame, F = L->num_frames;
    const long BH = (long)L->batch * L->heads;
    const int n_keys = F * T;
    #pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)n_keys);
        #pragma omp for schedule(static)
        for (long bh = 0; bh < BH; ++bh) {
            const uint16_t *Qb = q + bh * L->seq_pad * (long)D;
            const uint16_t *Kb = k + bh * L->seq_pad * (long)D;
            double acc[3] = {0.0, 0.0, 0.0};
            long nq = 0;
            for (int t = (F - 1) * T; t < F * T; t += query_stride) {
                double m = -INFINITY;
                for (int u = 0; u < n_keys; ++u) {
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d)
                        dot += bf16_val(Qb[(long)t * D + d]) * bf16_val(Kb[(long)u * D + d]);
                    s[u] = dot * scale;
                    if (s[u] > m) m = s[u];
                }
                double z = 0.0, g[3] = {0.0, 0.0, 0.0};
                for (int u = 0; u < n_keys; ++u) {
                    double e = exp(s[u] - m);
                    int f = u / T;
                    int grp = f == 0 ? 0 : (f == F - 1 ? 2 : 1);
                    z = z + e;
                    g[grp] += e;
                }
                for (int c = 0; c < 3; ++c) acc[c] += g[c] / z;
                ++nq;
            }
            for (int c = 0; c < 3; ++c) alpha[bh * 3 + c] = nq > 0 ? acc[c] / (double)nq : 0.0;
        }
        free(s);
    }
}

static const double *ora_dhp_l;
static int ora_dhp_cmp(const void *a, const void *b)
{
    int x = *(const int *)a, y = *(const int *)b;
    if (ora_dhp_l[x] < ora_dhp_l[y]) return -1;
    if (ora_dhp_l[x] > ora_dhp_l[y]) return 1;
    return (x > y) - (x < y);
}

/* Dynamic Head Programming for one set of H heads: label[h] = 0 sink,
 * 1 neighbor, 2 dummy, from alpha [H,3]. */
void ora_dhp(const double *alpha, int H, int n_dummy, int *label)
{
    double *l = (double *)malloc(sizeof(double) * (size_t)H);
    int *order = (int *)malloc(sizeof(int) * (size_t)H);
    for (int h = 0; h < H; ++h) {
        l[h] = alpha[h * 3] > alpha[h * 3 + 1] ? alpha[h * 3] : alpha[h * 3 + 1];
        order[h] = h;
    }
    ora_dhp_l = l;
    qsort(order, (size_t)H, sizeof(int), ora_dhp_cmp);
    for (int h = 0; h < H; ++h) label[h] = alpha[h * 3] > alpha[h * 3 + 1] ? 0 : 1;
    for (int r = 0; r < n_dummy && r < H; ++r) label[order[r]] = 2;
    free(l);
    free(order);
}

/* Threads OpenMP will use (reported next to oracle timings). */
int ora_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
