/*
 * nsa_oracle.c -- plain, slow, fp64 CPU oracle for the NSA compressed-attention
 * path.  TEST INFRASTRUCTURE ONLY: tests, the smoke check and the benchmark's
 * CPU-baseline leg call it; the product library never links, loads or calls it,
 * and it shares no code, header or table with the CUDA path.
 *
 * Sources (web pages; cited by page title and the section/equation used):
 *   [CMP]  "aclnnNsaCompress" (Ascend CANN API page) -- Formula section:
 *          K~cmp_t = { phi(k_{id+1 : id+l}) | 0 <= i <= floor((t-l)/d) }.
 *   [ATT]  "mindspore.ops.nsa_compress_attention" -- steps 1..7 of the
 *          description, the note list (TND layout, prefix-sum lengths,
 *          constraints) and the Returns list (output shapes).
 *   [RFA]  "lite_boost.ops.rain_fusion_attention" -- select_idx parameter:
 *          valid indices listed in ascending order first, then -1 padding;
 *          block-sparse attention over the listed KV blocks, causal mask
 *          (mask_type 0), GQA, attention_out and softmax_lse returns.
 *
 * Readings taken where the pages are silent or garbled (each one is listed in
 * the design notes of this repository):
 *   phi     weighted sum over the window with weights w[j][n] (shape l x N2),
 *           the same w for K and V; 0-based rows i*d .. i*d+l-1.
 *   n_cmp   floor((S-l)/d)+1 when S >= l, else 0 (floor, not C truncation).
 *   mask    compressed block i is visible to query position t iff i*d+l-1 <= t.
 *   offset  query row t_loc of sequence b sits at position
 *           t = t_loc + max(0, (n_cmp-1)*d + l - S_q) (bottom-right alignment;
 *           0 when n_cmp == 0).
 *   band    step 4 taken literally with out-of-range / invisible terms = 0;
 *           a = l'/d and b = l/d must be integers.
 *   group   step 5 sums over the query heads of one KV group (h / G == g).
 *   top-k   candidates j < n_sel with j*l' <= t; k* = min(count, #candidates)
 *           largest scores, ties to the smaller j, emitted ascending, then -1.
 *           A row that sees no compressed block emits all -1, zero output,
 *           max = -inf and sum = 0.
 *   stats   softmax_max = max of the scaled scores, softmax_sum = sum of
 *           exp(s - max) (natural exponent).
 *
 * Parity of the offset, candidate, ordering and empty-row readings is
 * unpinned: no page gives an example for them.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC (no fast-math: fp64 semantics kept).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------- */
/* Rounding fp64 -> storage dtype, round-to-nearest-even, from the IEEE-754    */
/* definition of binary16 (p = 11 bits, emin = -14) and bfloat16 (p = 8 bits, */
/* emin = -126).  dtype 0 = bfloat16, 1 = float16.                            */
/* ------------------------------------------------------------------------- */
static double round_to_storage(double x, int dtype)
{
    int p = (dtype == 0) ? 8 : 11;          /* significand bits incl. implicit */
    int emin = (dtype == 0) ? -126 : -14;   /* exponent of the smallest normal */
    int emax = (dtype == 0) ? 127 : 15;     /* exponent of the largest normal  */
    if (x == 0.0 || isnan(x) || isinf(x)) return x;
    int e;
    (void)frexp(x, &e);                     /* x = f * 2^e, 0.5 <= |f| < 1     */
    int qexp = e - p;                       /* exponent of one unit in the last place */
    if (qexp < emin - p + 1) qexp = emin - p + 1;  /* subnormal spacing */
    double q = ldexp(1.0, qexp);
    double y = nearbyint(x / q) * q;        /* default mode: ties to even      */
    double maxfin = ldexp(2.0 - ldexp(1.0, 1 - p), emax);
    if (fabs(y) > maxfin) y = (y > 0) ? INFINITY : -INFINITY;
    return y;
}

void oracle_round(const double* in, int64_t n, int dtype, double* out)
{
    for (int64_t i = 0; i < n; i++) out[i] = round_to_storage(in[i], dtype);
}

/* ------------------------------------------------------------------------- */
/* [CMP] Formula: number of compressed blocks of a sequence of S tokens is    */
/* floor((S-l)/d)+1 for S >= l (i runs 0..floor((S-l)/d)), 0 otherwise.       */
/* cu_seqlens holds the cumulative end of each sequence (no leading 0).       */
/* Writes cumulative ends of the compressed sequences.  Returns total.        */
/* ------------------------------------------------------------------------- */
int64_t oracle_compress_len(const int32_t* cu_seqlens, int batch, int l, int d,
                            int32_t* cu_cmp)
{
    int64_t total = 0;
    int32_t prev = 0;
    for (int b = 0; b < batch; b++) {
        int64_t S = (int64_t)cu_seqlens[b] - prev;
        prev = cu_seqlens[b];
        int64_t n = 0;
        /* count the i with 0 <= i and i*d + l <= S, one by one */
        for (int64_t i = 0; i * d + l <= S; i++) n++;
        total += n;
        cu_cmp[b] = (int32_t)total;
    }
    return total;
}

/* ------------------------------------------------------------------------- */
/* [CMP] Formula with phi = weighted window sum (reading above):              */
/*   out[c0+i][n][:] = sum_{j=0}^{l-1} w[j][n] * x[s0 + i*d + j][n][:]        */
/* x: (T, N2, D) fp64; w: (l, N2) fp64; out: (Tc, N2, D) fp64, unrounded.     */
/* ------------------------------------------------------------------------- */
void oracle_compress(const double* x, const double* w, int l, int d,
                     const int32_t* cu_seqlens, int batch, int n2, int dim,
                     const int32_t* cu_cmp, double* out)
{
    for (int b = 0; b < batch; b++) {
        int64_t s0 = (b == 0) ? 0 : cu_seqlens[b - 1];
        int64_t c0 = (b == 0) ? 0 : cu_cmp[b - 1];
        int64_t ncmp = cu_cmp[b] - c0;
        #pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < ncmp; i++) {
            for (int n = 0; n < n2; n++) {
                for (int e = 0; e < dim; e++) {
                    double acc = 0.0;
                    for (int j = 0; j < l; j++) {
                        double xv = x[((s0 + i * d + j) * n2 + n) * (int64_t)dim + e];
                        acc += w[(int64_t)j * n2 + n] * xv;
                    }
                    out[((c0 + i) * n2 + n) * (int64_t)dim + e] = acc;
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* [ATT] step 4, taken literally:                                              */
/*   P_slc[j] = sum_{m=0}^{a-1} sum_{n=0}^{b-1} P_cmp[a*j - m - n]             */
/* with a = l'/d and b = l/d.  P_cmp[c] counts only for 0 <= c < n_vis (the    */
/* visible compressed blocks); every other term is 0.  P holds n_vis values.  */
/* ------------------------------------------------------------------------- */
void oracle_importance(const double* P, int n_vis, int a, int b, int n_sel,
                       double* pslc)
{
    for (int j = 0; j < n_sel; j++) {
        double acc = 0.0;
        for (int m = 0; m < a; m++) {
            for (int n = 0; n < b; n++) {
                int64_t c = (int64_t)a * j - m - n;
                if (c >= 0 && c < n_vis) acc += P[c];
            }
        }
        pslc[j] = acc;
    }
}

/* ------------------------------------------------------------------------- */
/* [ATT] step 7 with the top-k reading above.  score has n_cand entries (the  */
/* candidates j = 0..n_cand-1).  Picks k* = min(count, n_cand) indices by     */
/* descending score, ties to the smaller j, then lists them ascending ([RFA]  */
/* select_idx convention) and pads with -1 up to count.                       */
/* ------------------------------------------------------------------------- */
void oracle_topk_excl(const double* score, int n_cand, const uint8_t* excl, int count, int32_t* idx);
void oracle_topk(const double* score, int n_cand, int count, int32_t* idx)
{
    oracle_topk_excl(score, n_cand, NULL, count, idx);
}

/* As above over the candidates j < n_cand with excl[j] == 0 (excl may be     */
/* NULL): [ATT] step 6, P'_slc = topk_mask(P'_slc), read as removing the      */
/* masked blocks from the candidate set.                                     */
void oracle_topk_excl(const double* score, int n_cand, const uint8_t* excl, int count, int32_t* idx)
{
    int n_in = 0;
    for (int j = 0; j < n_cand; j++)
        if (!(excl && excl[j])) n_in++;
    int kstar = (count < n_in) ? count : n_in;
    char* taken = (char*)calloc((size_t)(n_cand > 0 ? n_cand : 1), 1);
    for (int r = 0; r < kstar; r++) {
        int best = -1;
        for (int j = 0; j < n_cand; j++) {
            if (taken[j] || (excl && excl[j])) continue;
            if (best < 0 || score[j] > score[best]) best = j;   /* strict: earlier j wins ties */
        }
        taken[best] = 1;
    }
    int w = 0;
    for (int j = 0; j < n_cand; j++)
        if (taken[j]) idx[w++] = j;
    for (; w < count; w++) idx[w] = -1;
    free(taken);
}

/* ------------------------------------------------------------------------- */
/* [ATT] steps 1..7 for a list of query rows.                                  */
/*  q  (T1, N1, D1), kc (Tc, N2, D1), vc (Tc, N2, D2): fp64 values of the      */
/*     storage-dtype tensors (TND layout).                                     */
/*  cu_q / cu_cmp / cu_sel: cumulative ends per sequence (no leading 0).      */
/*  rows: global query-row indices to evaluate (nrows of them; NULL = all).   */
/*  q_compact: when non-zero, q holds only the listed rows, in list order.    */
/* Outputs, indexed by position r in the row list:                            */
/*  out   (nrows, N1, D2)  fp64, unrounded                                     */
/*  smax  (nrows, N1)      max of the scaled scores (-inf for empty rows)      */
/*  ssum  (nrows, N1)      sum of exp(s - max) (0 for empty rows)              */
/*  topk  (nrows, N2, count)                                                   */
/* Optional masks of [ATT] steps 1 and 6 (NULL = none), bool bytes, one (S1,  */
/* S2) matrix shared by every sequence and head, indexed by the row's query   */
/* index inside its sequence and the block index; a true entry removes the    */
/* pair: amask (S1, >= n_cmp) row stride am_s2, tmask (S1, >= n_sel) row      */
/* stride tm_s2.                                                              */
/*  score (nrows, N2, sel_cap) or NULL: P_slc' for j < min(n_sel, sel_cap)     */
/*  ncand (nrows, N2) or NULL: number of top-k candidates of the row (0 when   */
/*        the row sees no block)                                               */
/* Returns 0, or -1 when l % d or l' % d is nonzero.                           */
/* ------------------------------------------------------------------------- */
int oracle_compress_attention(const double* q, const double* kc, const double* vc,
                              double scale, int n1, int n2, int d1, int d2,
                              int l, int d, int lp, int count,
                              const int32_t* cu_q, const int32_t* cu_cmp,
                              const int32_t* cu_sel, int batch,
                              const int64_t* rows, int64_t nrows, int q_compact,
                              double* out, double* smax, double* ssum,
                              int32_t* topk, double* score, int sel_cap,
                              int32_t* ncand,
                              const uint8_t* amask, int64_t am_s2,
                              const uint8_t* tmask, int64_t tm_s2)
{
    if (l % d != 0 || lp % d != 0) return -1;
    const int a = lp / d, bb = l / d;
    const int G = n1 / n2;
    if (rows == NULL) nrows = cu_q[batch - 1];

    #pragma omp parallel
    {
        int max_cmp = 0, max_sel = 0;
        for (int s = 0; s < batch; s++) {
            int nc = cu_cmp[s] - (s ? cu_cmp[s - 1] : 0);
            int ns = cu_sel[s] - (s ? cu_sel[s - 1] : 0);
            if (nc > max_cmp) max_cmp = nc;
            if (ns > max_sel) max_sel = ns;
        }
        double* sc = (double*)malloc(sizeof(double) * (size_t)(max_cmp + 1));
        double* P = (double*)malloc(sizeof(double) * (size_t)(max_cmp + 1));
        double* pslc = (double*)malloc(sizeof(double) * (size_t)(max_sel + 1));
        double* grp = (double*)malloc(sizeof(double) * (size_t)(max_sel + 1));

        #pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < nrows; r++) {
            int64_t t = rows ? rows[r] : r;
            /* sequence that owns global row t (TND + prefix sums, [ATT] note) */
            int s = 0;
            while (cu_q[s] <= t) s++;
            int64_t q0 = s ? cu_q[s - 1] : 0;
            int64_t c0 = s ? cu_cmp[s - 1] : 0;
            int64_t Sq = cu_q[s] - q0;
            int n_cmp = (int)(cu_cmp[s] - c0);
            int n_sel = (int)(cu_sel[s] - (s ? cu_sel[s - 1] : 0));
            int64_t off = 0;
            if (n_cmp > 0) {
                off = (int64_t)(n_cmp - 1) * d + l - Sq;
                if (off < 0) off = 0;
            }
            int64_t tpos = (t - q0) + off;

            /* visible set: i < n_cmp with i*d + l - 1 <= tpos (counted one by one) */
            int n_vis = 0;
            for (int i = 0; i < n_cmp; i++)
                if ((int64_t)i * d + l - 1 <= tpos) n_vis++;
            /* step 1's optional atten_mask (S1, S2cmp): a true entry at (query  */
            /* row of the sequence, block) removes the block from the visible    */
            /* set; a row left without a block is an empty row                   */
            const int64_t tloc = t - q0;
            const uint8_t* arow = amask ? amask + tloc * am_s2 : NULL;
            const uint8_t* trow = tmask ? tmask + tloc * tm_s2 : NULL;
            int n_att = 0;
            for (int i = 0; i < n_vis; i++)
                if (!(arow && arow[i])) n_att++;

            /* candidates: j < n_sel with j*l' <= tpos */
            int n_cand = 0;
            for (int j = 0; j < n_sel; j++)
                if ((int64_t)j * lp <= tpos) n_cand++;
            int n_cand_in = 0;
            for (int j = 0; j < n_cand; j++)
                if (!(trow && trow[j])) n_cand_in++;

            for (int g = 0; g < n2; g++) {
                for (int j = 0; j < n_sel; j++) grp[j] = 0.0;
                for (int hh = 0; hh < G; hh++) {
                    int h = g * G + hh;
                    double* o = out + (r * n1 + h) * (int64_t)d2;
                    for (int e = 0; e < d2; e++) o[e] = 0.0;
                    if (n_att == 0) {
                        smax[r * n1 + h] = -INFINITY;
                        ssum[r * n1 + h] = 0.0;
                        continue;
                    }
                    /* step 1: QK = scale * query * key^T over the visible blocks */
                    const double* qr = q + ((q_compact ? r : t) * n1 + h) * (int64_t)d1;
                    for (int i = 0; i < n_vis; i++) {
                        const double* kr = kc + ((c0 + i) * n2 + g) * (int64_t)d1;
                        double acc = 0.0;
                        for (int k = 0; k < d1; k++) acc += qr[k] * kr[k];
                        sc[i] = scale * acc;
                    }
                    /* step 2: P_cmp = softmax(QK) over the attended blocks */
                    double m = -INFINITY;
                    for (int i = 0; i < n_vis; i++)
                        if (!(arow && arow[i]) && sc[i] > m) m = sc[i];
                    double L = 0.0;
                    for (int i = 0; i < n_vis; i++)
                        if (!(arow && arow[i])) L += exp(sc[i] - m);
                    for (int i = 0; i < n_vis; i++)
                        P[i] = (arow && arow[i]) ? 0.0 : exp(sc[i] - m) / L;
                    smax[r * n1 + h] = m;
                    ssum[r * n1 + h] = L;
                    /* step 3: attentionOut = P_cmp * value */
                    for (int i = 0; i < n_vis; i++) {
                        const double* vr = vc + ((c0 + i) * n2 + g) * (int64_t)d2;
                        for (int e = 0; e < d2; e++) o[e] += P[i] * vr[e];
                    }
                    /* step 4: importance score of this head */
                    oracle_importance(P, n_vis, a, bb, n_sel, pslc);
                    /* step 5: sum over the heads of the group */
                    for (int j = 0; j < n_sel; j++) grp[j] += pslc[j];
                }
                if (score) {
                    int lim = n_sel < sel_cap ? n_sel : sel_cap;
                    double* dst = score + (r * n2 + g) * (int64_t)sel_cap;
                    for (int j = 0; j < sel_cap; j++) dst[j] = (j < lim) ? grp[j] : 0.0;
                }
                if (ncand) ncand[r * n2 + g] = (n_att == 0) ? 0 : n_cand_in;
                /* steps 6-7: causal candidate set less the topk_mask, then top-k */
                int32_t* ti = topk + (r * n2 + g) * (int64_t)count;
                if (n_att == 0) {
                    for (int k = 0; k < count; k++) ti[k] = -1;
                } else {
                    oracle_topk_excl(grp, n_cand, trow, count, ti);
                }
            }
        }
        free(sc); free(P); free(pslc); free(grp);
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Selection attention ([RFA], block-sparse attention driven by index lists), */
/* in the reading that feeds it with the top-k of the compressed branch:       */
/* query row t_loc of sequence b sits at key position                          */
/* t = t_loc + (S_kv - S_q) (bottom-right alignment); for head h of group      */
/* g = h / G it attends to the raw keys p of the selection blocks listed for   */
/* (t, g) in sel (block j holds positions j*l' .. j*l'+l'-1), restricted to    */
/* p <= t (causal, mask_type 0) and p < S_kv.  The list is read as a set:      */
/* -1 entries, blocks past the end of the sequence and repeats are skipped.    */
/*   out[t,h,:] = sum_p softmax_p(scale * q . k_p) v_p                         */
/*   lse[t,h]   = m + log(sum_p exp(s_p - m))   (natural log)                  */
/* An empty key set gives out = 0 and lse = -inf.                              */
/*  q (T1,N1,D1) or (nrows,N1,D1) when q_compact; k (T2,N2,D1); v (T2,N2,D2);  */
/*  sel (T1,N2,count) int32 over all query rows; cu_q / cu_kv prefix sums;     */
/*  rows: global query rows to evaluate (NULL = all); out (nrows,N1,D2);       */
/*  lse (nrows,N1).                                                            */
/* ------------------------------------------------------------------------- */
int oracle_select_attention(const double* q, const double* k, const double* v,
                            const int32_t* sel, double scale, int n1, int n2,
                            int d1, int d2, int lp, int count,
                            const int32_t* cu_q, const int32_t* cu_kv, int batch,
                            const int64_t* rows, int64_t nrows, int q_compact,
                            double* out, double* lse)
{
    if (lp <= 0 || n2 <= 0 || n1 % n2 != 0) return -1;
    const int G = n1 / n2;
    if (rows == NULL) nrows = cu_q[batch - 1];

    #pragma omp parallel
    {
        int64_t max_kv = 0;
        for (int s = 0; s < batch; s++) {
            int64_t n = cu_kv[s] - (s ? cu_kv[s - 1] : 0);
            if (n > max_kv) max_kv = n;
        }
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)(max_kv + 1));
        double* sc = (double*)malloc(sizeof(double) * (size_t)(max_kv + 1));

        #pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < nrows; r++) {
            int64_t t = rows ? rows[r] : r;
            int s = 0;
            while (cu_q[s] <= t) s++;
            int64_t q0 = s ? cu_q[s - 1] : 0;
            int64_t k0 = s ? cu_kv[s - 1] : 0;
            int64_t Sq = cu_q[s] - q0;
            int64_t Skv = cu_kv[s] - k0;
            int64_t tpos = (t - q0) + (Skv - Sq);
            int64_t n_blk = (Skv + lp - 1) / lp;

            for (int g = 0; g < n2; g++) {
                /* the key set of (t, g): listed blocks, each once, causal */
                const int32_t* list = sel + (t * n2 + g) * (int64_t)count;
                int64_t nk = 0;
                for (int c = 0; c < count; c++) {
                    int64_t j = list[c];
                    if (j < 0 || j >= n_blk) continue;
                    int seen = 0;
                    for (int c2 = 0; c2 < c; c2++)
                        if (list[c2] == list[c]) seen = 1;
                    if (seen) continue;
                    for (int64_t p = j * lp; p < (j + 1) * lp && p < Skv; p++)
                        if (p <= tpos) keys[nk++] = p;
                }
                for (int hh = 0; hh < G; hh++) {
                    int h = g * G + hh;
                    double* o = out + (r * n1 + h) * (int64_t)d2;
                    for (int e = 0; e < d2; e++) o[e] = 0.0;
                    if (nk == 0) {
                        lse[r * n1 + h] = -INFINITY;
                        continue;
                    }
                    const double* qr = q + ((q_compact ? r : t) * n1 + h) * (int64_t)d1;
                    for (int64_t i = 0; i < nk; i++) {
                        const double* kr = k + ((k0 + keys[i]) * n2 + g) * (int64_t)d1;
                        double acc = 0.0;
                        for (int e = 0; e < d1; e++) acc += qr[e] * kr[e];
                        sc[i] = scale * acc;
                    }
                    double m = sc[0];
                    for (int64_t i = 1; i < nk; i++) if (sc[i] > m) m = sc[i];
                    double L = 0.0;
                    for (int64_t i = 0; i < nk; i++) L += exp(sc[i] - m);
                    for (int64_t i = 0; i < nk; i++) {
                        const double pw = exp(sc[i] - m) / L;
                        const double* vr = v + ((k0 + keys[i]) * n2 + g) * (int64_t)d2;
                        for (int e = 0; e < d2; e++) o[e] += pw * vr[e];
                    }
                    lse[r * n1 + h] = m + log(L);
                }
            }
        }
        free(keys); free(sc);
    }
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

/* ------------------------------------------------------------------------- */
/* Backward of [ATT] steps 1-3: the gradient of attention_out with respect   */
/* to q, kcmp and vcmp (the importance scores and the top-k are indices and  */
/* carry none).  Derived from the forward definition: for query row t, head  */
/* h of group g and its attended blocks i (visible by the causal rule and    */
/* not removed by amask), with s_i = scale q.k_i, P = softmax(s), O = sum    */
/* P_i v_i and the incoming dO:                                              */
/*   dv_i += P_i dO                                                          */
/*   dP_i  = dO . v_i,   dS_i = P_i (dP_i - sum_j P_j dP_j)                  */
/*   dq    = scale sum_i dS_i k_i,   dk_i += scale dS_i q                    */
/* A row that attends to nothing contributes nothing.  dq (T1, N1, D1);      */
/* dkc (Tc, N2, D1) and dvc (Tc, N2, D2) sum over the rows and the G heads  */
/* of each group.  Single-threaded (the sums are shared between rows).       */
/* ------------------------------------------------------------------------- */
int oracle_compress_attention_backward(const double* q, const double* kc, const double* vc,
                                       const double* dout, double scale, int n1, int n2,
                                       int d1, int d2, int l, int d,
                                       const int32_t* cu_q, const int32_t* cu_cmp, int batch,
                                       const uint8_t* amask, int64_t am_s2,
                                       double* dq, double* dkc, double* dvc)
{
    if (n2 <= 0 || n1 % n2 != 0) return -1;
    const int G = n1 / n2;
    const int64_t T1 = batch ? cu_q[batch - 1] : 0;
    const int64_t Tc = batch ? cu_cmp[batch - 1] : 0;
    for (int64_t x = 0; x < T1 * n1 * d1; x++) dq[x] = 0.0;
    for (int64_t x = 0; x < Tc * n2 * d1; x++) dkc[x] = 0.0;
    for (int64_t x = 0; x < Tc * n2 * d2; x++) dvc[x] = 0.0;
    int max_cmp = 1;
    for (int s = 0; s < batch; s++) {
        int nc = cu_cmp[s] - (s ? cu_cmp[s - 1] : 0);
        if (nc > max_cmp) max_cmp = nc;
    }
    double* sc = (double*)malloc(sizeof(double) * (size_t)max_cmp);
    double* P = (double*)malloc(sizeof(double) * (size_t)max_cmp);
    double* dP = (double*)malloc(sizeof(double) * (size_t)max_cmp);
    char* att = (char*)malloc((size_t)max_cmp);
    for (int s = 0; s < batch; s++) {
        const int64_t q0 = s ? cu_q[s - 1] : 0, c0 = s ? cu_cmp[s - 1] : 0;
        const int64_t Sq = cu_q[s] - q0;
        const int n_cmp = (int)(cu_cmp[s] - c0);
        int64_t off = 0;
        if (n_cmp > 0) {
            off = (int64_t)(n_cmp - 1) * d + l - Sq;
            if (off < 0) off = 0;
        }
        for (int64_t tl = 0; tl < Sq; tl++) {
            const int64_t t = q0 + tl, tpos = tl + off;
            int n_att = 0;
            for (int i = 0; i < n_cmp; i++) {
                att[i] = ((int64_t)i * d + l - 1 <= tpos) && !(amask && amask[tl * am_s2 + i]);
                n_att += att[i];
            }
            if (n_att == 0) continue;
            for (int h = 0; h < n1; h++) {
                const int g = h / G;
                const double* qr = q + (t * n1 + h) * (int64_t)d1;
                const double* dor = dout + (t * n1 + h) * (int64_t)d2;
                double m = -INFINITY;
                for (int i = 0; i < n_cmp; i++) {
                    if (!att[i]) continue;
                    const double* kr = kc + ((c0 + i) * n2 + g) * (int64_t)d1;
                    double acc = 0.0;
                    for (int e = 0; e < d1; e++) acc += qr[e] * kr[e];
                    sc[i] = scale * acc;
                    if (sc[i] > m) m = sc[i];
                }
                double L = 0.0;
                for (int i = 0; i < n_cmp; i++) if (att[i]) L += exp(sc[i] - m);
                double delta = 0.0;
                for (int i = 0; i < n_cmp; i++) {
                    if (!att[i]) continue;
                    P[i] = exp(sc[i] - m) / L;
                    const double* vr = vc + ((c0 + i) * n2 + g) * (int64_t)d2;
                    double acc = 0.0;
                    for (int e = 0; e < d2; e++) acc += dor[e] * vr[e];
                    dP[i] = acc;
                    delta += P[i] * acc;
                }
                double* dqr = dq + (t * n1 + h) * (int64_t)d1;
                for (int i = 0; i < n_cmp; i++) {
                    if (!att[i]) continue;
                    const double dS = P[i] * (dP[i] - delta);
                    const double* kr = kc + ((c0 + i) * n2 + g) * (int64_t)d1;
                    double* dkr = dkc + ((c0 + i) * n2 + g) * (int64_t)d1;
                    double* dvr = dvc + ((c0 + i) * n2 + g) * (int64_t)d2;
                    for (int e = 0; e < d1; e++) {
                        dqr[e] += scale * dS * kr[e];
                        dkr[e] += scale * dS * qr[e];
                    }
                    for (int e = 0; e < d2; e++) dvr[e] += P[i] * dor[e];
                }
            }
        }
    }
    free(sc); free(P); free(dP); free(att);
    return 0;
}

/* Backward of the compression ([NSA-C] Formula, phi = weighted window sum): */
/* out[c0+i, n, :] = sum_{j<l} w[j, n] x[s0 + i d + j, n, :] is linear in x  */
/* and w, so dx[s0 + i d + j, n, :] += w[j, n] dout[c0+i, n, :] and          */
/* dw[j, n] += x[s0 + i d + j, n, :] . dout[c0+i, n, :].  dx (T, N2, D) and  */
/* dw (l, N2) are zeroed here; for K and V sharing w, dw is their sum.       */
int oracle_compress_backward(const double* x, const double* w, const double* dout, int l, int d,
                             const int32_t* cu, int batch, int n2, int dim, double* dx, double* dw)
{
    const int64_t T = batch ? cu[batch - 1] : 0;
    for (int64_t e = 0; e < T * n2 * dim; e++) dx[e] = 0.0;
    for (int e = 0; e < l * n2; e++) dw[e] = 0.0;
    int64_t c0 = 0;
    for (int s = 0; s < batch; s++) {
        const int64_t s0 = s ? cu[s - 1] : 0, S = cu[s] - s0;
        const int64_t n_cmp = (S < l) ? 0 : (S - l) / d + 1;
        for (int64_t i = 0; i < n_cmp; i++) {
            for (int j = 0; j < l; j++) {
                const int64_t row = s0 + i * d + j;
                for (int n = 0; n < n2; n++) {
                    const double* gr = dout + ((c0 + i) * n2 + n) * (int64_t)dim;
                    const double* xr = x + (row * n2 + n) * (int64_t)dim;
                    double* dxr = dx + (row * n2 + n) * (int64_t)dim;
                    double acc = 0.0;
                    for (int e = 0; e < dim; e++) {
                        dxr[e] += w[j * n2 + n] * gr[e];
                        acc += xr[e] * gr[e];
                    }
                    dw[j * n2 + n] += acc;
                }
            }
        }
        c0 += n_cmp;
    }
    return 0;
}
