/*
 * oracle.c -- TEST INFRASTRUCTURE ONLY.  The plain, slow, single-threaded
 * fp64 CPU statement of what sparse-graph causal attention computes.  Only
 * tests/, the smoke check and the bench's CPU-baseline leg load it; the
 * library never does.  It shares no code, header or table with the CUDA path.
 *
 * Sources (web pages; section names as printed on them):
 *  - "SpatialLM-Mini sped up training with a 16K context by 2.47x on an
 *    RTX 3050", section "How tokens choose whom to listen to": the allowed
 *    positions of a token are itself, a few nearby predecessors and the
 *    positions at distance 1, 2, 4, 8, ...; no position ahead; the list is
 *    fixed in advance.
 *  - "MiniGPT (Part 6)", section "A mask is not enough", first listing: the
 *    window keeps key j for query i when j <= i and i - j < w.  Second
 *    listing (chunked_swa): scores are (q . k) * scale, masked, then softmax
 *    over the kept keys, then multiplied with V.
 *  - "Longer Attention Span: Increasing Transformer Context Length with
 *    Sparse Graph Processing Techniques", Abstract: tokens are graph nodes,
 *    the mask gives the edges, and only the needed (edge) computations are
 *    performed.
 *
 * Everything is written as the plain definition: per query, loop over its
 * neighbour list, fp64 arithmetic, no blocking, no reordering.
 *
 * Element types of the attention inputs: 0 = bf16 (raw uint16 bits),
 * 1 = fp32, 2 = fp64.  Conversions to double are exact.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_BAD_ROWPTR 1
#define OR_LOOKAHEAD 2
#define OR_NEGATIVE 3
#define OR_BAD_ARG 4
#define OR_NOMEM 5

/* ---------- element access ---------- */

static double elem(const void *base, int dtype, int64_t idx) {
    if (dtype == 0) {
        uint16_t h = ((const uint16_t *)base)[idx];
        uint32_t bits = ((uint32_t)h) << 16; /* bf16 is the top half of fp32 */
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    if (dtype == 1) return (double)((const float *)base)[idx];
    return ((const double *)base)[idx];
}

static int cmp_i32(const void *a, const void *b) {
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* ---------- graph: the fixed neighbour set ---------- */

/* Number of neighbours of query i: the window {i-W+1..i} clipped at 0,
 * plus the distances 2^k (k from exps[]) that reach a position >= 0 and are
 * not already inside the window.  Written by listing the set and counting. */
static int64_t structured_row(int64_t i, int32_t W, const int32_t *exps, int32_t n_exps,
                              int32_t *buf /* may be NULL */) {
    int64_t cnt = 0;
    int64_t lo = i - (int64_t)W + 1;
    if (lo < 0) lo = 0;
    for (int64_t j = lo; j <= i; ++j) {
        if (buf) buf[cnt] = (int32_t)j;
        ++cnt;
    }
    /* distance links; each distinct distance appears once */
    for (int32_t a = 0; a < n_exps; ++a) {
        int32_t k = exps[a];
        if (k < 0 || k > 62) continue;
        int dup = 0;
        for (int32_t b = 0; b < a; ++b)
            if (exps[b] == k) dup = 1;
        if (dup) continue;
        int64_t dist = (int64_t)1 << k;
        int64_t j = i - dist;
        if (j < 0) continue;          /* no position before the start */
        if (j >= lo) continue;        /* already in the window */
        if (buf) buf[cnt] = (int32_t)j;
        ++cnt;
    }
    if (buf) qsort(buf, (size_t)cnt, sizeof(int32_t), cmp_i32);
    return cnt;
}

int64_t oracle_graph_structured_nnz(int64_t T, int32_t W, const int32_t *exps, int32_t n_exps) {
    int64_t nnz = 0;
    for (int64_t i = 0; i < T; ++i) nnz += structured_row(i, W, exps, n_exps, NULL);
    return nnz;
}

/* rowptr[T+1], colidx[nnz]; each row ascending. */
int oracle_graph_structured(int64_t T, int32_t W, const int32_t *exps, int32_t n_exps,
                            int64_t *rowptr, int32_t *colidx) {
    if (T < 0 || W < 1) return OR_BAD_ARG;
    rowptr[0] = 0;
    for (int64_t i = 0; i < T; ++i) {
        int64_t c = structured_row(i, W, exps, n_exps, colidx + rowptr[i]);
        rowptr[i + 1] = rowptr[i] + c;
    }
    return OR_OK;
}

/* The lists of selected rows only (for sampled checks of long sequences):
 * rows[0..n), rowptr[n+1]; pass colidx = NULL to get rowptr alone. */
int oracle_graph_structured_rows(int64_t n, const int64_t *rows, int32_t W, const int32_t *exps,
                                 int32_t n_exps, int64_t *rowptr, int32_t *colidx) {
    if (n < 0 || W < 1) return OR_BAD_ARG;
    rowptr[0] = 0;
    for (int64_t r = 0; r < n; ++r) {
        if (rows[r] < 0) return OR_BAD_ARG;
        int64_t c = structured_row(rows[r], W, exps, n_exps, colidx ? colidx + rowptr[r] : NULL);
        rowptr[r + 1] = rowptr[r] + c;
    }
    return OR_OK;
}

/* Normalise a caller's neighbour lists: per row sort ascending and drop
 * repeats; reject a key after the query (no look-ahead), a negative key and
 * a malformed row pointer.  out_rowptr[T+1], out_colidx[<= nnz_in].
 * Returns the status; *nnz_out gets the normalised edge count. */
int oracle_graph_normalize(int64_t T, const int64_t *rowptr, const int32_t *colidx,
                           int64_t *out_rowptr, int32_t *out_colidx, int64_t *nnz_out) {
    if (T < 0) return OR_BAD_ARG;
    if (rowptr[0] != 0) return OR_BAD_ROWPTR;
    for (int64_t i = 0; i < T; ++i)
        if (rowptr[i + 1] < rowptr[i]) return OR_BAD_ROWPTR;
    for (int64_t i = 0; i < T; ++i)
        for (int64_t e = rowptr[i]; e < rowptr[i + 1]; ++e) {
            if (colidx[e] < 0) return OR_NEGATIVE;
            if ((int64_t)colidx[e] > i) return OR_LOOKAHEAD;
        }
    int64_t w = 0;
    out_rowptr[0] = 0;
    for (int64_t i = 0; i < T; ++i) {
        int64_t n = rowptr[i + 1] - rowptr[i];
        int32_t *row = out_colidx + w;
        memcpy(row, colidx + rowptr[i], (size_t)n * sizeof(int32_t));
        qsort(row, (size_t)n, sizeof(int32_t), cmp_i32);
        int64_t u = 0;
        for (int64_t e = 0; e < n; ++e)
            if (u == 0 || row[u - 1] != row[e]) row[u++] = row[e];
        w += u;
        out_rowptr[i + 1] = w;
    }
    *nnz_out = w;
    return OR_OK;
}

/* Transpose: for key j, the queries i with j in N(i), ascending in i. */
int oracle_graph_reverse(int64_t T, const int64_t *rowptr, const int32_t *colidx,
                         int64_t *rev_rowptr, int32_t *rev_colidx) {
    int64_t nnz = rowptr[T];
    int64_t *fill = (int64_t *)calloc((size_t)T + 1, sizeof(int64_t));
    if (!fill) return OR_NOMEM;
    for (int64_t e = 0; e < nnz; ++e) fill[colidx[e] + 1] += 1;
    rev_rowptr[0] = 0;
    for (int64_t j = 0; j < T; ++j) rev_rowptr[j + 1] = rev_rowptr[j] + fill[j + 1];
    for (int64_t j = 0; j < T; ++j) fill[j] = rev_rowptr[j];
    for (int64_t i = 0; i < T; ++i) /* ascending i keeps each list sorted */
        for (int64_t e = rowptr[i]; e < rowptr[i + 1]; ++e) {
            int32_t j = colidx[e];
            rev_colidx[fill[j]++] = (int32_t)i;
        }
    free(fill);
    return OR_OK;
}

/* ---------- attention over the graph ---------- */

/* Exact copy of n elements of any input type into a new fp64 array. */
static double *to_f64(const void *base, int dtype, int64_t n) {
    double *a = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    if (!a) return NULL;
    for (int64_t x = 0; x < n; ++x) a[x] = elem(base, dtype, x);
    return a;
}

/* One query row: s_j = scale * q.k_j for j in its list; m = max s;
 * l = sum exp(s_j - m); out = sum exp(s_j - m) v_j / l; lse = m + ln l.
 * An empty list gives out = 0 and lse = -inf. */
static void row_forward(int32_t D, const double *q, int64_t qrow, const double *k,
                        const double *v, const int32_t *nbr, int64_t deg, double scale,
                        double *s /* scratch[deg] */, double *out, double *lse) {
    for (int32_t d = 0; d < D; ++d) out[d] = 0.0;
    if (deg == 0) {
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int64_t e = 0; e < deg; ++e) {
        int64_t j = nbr[e];
        double dot = 0.0;
        for (int32_t d = 0; d < D; ++d) dot += q[qrow * D + d] * k[j * D + d];
        s[e] = scale * dot;
        if (s[e] > m) m = s[e];
    }
    double l = 0.0;
    for (int64_t e = 0; e < deg; ++e) l += exp(s[e] - m);
    for (int64_t e = 0; e < deg; ++e) {
        int64_t j = nbr[e];
        double p = exp(s[e] - m) / l;
        for (int32_t d = 0; d < D; ++d) out[d] += p * v[j * D + d];
    }
    *lse = m + log(l);
}

static int64_t max_degree(int64_t nq, const int64_t *rowptr) {
    int64_t mx = 0;
    for (int64_t i = 0; i < nq; ++i)
        if (rowptr[i + 1] - rowptr[i] > mx) mx = rowptr[i + 1] - rowptr[i];
    return mx;
}

/* Forward for nq query rows.  Query row r is q[r*D..]; its neighbours are
 * colidx[rowptr[r]..rowptr[r+1]), indexing rows of k and v.  out[nq*D],
 * lse[nq] (natural log). */
int oracle_attn_fwd(int64_t nq, int32_t D, int dtype, const void *q, const void *k,
                    const void *v, const int64_t *rowptr, const int32_t *colidx, double scale,
                    double *out, double *lse) {
    if (nq < 0 || D < 1 || dtype < 0 || dtype > 2) return OR_BAD_ARG;
    int64_t nk = 0; /* key rows referenced: 1 + the largest index */
    for (int64_t e = 0; e < rowptr[nq]; ++e)
        if ((int64_t)colidx[e] + 1 > nk) nk = (int64_t)colidx[e] + 1;
    double *s = (double *)malloc(sizeof(double) * (size_t)(max_degree(nq, rowptr) + 1));
    double *qd = to_f64(q, dtype, nq * D), *kd = to_f64(k, dtype, nk * D);
    double *vd = to_f64(v, dtype, nk * D);
    int st = OR_OK;
    if (!s || !qd || !kd || !vd) {
        st = OR_NOMEM;
    } else {
        for (int64_t r = 0; r < nq; ++r)
            row_forward(D, qd, r, kd, vd, colidx + rowptr[r], rowptr[r + 1] - rowptr[r], scale, s,
                        out + r * D, lse + r);
    }
    free(s);
    free(qd);
    free(kd);
    free(vd);
    return st;
}

/* Backward of the forward above for upstream gradient dout[nq*D].
 * For each query i (its own fp64 forward recomputed):
 *   P_ij = exp(s_ij - lse_i), dP_ij = dO_i . v_j, Delta_i = dO_i . out_i,
 *   dS_ij = P_ij (dP_ij - Delta_i),
 *   dQ_i += scale * dS_ij k_j,  dK_j += scale * dS_ij q_i,  dV_j += P_ij dO_i.
 * dq[nq*D]; dk, dv [nk*D] are overwritten (zeroed first).  dK_j and dV_j
 * are complete for every key whose queries are all among the nq rows. */
int oracle_attn_bwd(int64_t nq, int64_t nk, int32_t D, int dtype, const void *q, const void *k,
                    const void *v, const void *dout, const int64_t *rowptr, const int32_t *colidx,
                    double scale, double *dq, double *dk, double *dv) {
    if (nq < 0 || nk < 0 || D < 1 || dtype < 0 || dtype > 2) return OR_BAD_ARG;
    int64_t mdeg = max_degree(nq, rowptr);
    double *s = (double *)malloc(sizeof(double) * (size_t)(mdeg + 1));
    double *o = (double *)malloc(sizeof(double) * (size_t)D);
    double *qd = to_f64(q, dtype, nq * D), *kd = to_f64(k, dtype, nk * D);
    double *vd = to_f64(v, dtype, nk * D), *dod = to_f64(dout, dtype, nq * D);
    int st = OR_OK;
    if (!s || !o || !qd || !kd || !vd || !dod) {
        st = OR_NOMEM;
        goto done;
    }
    memset(dq, 0, sizeof(double) * (size_t)(nq * D));
    memset(dk, 0, sizeof(double) * (size_t)(nk * D));
    memset(dv, 0, sizeof(double) * (size_t)(nk * D));
    for (int64_t i = 0; i < nq; ++i) {
        const int32_t *nbr = colidx + rowptr[i];
        int64_t deg = rowptr[i + 1] - rowptr[i];
        double lse;
        row_forward(D, qd, i, kd, vd, nbr, deg, scale, s, o, &lse);
        if (deg == 0) continue;
        double delta = 0.0;
        for (int32_t d = 0; d < D; ++d) delta += dod[i * D + d] * o[d];
        for (int64_t e = 0; e < deg; ++e) {
            int64_t j = nbr[e];
            double p = exp(s[e] - lse);
            double dp = 0.0;
            for (int32_t d = 0; d < D; ++d) dp += dod[i * D + d] * vd[j * D + d];
            double ds = p * (dp - delta);
            for (int32_t d = 0; d < D; ++d) {
                dq[i * D + d] += scale * ds * kd[j * D + d];
                dk[j * D + d] += scale * ds * qd[i * D + d];
                dv[j * D + d] += p * dod[i * D + d];
            }
        }
    }
done:
    free(s);
    free(o);
    free(qd);
    free(kd);
    free(vd);
    free(dod);
    return st;
}

/* ---------- learned-coordinate scoring on the same graph ----------
 * "SpatialLM-Mini ...", section "How tokens choose whom to listen to": the
 * hidden state of each token gives a learnable three-dimensional query
 * coordinate and key coordinate, and the shorter the distance between them,
 * the higher the weight of the edge; the neighbour list stays fixed.  The
 * page does not spell out the "additional learnable parameters" that adjust
 * the weight, so the plainest pinnable form is taken: one positive scale,
 *     s_ij = -scale * |a_i - c_j|^2      for j in N(i)
 * (a_i: query coordinate, c_j: key coordinate, both 3 values), softmax over
 * N(i), out_i = sum_j p_ij v_j, lse_i = ln sum_j exp(s_ij).
 * Coordinates are read with element type cdtype (1 fp32, 2 fp64), v and dout
 * with dtype (0 bf16, 1 fp32, 2 fp64).  Loops as in the dot-product
 * statement above: per query, over its neighbour list, fp64. */
static void row_forward_dist(int32_t D, const double *a, int64_t qrow, const double *c,
                             const double *v, const int32_t *nbr, int64_t deg, double scale,
                             double *w /* scratch[deg] */, double *out, double *lz) {
    for (int32_t d = 0; d < D; ++d) out[d] = 0.0;
    if (deg == 0) {
        *lz = -INFINITY; /* empty list */
        return;
    }
    double mx = -INFINITY;
    for (int64_t e = 0; e < deg; ++e) {
        int64_t j = nbr[e];
        double dist2 = 0.0;
        for (int x = 0; x < 3; ++x) {
            double diff = a[qrow * 3 + x] - c[j * 3 + x];
            dist2 += diff * diff;
        }
        w[e] = -scale * dist2;
        if (w[e] > mx) mx = w[e];
    }
    double z = 0.0;
    for (int64_t e = 0; e < deg; ++e) z += exp(w[e] - mx);
    for (int64_t e = 0; e < deg; ++e) {
        int64_t j = nbr[e];
        double pw = exp(w[e] - mx) / z;
        for (int32_t d = 0; d < D; ++d) out[d] += pw * v[j * D + d];
    }
    *lz = mx + log(z);
}

/* Forward: a [nq*3], c [nk*3] coordinates; v [nk*D]; out [nq*D], lse [nq]. */
int oracle_dist_fwd(int64_t nq, int32_t D, int cdtype, int dtype, const void *a, const void *c,
                    const void *v, const int64_t *rowptr, const int32_t *colidx, double scale,
                    double *out, double *lse) {
    if (nq < 0 || D < 1 || cdtype < 1 || cdtype > 2 || dtype < 0 || dtype > 2) return OR_BAD_ARG;
    int64_t nk = 0;
    for (int64_t e = 0; e < rowptr[nq]; ++e)
        if ((int64_t)colidx[e] + 1 > nk) nk = (int64_t)colidx[e] + 1;
    double *s = (double *)malloc(sizeof(double) * (size_t)(max_degree(nq, rowptr) + 1));
    double *ad = to_f64(a, cdtype, nq * 3), *cd = to_f64(c, cdtype, nk * 3);
    double *vd = to_f64(v, dtype, nk * D);
    int st = OR_OK;
    if (!s || !ad || !cd || !vd) {
        st = OR_NOMEM;
    } else {
        for (int64_t r = 0; r < nq; ++r)
            row_forward_dist(D, ad, r, cd, vd, colidx + rowptr[r], rowptr[r + 1] - rowptr[r],
                             scale, s, out + r * D, lse + r);
    }
    free(s);
    free(ad);
    free(cd);
    free(vd);
    return st;
}

/* Backward for upstream gradient dout[nq*D].  With the same P, dP, Delta and
 * dS = P (dP - Delta) as the dot-product statement, and
 *     d s_ij / d a_i = -2 scale (a_i - c_j),   d s_ij / d c_j = +2 scale (a_i - c_j):
 *   da_i += dS_ij * (-2 scale (a_i - c_j)),  dc_j -= the same,  dv_j += P_ij dO_i.
 * da [nq*3], dc [nk*3], dv [nk*D] are overwritten (zeroed first). */
int oracle_dist_bwd(int64_t nq, int64_t nk, int32_t D, int cdtype, int dtype, const void *a,
                    const void *c, const void *v, const void *dout, const int64_t *rowptr,
                    const int32_t *colidx, double scale, double *da, double *dc, double *dv) {
    if (nq < 0 || nk < 0 || D < 1 || cdtype < 1 || cdtype > 2 || dtype < 0 || dtype > 2)
        return OR_BAD_ARG;
    int64_t mdeg = max_degree(nq, rowptr);
    double *s = (double *)malloc(sizeof(double) * (size_t)(mdeg + 1));
    double *o = (double *)malloc(sizeof(double) * (size_t)D);
    double *ad = to_f64(a, cdtype, nq * 3), *cd = to_f64(c, cdtype, nk * 3);
    double *vd = to_f64(v, dtype, nk * D), *dod = to_f64(dout, dtype, nq * D);
    int st = OR_OK;
    if (!s || !o || !ad || !cd || !vd || !dod) {
        st = OR_NOMEM;
        goto done;
    }
    memset(da, 0, sizeof(double) * (size_t)(nq * 3));
    memset(dc, 0, sizeof(double) * (size_t)(nk * 3));
    memset(dv, 0, sizeof(double) * (size_t)(nk * D));
    for (int64_t i = 0; i < nq; ++i) {
        const int32_t *nbr = colidx + rowptr[i];
        int64_t deg = rowptr[i + 1] - rowptr[i];
        double lz;
        row_forward_dist(D, ad, i, cd, vd, nbr, deg, scale, s, o, &lz);
        if (deg == 0) continue;
        double dlt = 0.0; /* Delta_i */
        for (int32_t d = 0; d < D; ++d) dlt += dod[i * D + d] * o[d];
        for (int64_t e = 0; e < deg; ++e) {
            int64_t j = nbr[e];
            double pe = exp(s[e] - lz);
            double dpe = 0.0;
            for (int32_t d = 0; d < D; ++d) dpe += dod[i * D + d] * vd[j * D + d];
            double dse = pe * (dpe - dlt);
            for (int x = 0; x < 3; ++x) {
                double g = dse * (-2.0 * scale * (ad[i * 3 + x] - cd[j * 3 + x]));
                da[i * 3 + x] += g;
                dc[j * 3 + x] -= g;
            }
            for (int32_t d = 0; d < D; ++d) dv[j * D + d] += pe * dod[i * D + d];
        }
    }
done:
    free(s);
    free(o);
    free(ad);
    free(cd);
    free(vd);
    free(dod);
    return st;
}
