/*
 * na2d_oracle.c -- fp64 CPU oracle for 2D (dilated) neighborhood attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct
 * reference that the CUDA library is checked against.  Only the test suite,
 * the smoke check and the benchmark's CPU-baseline leg may load it.  It shares
 * no code, header, table or helper with the CUDA library in
 * neighborhood_attention_na2d_b200/csrc, and it never calls into it.
 *
 * What it computes (sources are the web pages on NAT / DiNAT):
 *   - "Neighborhood Attention Transformer" (GitHub README mirror), figure
 *     caption under the abstract: every query attends to its nearest
 *     neighbourhood; with the neighbourhood as large as the image this is plain
 *     dot-product self attention; the image edges are special cases.
 *   - "Dilated Neighborhood Attention Transformer" (HF docs) overview and the
 *     gitcode DiNAT article, section "DiNAT 的核心思想": DiNA samples the
 *     neighbourhood every d pixels; the layer is
 *         scores = natten2dqkrpb(q, k, rpb, kernel_size, dilation)
 *         probs  = softmax(scores, dim=-1)
 *         out    = natten2dav(probs, v, kernel_size, dilation)
 *   - The pages never write the window rule out.  The rule used here is the
 *     NATTEN clamp rule stated in the problem statement, per axis, for a
 *     coordinate i on an axis of length L, kernel size k, dilation d, r = k/2:
 *         g  = i mod d,  i' = floor(i / d),  Lg = ceil((L - g) / d)
 *         s' = clamp(i' - r, 0, Lg - k)
 *         key_t = g + d * (s' + t),  t = 0 .. k-1
 *     and the relative position bias of key t is rpb[.., s' + t - i' + k - 1].
 *   - score = (q . k) / sqrt(D) + rpb[h, dy, dx]; softmax over the k*k
 *     neighbours; out = sum_n p_n v_n.
 *
 * Layouts: q, k, v, out are [B, heads, H, W, D] row-major fp64; rpb is
 * [heads, 2k-1, 2k-1] fp64 or NULL (zero bias); attn is [B, heads, H, W, k*k]
 * with neighbour n = ty * k + tx (row-major over the window).
 *
 * No tiling, no fusion, no reordering: one query at a time, in the order the
 * pages give (scores, then softmax, then the weighted sum).  The optional
 * thread count only splits the independent (b, head) slices across threads.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------------------
 * The per-axis neighbourhood rule.  Returns 0 on success, -1 when the axis is
 * too short for the window (some dilation group shorter than k).
 * ------------------------------------------------------------------------- */
int oracle_axis_window(int L, int k, int d, int i, int *g_out, int *ip_out,
                       int *start_out)
{
    if (L < 1 || k < 1 || d < 1 || i < 0 || i >= L) return -1;
    int r = k / 2;
    int g = i % d;
    int ip = i / d;
    int Lg = (L - g + d - 1) / d;          /* ceil((L - g) / d) */
    if (Lg < k) return -1;
    int s = ip - r;
    if (s < 0) s = 0;                      /* clamp(i' - r, 0, Lg - k) */
    if (s > Lg - k) s = Lg - k;
    *g_out = g;
    *ip_out = ip;
    *start_out = s;
    return 0;
}

/* Lists the k key coordinates of query coordinate i along one axis, and the
 * k bias indices (s' + t - i' + k - 1) that go with them. */
int oracle_axis_neighbors(int L, int k, int d, int i, int *keys, int *bias_idx)
{
    int g, ip, s;
    if (oracle_axis_window(L, k, d, i, &g, &ip, &s) != 0) return -1;
    for (int t = 0; t < k; ++t) {
        keys[t] = g + d * (s + t);
        bias_idx[t] = s + t - ip + k - 1;
    }
    return 0;
}

typedef struct {
    int B, heads, H, W, D, k, d;
} oracle_shape;

static int shape_ok(const oracle_shape *p)
{
    if (p->B < 0 || p->heads < 0 || p->H < 1 || p->W < 1 || p->D < 1) return 0;
    if (p->k < 1 || p->d < 1) return 0;
    /* every dilation group must hold at least k positions on both axes */
    if (p->H / p->d < p->k || p->W / p->d < p->k) return 0;
    return 1;
}

/* ---------------------------------------------------------------------------
 * Stage 1: scores (natten2dqkrpb).  attn[b,h,i,j,n] = q.k_n / sqrt(D) + bias.
 * ------------------------------------------------------------------------- */
static void qk_rpb_slice(const oracle_shape *p, int bh, const double *q,
                         const double *kk, const double *rpb, double *attn)
{
    const int H = p->H, W = p->W, D = p->D, k = p->k, d = p->d;
    const int h = bh % p->heads;
    const int nb = 2 * k - 1;
    const double scale = 1.0 / sqrt((double)D);
    const double *qs = q + (size_t)bh * H * W * D;
    const double *ks = kk + (size_t)bh * H * W * D;
    double *as = attn + (size_t)bh * H * W * k * k;
    int *ky = malloc(sizeof(int) * k), *by = malloc(sizeof(int) * k);
    int *kx = malloc(sizeof(int) * k), *bx = malloc(sizeof(int) * k);
    for (int i = 0; i < H; ++i) {
        oracle_axis_neighbors(H, k, d, i, ky, by);
        for (int j = 0; j < W; ++j) {
            oracle_axis_neighbors(W, k, d, j, kx, bx);
            const double *qv = qs + ((size_t)i * W + j) * D;
            double *row = as + ((size_t)i * W + j) * k * k;
            for (int ty = 0; ty < k; ++ty) {
                for (int tx = 0; tx < k; ++tx) {
                    const double *kv = ks + ((size_t)ky[ty] * W + kx[tx]) * D;
                    double dot = 0.0;
                    for (int c = 0; c < D; ++c) dot += qv[c] * kv[c];
                    double bias = 0.0;
                    if (rpb) bias = rpb[((size_t)h * nb + by[ty]) * nb + bx[tx]];
                    row[ty * k + tx] = dot * scale + bias;
                }
            }
        }
    }
    free(ky); free(by); free(kx); free(bx);
}

/* ---------------------------------------------------------------------------
 * Stage 2: softmax over the last dimension (the k*k neighbours), in place.
 * ------------------------------------------------------------------------- */
static void softmax_slice(const oracle_shape *p, int bh, double *attn)
{
    const int n = p->k * p->k;
    const size_t rows = (size_t)p->H * p->W;
    double *as = attn + (size_t)bh * rows * n;
    for (size_t r = 0; r < rows; ++r) {
        double *row = as + r * n;
        double m = row[0];
        for (int t = 1; t < n; ++t)
            if (row[t] > m) m = row[t];
        double sum = 0.0;
        for (int t = 0; t < n; ++t) {
            row[t] = exp(row[t] - m);
            sum += row[t];
        }
        for (int t = 0; t < n; ++t) row[t] /= sum;
    }
}

/* ---------------------------------------------------------------------------
 * Stage 3: weighted sum of values (natten2dav).  out[.., c] = sum_n p_n v_n[c].
 * ------------------------------------------------------------------------- */
static void av_slice(const oracle_shape *p, int bh, const double *attn,
                     const double *v, double *out)
{
    const int H = p->H, W = p->W, D = p->D, k = p->k, d = p->d;
    const double *as = attn + (size_t)bh * H * W * k * k;
    const double *vs = v + (size_t)bh * H * W * D;
    double *os = out + (size_t)bh * H * W * D;
    int *ky = malloc(sizeof(int) * k), *by = malloc(sizeof(int) * k);
    int *kx = malloc(sizeof(int) * k), *bx = malloc(sizeof(int) * k);
    for (int i = 0; i < H; ++i) {
        oracle_axis_neighbors(H, k, d, i, ky, by);
        for (int j = 0; j < W; ++j) {
            oracle_axis_neighbors(W, k, d, j, kx, bx);
            const double *row = as + ((size_t)i * W + j) * k * k;
            double *o = os + ((size_t)i * W + j) * D;
            for (int c = 0; c < D; ++c) o[c] = 0.0;
            for (int ty = 0; ty < k; ++ty)
                for (int tx = 0; tx < k; ++tx) {
                    const double pw = row[ty * k + tx];
                    const double *vv = vs + ((size_t)ky[ty] * W + kx[tx]) * D;
                    for (int c = 0; c < D; ++c) o[c] += pw * vv[c];
                }
        }
    }
    free(ky); free(by); free(kx); free(bx);
}

/* ---------------------------------------------------------------------------
 * The fused definition: the three stages above, one query at a time, with the
 * k*k scores kept in a small per-query buffer instead of a full attn tensor.
 * ------------------------------------------------------------------------- */
static void forward_slice(const oracle_shape *p, int bh, const double *q,
                          const double *kk, const double *v, const double *rpb,
                          double *out)
{
    const int H = p->H, W = p->W, D = p->D, k = p->k, d = p->d;
    const int h = bh % p->heads;
    const int nb = 2 * k - 1;
    const double scale = 1.0 / sqrt((double)D);
    const size_t base = (size_t)bh * H * W * D;
    int *ky = malloc(sizeof(int) * k), *by = malloc(sizeof(int) * k);
    int *kx = malloc(sizeof(int) * k), *bx = malloc(sizeof(int) * k);
    double *sc = malloc(sizeof(double) * k * k);
    for (int i = 0; i < H; ++i) {
        oracle_axis_neighbors(H, k, d, i, ky, by);
        for (int j = 0; j < W; ++j) {
            oracle_axis_neighbors(W, k, d, j, kx, bx);
            const double *qv = q + base + ((size_t)i * W + j) * D;
            /* scores */
            for (int ty = 0; ty < k; ++ty)
                for (int tx = 0; tx < k; ++tx) {
                    const double *kv = kk + base + ((size_t)ky[ty] * W + kx[tx]) * D;
                    double dot = 0.0;
                    for (int c = 0; c < D; ++c) dot += qv[c] * kv[c];
                    double bias = 0.0;
                    if (rpb) bias = rpb[((size_t)h * nb + by[ty]) * nb + bx[tx]];
                    sc[ty * k + tx] = dot * scale + bias;
                }
            /* softmax */
            double m = sc[0];
            for (int t = 1; t < k * k; ++t)
                if (sc[t] > m) m = sc[t];
            double sum = 0.0;
            for (int t = 0; t < k * k; ++t) {
                sc[t] = exp(sc[t] - m);
                sum += sc[t];
            }
            /* weighted sum of values */
            double *o = out + base + ((size_t)i * W + j) * D;
            for (int c = 0; c < D; ++c) o[c] = 0.0;
            for (int ty = 0; ty < k; ++ty)
                for (int tx = 0; tx < k; ++tx) {
                    const double pw = sc[ty * k + tx] / sum;
                    const double *vv = v + base + ((size_t)ky[ty] * W + kx[tx]) * D;
                    for (int c = 0; c < D; ++c) o[c] += pw * vv[c];
                }
        }
    }
    free(ky); free(by); free(kx); free(bx); free(sc);
}

/* ---------------------------------------------------------------------------
 * Splitting the independent (b, head) slices over threads.
 * ------------------------------------------------------------------------- */
enum { OP_QK = 0, OP_SOFTMAX = 1, OP_AV = 2, OP_FORWARD = 3 };

typedef struct {
    int op;
    const oracle_shape *p;
    int bh_begin, bh_end;
    const double *q, *k, *v, *rpb, *attn_in;
    double *attn, *out;
} job;

static void *run_job(void *arg)
{
    job *jb = (job *)arg;
    for (int bh = jb->bh_begin; bh < jb->bh_end; ++bh) {
        switch (jb->op) {
        case OP_QK: qk_rpb_slice(jb->p, bh, jb->q, jb->k, jb->rpb, jb->attn); break;
        case OP_SOFTMAX: softmax_slice(jb->p, bh, jb->attn); break;
        case OP_AV: av_slice(jb->p, bh, jb->attn_in, jb->v, jb->out); break;
        default: forward_slice(jb->p, bh, jb->q, jb->k, jb->v, jb->rpb, jb->out); break;
        }
    }
    return NULL;
}

static int dispatch(job proto, int nthreads)
{
    const int nbh = proto.p->B * proto.p->heads;
    if (nbh == 0) return 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > nbh) nthreads = nbh;
    pthread_t *tid = malloc(sizeof(pthread_t) * nthreads);
    int *created = calloc(nthreads, sizeof(int));
    job *jobs = malloc(sizeof(job) * nthreads);
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = proto;
        jobs[t].bh_begin = (int)((long long)nbh * t / nthreads);
        jobs[t].bh_end = (int)((long long)nbh * (t + 1) / nthreads);
        if (t == nthreads - 1)
            run_job(&jobs[t]);   /* the calling thread takes the last share */
        else if (pthread_create(&tid[t], NULL, run_job, &jobs[t]) == 0)
            created[t] = 1;
        else
            run_job(&jobs[t]);   /* no thread available: run it here */
    }
    for (int t = 0; t < nthreads - 1; ++t)
        if (created[t]) pthread_join(tid[t], NULL);
    free(tid);
    free(created);
    free(jobs);
    return 0;
}

static oracle_shape make_shape(int B, int heads, int H, int W, int D, int k, int d)
{
    oracle_shape s = {B, heads, H, W, D, k, d};
    return s;
}

int oracle_na2d_qk_rpb(int B, int heads, int H, int W, int D, int k, int d,
                       const double *q, const double *kk, const double *rpb,
                       double *attn, int nthreads)
{
    oracle_shape p = make_shape(B, heads, H, W, D, k, d);
    if (!shape_ok(&p)) return -1;
    job jb;
    memset(&jb, 0, sizeof jb);
    jb.op = OP_QK; jb.p = &p; jb.q = q; jb.k = kk; jb.rpb = rpb; jb.attn = attn;
    return dispatch(jb, nthreads);
}

int oracle_na2d_softmax(int B, int heads, int H, int W, int D, int k, int d,
                        double *attn, int nthreads)
{
    oracle_shape p = make_shape(B, heads, H, W, D, k, d);
    if (!shape_ok(&p)) return -1;
    job jb;
    memset(&jb, 0, sizeof jb);
    jb.op = OP_SOFTMAX; jb.p = &p; jb.attn = attn;
    return dispatch(jb, nthreads);
}

int oracle_na2d_av(int B, int heads, int H, int W, int D, int k, int d,
                   const double *attn, const double *v, double *out, int nthreads)
{
    oracle_shape p = make_shape(B, heads, H, W, D, k, d);
    if (!shape_ok(&p)) return -1;
    job jb;
    memset(&jb, 0, sizeof jb);
    jb.op = OP_AV; jb.p = &p; jb.attn_in = attn; jb.v = v; jb.out = out;
    return dispatch(jb, nthreads);
}

int oracle_na2d_forward(int B, int heads, int H, int W, int D, int k, int d,
                        const double *q, const double *kk, const double *v,
                        const double *rpb, double *out, int nthreads)
{
    oracle_shape p = make_shape(B, heads, H, W, D, k, d);
    if (!shape_ok(&p)) return -1;
    job jb;
    memset(&jb, 0, sizeof jb);
    jb.op = OP_FORWARD; jb.p = &p; jb.q = q; jb.k = kk; jb.v = v; jb.rpb = rpb;
    jb.out = out;
    return dispatch(jb, nthreads);
}

/* ---------------------------------------------------------------------------
 * Backward of the fused definition.  The layer is trained end to end (gitcode
 * DiNAT article, section "微调示例：加载预训练权重继续训练", fine-tuning; the
 * HF tests it describes in "源码与测试导览" run forward and backward), so the
 * gradients of out with respect to q, k, v and rpb are part of the method.
 * They are the chain rule through the three stages, for one query with
 * scores s_n, weights p_n = softmax(s)_n and output o = sum_n p_n v_n, given
 * the output gradient g = dL/do:
 *     dL/dv_n    += p_n g                 (key n's value, from every query
 *                                          whose window holds key n)
 *     dL/dp_n     = g . v_n
 *     dL/ds_n     = p_n (dL/dp_n - sum_m p_m dL/dp_m)    (softmax Jacobian)
 *     dL/dq      += sum_n dL/ds_n k_n / sqrt(D)
 *     dL/dk_n    += dL/ds_n q / sqrt(D)
 *     dL/drpb[h, by_n, bx_n] += dL/ds_n
 * One query at a time, recomputing the forward's scores and softmax exactly
 * as forward_slice does.  dq, dk, dv of the slice are overwritten; the bias
 * gradient is added into drpb_acc ([heads, 2k-1, 2k-1]).
 * ------------------------------------------------------------------------- */
static void backward_slice(const oracle_shape *p, int bh, const double *q,
                           const double *kk, const double *v, const double *rpb,
                           const double *dout, double *dq, double *dk, double *dv,
                           double *drpb_acc)
{
    const int H = p->H, W = p->W, D = p->D, k = p->k, d = p->d;
    const int h = bh % p->heads;
    const int nb = 2 * k - 1;
    const double scale = 1.0 / sqrt((double)D);
    const size_t base = (size_t)bh * H * W * D;
    int *ky = malloc(sizeof(int) * k), *by = malloc(sizeof(int) * k);
    int *kx = malloc(sizeof(int) * k), *bx = malloc(sizeof(int) * k);
    double *sc = malloc(sizeof(double) * k * k);
    double *dp = malloc(sizeof(double) * k * k);
    for (size_t e = 0; e < (size_t)H * W * D; ++e) {
        dq[base + e] = 0.0;
        dk[base + e] = 0.0;
        dv[base + e] = 0.0;
    }
    for (int i = 0; i < H; ++i) {
        oracle_axis_neighbors(H, k, d, i, ky, by);
        for (int j = 0; j < W; ++j) {
            oracle_axis_neighbors(W, k, d, j, kx, bx);
            const double *qv = q + base + ((size_t)i * W + j) * D;
            const double *g = dout + base + ((size_t)i * W + j) * D;
            /* scores and softmax, as in the forward */
            for (int ty = 0; ty < k; ++ty)
                for (int tx = 0; tx < k; ++tx) {
                    const double *kv = kk + base + ((size_t)ky[ty] * W + kx[tx]) * D;
                    double dot = 0.0;
                    for (int c = 0; c < D; ++c) dot += qv[c] * kv[c];
                    double bias = 0.0;
                    if (rpb) bias = rpb[((size_t)h * nb + by[ty]) * nb + bx[tx]];
                    sc[ty * k + tx] = dot * scale + bias;
                }
            double m = sc[0];
            for (int t = 1; t < k * k; ++t)
                if (sc[t] > m) m = sc[t];
            double sum = 0.0;
            for (int t = 0; t < k * k; ++t) {
                sc[t] = exp(sc[t] - m);
                sum += sc[t];
            }
            for (int t = 0; t < k * k; ++t) sc[t] /= sum;       /* p_n */
            /* dL/dp_n = g . v_n, and the weighted mean sum_m p_m dL/dp_m */
            double pdp = 0.0;
            for (int ty = 0; ty < k; ++ty)
                for (int tx = 0; tx < k; ++tx) {
                    const double *vv = v + base + ((size_t)ky[ty] * W + kx[tx]) * D;
                    double dot = 0.0;
                    for (int c = 0; c < D; ++c) dot += g[c] * vv[c];
                    dp[ty * k + tx] = dot;
                    pdp += sc[ty * k + tx] * dot;
                }
            double *dqv = dq + base + ((size_t)i * W + j) * D;
            for (int ty = 0; ty < k; ++ty)
                for (int tx = 0; tx < k; ++tx) {
                    const int n = ty * k + tx;
                    const size_t key = base + ((size_t)ky[ty] * W + kx[tx]) * D;
                    const double ds = sc[n] * (dp[n] - pdp);        /* dL/ds_n */
                    for (int c = 0; c < D; ++c) {
                        dv[key + c] += sc[n] * g[c];
                        dqv[c] += ds * kk[key + c] * scale;
                        dk[key + c] += ds * qv[c] * scale;
                    }
                    drpb_acc[((size_t)h * nb + by[ty]) * nb + bx[tx]] += ds;
                }
        }
    }
    free(ky); free(by); free(kx); free(bx); free(sc); free(dp);
}

typedef struct {
    const oracle_shape *p;
    int bh_begin, bh_end;
    const double *q, *k, *v, *rpb, *dout;
    double *dq, *dk, *dv, *drpb_acc;
} bjob;

static void *run_bjob(void *arg)
{
    bjob *jb = (bjob *)arg;
    for (int bh = jb->bh_begin; bh < jb->bh_end; ++bh)
        backward_slice(jb->p, bh, jb->q, jb->k, jb->v, jb->rpb, jb->dout, jb->dq, jb->dk, jb->dv,
                       jb->drpb_acc);
    return NULL;
}

/* Gradients of the fused forward.  dq, dk, dv: [B, heads, H, W, D]; drpb:
 * [heads, 2k-1, 2k-1] or NULL (not wanted).  Threads split the (b, head)
 * slices; each thread sums its bias gradient privately and the sums are added
 * in thread order, so the result does not depend on timing. */
int oracle_na2d_backward(int B, int heads, int H, int W, int D, int k, int d,
                         const double *q, const double *kk, const double *v,
                         const double *rpb, const double *dout, double *dq,
                         double *dk, double *dv, double *drpb, int nthreads)
{
    oracle_shape p = make_shape(B, heads, H, W, D, k, d);
    if (!shape_ok(&p)) return -1;
    const int nb = 2 * k - 1;
    const size_t ntab = (size_t)heads * nb * nb;
    if (drpb)
        for (size_t e = 0; e < ntab; ++e) drpb[e] = 0.0;
    const int nbh = B * heads;
    if (nbh == 0) return 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > nbh) nthreads = nbh;
    pthread_t *tid = malloc(sizeof(pthread_t) * nthreads);
    int *created = calloc(nthreads, sizeof(int));
    bjob *jobs = malloc(sizeof(bjob) * nthreads);
    double *acc = calloc((size_t)nthreads * (ntab ? ntab : 1), sizeof(double));
    for (int t = 0; t < nthreads; ++t) {
        bjob jb = {&p, (int)((long long)nbh * t / nthreads), (int)((long long)nbh * (t + 1) / nthreads),
                   q, kk, v, rpb, dout, dq, dk, dv, acc + (size_t)t * ntab};
        jobs[t] = jb;
        if (t == nthreads - 1)
            run_bjob(&jobs[t]);
        else if (pthread_create(&tid[t], NULL, run_bjob, &jobs[t]) == 0)
            created[t] = 1;
        else
            run_bjob(&jobs[t]);
    }
    for (int t = 0; t < nthreads - 1; ++t)
        if (created[t]) pthread_join(tid[t], NULL);
    if (drpb)
        for (int t = 0; t < nthreads; ++t)
            for (size_t e = 0; e < ntab; ++e) drpb[e] += acc[(size_t)t * ntab + e];
    free(acc);
    free(tid);
    free(created);
    free(jobs);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Attention dropout and the returned attention weights.
 *
 * The layer applies dropout to the attention weights between the softmax and
 * natten2dav (gitcode DiNAT article, section "DiNAT 的核心思想"), and with
 * output_attentions returns those weights ("Dilated Neighborhood Attention
 * Transformer", HF docs, DinatModel outputs, `attentions`).  Dropout keeps a
 * weight with probability 1 - p and scales kept weights by 1 / (1 - p).
 *
 * The random draw is a counter-based generator so that the GPU and this
 * oracle draw the same mask: Philox4x32-10 from its publication (Salmon,
 * Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011):
 * ten rounds; a round multiplies counter words 0 and 2 by 0xD2511F53 and
 * 0xCD9E8D57 into 64-bit products and forms (hi(c2*M1) ^ c1 ^ k0, lo(c2*M1),
 * hi(c0*M0) ^ c3 ^ k1, lo(c0*M0)); the key is bumped by (0x9E3779B9,
 * 0xBB67AE85) before every round but the first.
 * Weight e (its linear index in [B, heads, H, W, k*k]) is kept when word
 * e mod 4 of Philox(counter = (e/4 low 32 bits, e/4 high 32, offset low,
 * offset high), key = (seed low, seed high)) is >= round(p * 2^32).
 * ------------------------------------------------------------------------- */
void oracle_philox4x32_10(const unsigned int ctr[4], const unsigned int key[2], unsigned int out[4])
{
    unsigned int c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    unsigned int k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        unsigned long long prod0 = (unsigned long long)0xD2511F53u * c0;
        unsigned long long prod1 = (unsigned long long)0xCD9E8D57u * c2;
        unsigned int n0 = (unsigned int)(prod1 >> 32) ^ c1 ^ k0;
        unsigned int n1 = (unsigned int)prod1;
        unsigned int n2 = (unsigned int)(prod0 >> 32) ^ c3 ^ k1;
        unsigned int n3 = (unsigned int)prod0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

static unsigned int drop_threshold(double p)
{
    double t = p * 4294967296.0;
    if (t >= 4294967295.0) return 0xFFFFFFFFu;
    return (unsigned int)(t + 0.5);
}

/* dropout factor of weight e: 0 (dropped) or 1 / (1 - p) (kept) */
static double drop_factor(unsigned long long e, double p, unsigned long long seed, unsigned long long offset)
{
    if (p <= 0.0) return 1.0;
    unsigned long long blk = e >> 2;
    unsigned int ctr[4] = {(unsigned int)blk, (unsigned int)(blk >> 32), (unsigned int)offset,
                           (unsigned int)(offset >> 32)};
    unsigned int key[2] = {(unsigned int)seed, (unsigned int)(seed >> 32)};
    unsigned int w[4];
    oracle_philox4x32_10(ctr, key, w);
    return w[e & 3] >= drop_threshold(p) ? 1.0 / (1.0 - p) : 0.0;
}

/* Fused definition with dropout and the weights written out: as
 * forward_slice, then p_n <- factor_n p_n, attn[.., n] = p_n (if attn), and
 * out = sum_n p_n v_n. */
static void forward_ex_slice(const oracle_shape *p, int bh, const double *q, const double *kk, const double *v,
                             const double *rpb, double *out, double *attn, double dp, unsigned long long seed,
                             unsigned long long offset, int Hr, int Wr)
{
    const int H = p->H, W = p->W, D = p->D, k = p->k, d = p->d;
    const int h = bh % p->heads;
    const int nb = 2 * k - 1;
    const double scale = 1.0 / sqrt((double)D);
    const size_t base = (size_t)bh * H * W * D;
    int *ky = malloc(sizeof(int) * k), *by = malloc(sizeof(int) * k);
    int *kx = malloc(sizeof(int) * k), *bx = malloc(sizeof(int) * k);
    double *sc = malloc(sizeof(double) * k * k);
    for (int i = 0; i < H; ++i) {
        oracle_axis_neighbors(H, k, d, i, ky, by);
        for (int j = 0; j < W; ++j) {
            oracle_axis_neighbors(W, k, d, j, kx, bx);
            const double *qv = q + base + ((size_t)i * W + j) * D;
            for (int ty = 0; ty < k; ++ty)
                for (int tx = 0; tx < k; ++tx) {
                    const double *kv = kk + base + ((size_t)ky[ty] * W + kx[tx]) * D;
                    double dot = 0.0;
                    for (int c = 0; c < D; ++c) dot += qv[c] * kv[c];
                    double bias = 0.0;
                    if (rpb) bias = rpb[((size_t)h * nb + by[ty]) * nb + bx[tx]];
                    sc[ty * k + tx] = dot * scale + bias;
                }
            double m = sc[0];
            for (int t = 1; t < k * k; ++t)
                if (sc[t] > m) m = sc[t];
            double sum = 0.0;
            for (int t = 0; t < k * k; ++t) {
                sc[t] = exp(sc[t] - m);
                sum += sc[t];
            }
            /* weights are numbered over the real Hr x Wr map (padded queries
             * are cropped and draw nothing) */
            const int real = i < Hr && j < Wr;
            const unsigned long long row = ((unsigned long long)bh * Hr + i) * Wr + j;
            for (int t = 0; t < k * k; ++t) {
                sc[t] = sc[t] / sum * (real ? drop_factor(row * (unsigned long long)(k * k) + t, dp, seed, offset) : 1.0);
                if (attn && real) attn[row * (size_t)(k * k) + t] = sc[t];
            }
            double *o = out + base + ((size_t)i * W + j) * D;
            for (int c = 0; c < D; ++c) o[c] = 0.0;
            for (int ty = 0; ty < k; ++ty)
                for (int tx = 0; tx < k; ++tx) {
                    const double *vv = v + base + ((size_t)ky[ty] * W + kx[tx]) * D;
                    for (int c = 0; c < D; ++c) o[c] += sc[ty * k + tx] * vv[c];
                }
        }
    }
    free(ky); free(by); free(kx); free(bx); free(sc);
}

/* Backward with dropout: out = sum_n f_n p_n v_n with dropout factors f_n.
 *     dL/dv_n += f_n p_n g,   dL/dp_n = f_n (g . v_n),
 *     dL/ds_n = p_n (dL/dp_n - sum_m p_m dL/dp_m), then as backward_slice. */
static void backward_ex_slice(const oracle_shape *p, int bh, const double *q, const double *kk, const double *v,
                              const double *rpb, const double *dout, double *dq, double *dk, double *dv,
                              double *drpb_acc, double dp_, unsigned long long seed, unsigned long long offset,
                              int Hr, int Wr)
{
    const int H = p->H, W = p->W, D = p->D, k = p->k, d = p->d;
    const int h = bh % p->heads;
    const int nb = 2 * k - 1;
    const double scale = 1.0 / sqrt((double)D);
    const size_t base = (size_t)bh * H * W * D;
    int *ky = malloc(sizeof(int) * k), *by = malloc(sizeof(int) * k);
    int *kx = malloc(sizeof(int) * k), *bx = malloc(sizeof(int) * k);
    double *sc = malloc(sizeof(double) * k * k), *dp = malloc(sizeof(double) * k * k);
    double *f = malloc(sizeof(double) * k * k);
    for (size_t e = 0; e < (size_t)H * W * D; ++e) {
        dq[base + e] = 0.0;
        dk[base + e] = 0.0;
        dv[base + e] = 0.0;
    }
    for (int i = 0; i < H; ++i) {
        oracle_axis_neighbors(H, k, d, i, ky, by);
        for (int j = 0; j < W; ++j) {
            oracle_axis_neighbors(W, k, d, j, kx, bx);
            const double *qv = q + base + ((size_t)i * W + j) * D;
            const double *g = dout + base + ((size_t)i * W + j) * D;
            for (int ty = 0; ty < k; ++ty)
                for (int tx = 0; tx < k; ++tx) {
                    const double *kv = kk + base + ((size_t)ky[ty] * W + kx[tx]) * D;
                    double dot = 0.0;
                    for (int c = 0; c < D; ++c) dot += qv[c] * kv[c];
                    double bias = 0.0;
                    if (rpb) bias = rpb[((size_t)h * nb + by[ty]) * nb + bx[tx]];
                    sc[ty * k + tx] = dot * scale + bias;
                }
            double m = sc[0];
            for (int t = 1; t < k * k; ++t)
                if (sc[t] > m) m = sc[t];
            double sum = 0.0;
            for (int t = 0; t < k * k; ++t) {
                sc[t] = exp(sc[t] - m);
                sum += sc[t];
            }
            const int real = i < Hr && j < Wr;
            const unsigned long long row = ((unsigned long long)bh * Hr + i) * Wr + j;
            for (int t = 0; t < k * k; ++t) {
                sc[t] /= sum;
                f[t] = real ? drop_factor(row * (unsigned long long)(k * k) + t, dp_, seed, offset) : 1.0;
            }
            double pdp = 0.0;
            for (int ty = 0; ty < k; ++ty)
                for (int tx = 0; tx < k; ++tx) {
                    const double *vv = v + base + ((size_t)ky[ty] * W + kx[tx]) * D;
                    double dot = 0.0;
                    for (int c = 0; c < D; ++c) dot += g[c] * vv[c];
                    dp[ty * k + tx] = f[ty * k + tx] * dot;
                    pdp += sc[ty * k + tx] * dp[ty * k + tx];
                }
            double *dqv = dq + base + ((size_t)i * W + j) * D;
            for (int ty = 0; ty < k; ++ty)
                for (int tx = 0; tx < k; ++tx) {
                    const int n = ty * k + tx;
                    const size_t key = base + ((size_t)ky[ty] * W + kx[tx]) * D;
                    const double ds = sc[n] * (dp[n] - pdp);
                    for (int c = 0; c < D; ++c) {
                        dv[key + c] += f[n] * sc[n] * g[c];
                        dqv[c] += ds * kk[key + c] * scale;
                        dk[key + c] += ds * qv[c] * scale;
                    }
                    drpb_acc[((size_t)h * nb + by[ty]) * nb + bx[tx]] += ds;
                }
        }
    }
    free(ky); free(by); free(kx); free(bx); free(sc); free(dp); free(f);
}

/* Forward with optional weights output (attn, may be NULL) and dropout
 * probability dp (0: none); single-threaded per call, slices in order.  The
 * arrays may be a zero-padded map whose real part is the top-left Hr x Wr
 * (Hr = H, Wr = W without padding): weights are numbered over the real map,
 * and attn holds [B, heads, Hr, Wr, k*k]. */
int oracle_na2d_forward_ex(int B, int heads, int H, int W, int D, int k, int d, const double *q,
                           const double *kk, const double *v, const double *rpb, double *out, double *attn,
                           double dp, unsigned long long seed, unsigned long long offset, int Hr, int Wr)
{
    oracle_shape p = make_shape(B, heads, H, W, D, k, d);
    if (!shape_ok(&p) || Hr < 1 || Hr > H || Wr < 1 || Wr > W) return -1;
    for (int bh = 0; bh < B * heads; ++bh)
        forward_ex_slice(&p, bh, q, kk, v, rpb, out, attn, dp, seed, offset, Hr, Wr);
    return 0;
}

int oracle_na2d_backward_ex(int B, int heads, int H, int W, int D, int k, int d, const double *q,
                            const double *kk, const double *v, const double *rpb, const double *dout, double *dq,
                            double *dk, double *dv, double *drpb, double dp, unsigned long long seed,
                            unsigned long long offset, int Hr, int Wr)
{
    oracle_shape p = make_shape(B, heads, H, W, D, k, d);
    if (!shape_ok(&p) || Hr < 1 || Hr > H || Wr < 1 || Wr > W) return -1;
    const size_t ntab = (size_t)heads * (2 * k - 1) * (2 * k - 1);
    double *acc = calloc(ntab ? ntab : 1, sizeof(double));
    for (int bh = 0; bh < B * heads; ++bh)
        backward_ex_slice(&p, bh, q, kk, v, rpb, dout, dq, dk, dv, acc, dp, seed, offset, Hr, Wr);
    if (drpb)
        for (size_t e = 0; e < ntab; ++e) drpb[e] = acc[e];
    free(acc);
    return 0;
}
