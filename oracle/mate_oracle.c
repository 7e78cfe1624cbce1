/*
 * MATE token-mix oracle: a plain, sequential, fp64 CPU statement of what the
 * token-mixing core of LinGen's MATE block computes.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
 * load this file: only the tests, the smoke check and the bench's CPU
 * baseline do. It shares no code, header, table or helper with the CUDA
 * library; it is written straight from the pages' description.
 *
 * Sources (cited by page title and section):
 *   [QbitAI]  "LinGen ... 视频生成 ..." news article (QbitAI), section
 *             "方法：线性复杂度的MATE模块" (method: the MATE module).
 *   [Review]  "LinGen: Towards High-Resolution Minute-Length Text-to-Video
 *             Generation with Linear Computational Complexity", xllm-io paper
 *             review, section 三 "技术架构" (architecture): "MA-Branch" items
 *             1-3 and "TE-Branch".
 *
 * Every floating-point step runs in double precision, in the order the
 * method states it. OpenMP only splits independent (batch, head, direction)
 * or (batch, window, head) work items; it never reorders a sum.
 *
 * Readings of points the pages leave open (each also listed in the design
 * notes of the repository):
 *   R1 scan priorities: SR = (W, H, T), SC = (H, W, T), TR = (T, W, H),
 *      TC = (T, H, W), first entry = first priority = fastest-varying axis.
 *   R2 the flip is n -> N-1-n for 0-indexed n (the review prints the
 *      1-indexed form T*H*W - n).
 *   R3 review tokens: non-overlapping average pooling, stride = kernel, of
 *      the scan inputs x, dt, B, C; the pooled grid is unrolled in the same
 *      scan order; the prefix is [R, flip(R)]; the same prefix precedes the
 *      forward and the flipped sequence; outputs at prefix positions are
 *      dropped.
 *   R4 bidirectional: the same A, D, dt, B, C serve both directions; the
 *      flipped sequence's outputs are flipped back and summed with the
 *      forward outputs (so D*x appears twice).
 *   R5 TESA windows: per axis, window boundaries sit at coordinates that are
 *      congruent to the shift modulo the window size; the windows at the two
 *      ends are partial. Plain softmax(q k^T / sqrt(d)) v per head inside each
 *      window, no mask inside a window, no position bias.
 *   R6 Zigzag scan (named, not defined, by the pages): the 3D boustrophedon
 *      of oracle_zigzag, used only as the comparison order.
 *   R7 MATE composition: the two branch outputs (different widths) are each
 *      projected to the model width and added; no gate, no bias.
 *   R8 MA-branch front-end (oracle/__init__.py, Oracle.frontend): the standard
 *      Mamba2 input side, in_proj to [z | x B C | dt], a causal depthwise
 *      conv of width 4 with bias along the forward scan order, SiLU, and
 *      softplus(dt + bias); one result feeds both scan directions.
 *   R9 MA-branch output side (oracle_gate_norm): the standard Mamba2 gated RMS
 *      norm, gate first: v = y * SiLU(z), then each group of `group`
 *      consecutive channels is divided by the root of its mean square plus eps
 *      and scaled by the per-channel weight. The pages name the block only.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL -1
#define ORACLE_ENOMEM -2

enum { AXIS_T = 0, AXIS_H = 1, AXIS_W = 2 };

/* Rotary Major Scan orders ([Review] MA-Branch item 2; [QbitAI]: "W, H and T
 * have the first, second and third priority when unrolled in the example;
 * swapping the priorities gives the other scans"). Row = W before H,
 * column = H before W; spatial = T last, temporal = T first (reading R1). */
static const int kScanPriority[4][3] = {
    {AXIS_W, AXIS_H, AXIS_T}, /* 0: spatial-row major    */
    {AXIS_H, AXIS_W, AXIS_T}, /* 1: spatial-column major */
    {AXIS_T, AXIS_W, AXIS_H}, /* 2: temporal-row major   */
    {AXIS_T, AXIS_H, AXIS_W}, /* 3: temporal-column major */
};

/* Unroll a T x H x W grid into a 1D sequence with the given axis priorities
 * (priority[0] varies fastest). seq[n] = grid offset (t*H + h)*W + w of the
 * n-th token of the sequence. */
int oracle_unroll(int T, int H, int W, const int priority[3], int32_t *seq)
{
    if (T <= 0 || H <= 0 || W <= 0 || !priority || !seq) return ORACLE_EINVAL;
    int extent[3] = {T, H, W};
    int seen[3] = {0, 0, 0};
    for (int i = 0; i < 3; ++i) {
        if (priority[i] < 0 || priority[i] > 2 || seen[priority[i]]) return ORACLE_EINVAL;
        seen[priority[i]] = 1;
    }
    const int a0 = priority[0], a1 = priority[1], a2 = priority[2];
    int c[3];
    int64_t n = 0;
    for (c[a2] = 0; c[a2] < extent[a2]; ++c[a2])
        for (c[a1] = 0; c[a1] < extent[a1]; ++c[a1])
            for (c[a0] = 0; c[a0] < extent[a0]; ++c[a0])
                seq[n++] = (int32_t)(((int64_t)c[AXIS_T] * H + c[AXIS_H]) * W + c[AXIS_W]);
    return ORACLE_OK;
}

/* The Zigzag scan the pages set against RMS ([QbitAI] method section: Zigzag
 * and Hilbert scans keep neighbours together but need costly reorderings;
 * [Review] 5.5 Table 2, "Zigzag"). The pages do not define it; reading R6:
 * a 3D boustrophedon whose every step moves to a neighbouring token. Frames
 * are visited in time order; even frames take their rows top to bottom, odd
 * frames bottom to top; the k-th row visited overall (k from 0) is walked
 * along W left to right when k is even and right to left when k is odd. */
int oracle_zigzag(int T, int H, int W, int32_t *seq)
{
    if (T <= 0 || H <= 0 || W <= 0 || !seq) return ORACLE_EINVAL;
    int64_t n = 0, row = 0;
    for (int t = 0; t < T; ++t) {
        for (int i = 0; i < H; ++i, ++row) {
            const int h = (t % 2 == 0) ? i : H - 1 - i;
            for (int j = 0; j < W; ++j) {
                const int w = (row % 2 == 0) ? j : W - 1 - j;
                seq[n++] = (int32_t)(((int64_t)t * H + h) * W + w);
            }
        }
    }
    return ORACLE_OK;
}

/* The scan sequence of a mode (0-3: the RMS orders, 4: Zigzag), optionally
 * flipped ([Review] MA-Branch item 2: every layer scans the sequence and its
 * flip; reading R2). */
int oracle_rms_sequence(int T, int H, int W, int mode, int flip, int32_t *seq)
{
    if (mode < 0 || mode > 4) return ORACLE_EINVAL;
    int rc = mode == 4 ? oracle_zigzag(T, H, W, seq) : oracle_unroll(T, H, W, kScanPriority[mode], seq);
    if (rc != ORACLE_OK || !flip) return rc;
    int64_t N = (int64_t)T * H * W;
    for (int64_t i = 0, j = N - 1; i < j; ++i, --j) {
        int32_t tmp = seq[i];
        seq[i] = seq[j];
        seq[j] = tmp;
    }
    return ORACLE_OK;
}

/* Non-overlapping average pooling of a grid tensor with `ch` channels per
 * token over pt x ph x pw boxes (reading R3). grid: (T, H, W, ch);
 * pooled: (T/pt, H/ph, W/pw, ch). */
int oracle_avg_pool(const double *grid, int T, int H, int W, int ch,
                    int pt, int ph, int pw, double *pooled)
{
    if (pt <= 0 || ph <= 0 || pw <= 0 || T % pt || H % ph || W % pw) return ORACLE_EINVAL;
    const int Tp = T / pt, Hp = H / ph, Wp = W / pw;
    const double inv = 1.0 / ((double)pt * ph * pw);
    for (int tp = 0; tp < Tp; ++tp)
        for (int hp = 0; hp < Hp; ++hp)
            for (int wp = 0; wp < Wp; ++wp) {
                double *dst = pooled + (((int64_t)tp * Hp + hp) * Wp + wp) * ch;
                for (int k = 0; k < ch; ++k) dst[k] = 0.0;
                for (int t = tp * pt; t < (tp + 1) * pt; ++t)
                    for (int h = hp * ph; h < (hp + 1) * ph; ++h)
                        for (int w = wp * pw; w < (wp + 1) * pw; ++w) {
                            const double *src = grid + (((int64_t)t * H + h) * W + w) * ch;
                            for (int k = 0; k < ch; ++k) dst[k] += src[k];
                        }
                for (int k = 0; k < ch; ++k) dst[k] *= inv;
            }
    return ORACLE_OK;
}

/* Mamba2 selective state-space scan, one head, one direction, over an
 * explicit token sequence of length L ([Review] MA-Branch item 1: Mamba2 /
 * SSD). With state h (P x Ns, zero at the start):
 *     h_t = exp(dt_t * A) * h_{t-1} + dt_t * x_t B_t^T
 *     y_t = h_t C_t + D * x_t
 * x: L rows of stride xs (P used), dt: L values of stride ds, B and C: L rows
 * of stride bs (Ns used), y: L rows of stride ys. */
static void scan_one_head(int64_t L, int P, int Ns,
                          const double *x, int64_t xs, const double *dt, int64_t ds,
                          const double *B, const double *C, int64_t bs,
                          double A, double D, double *y, int64_t ys, double *h)
{
    memset(h, 0, sizeof(double) * (size_t)P * Ns);
    for (int64_t t = 0; t < L; ++t) {
        const double *xt = x + t * xs, *Bt = B + t * bs, *Ct = C + t * bs;
        const double dtt = dt[t * ds];
        const double decay = exp(dtt * A);
        double *yt = y + t * ys;
        for (int p = 0; p < P; ++p) {
            double acc = 0.0;
            for (int n = 0; n < Ns; ++n) {
                double *hpn = h + (size_t)p * Ns + n;
                *hpn = decay * (*hpn) + dtt * xt[p] * Bt[n];
                acc += (*hpn) * Ct[n];
            }
            yt[p] = acc + D * xt[p];
        }
    }
}

/* One-direction scan of a whole multi-head sequence. xs: (L, nh, P);
 * dts: (L, nh); Bs, Cs: (L, G, Ns); ys: (L, nh, P). Head h reads group
 * h / (nh / G). Exposed so that tests can pin the recurrence alone. */
int oracle_ssd_scan(int64_t L, int nh, int P, int Ns, int G,
                    const double *xs, const double *dts, const double *A,
                    const double *Bs, const double *Cs, const double *D, double *ys)
{
    if (L < 0 || nh <= 0 || P <= 0 || Ns <= 0 || G <= 0 || nh % G) return ORACLE_EINVAL;
    const int heads_per_group = nh / G;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int hd = 0; hd < nh; ++hd) {
        double *h = (double *)malloc(sizeof(double) * (size_t)P * Ns);
        if (!h) {
#pragma omp atomic write
            err = 1;
            continue;
        }
        const int g = hd / heads_per_group;
        scan_one_head(L, P, Ns, xs + (size_t)hd * P, (int64_t)nh * P, dts + hd, nh,
                      Bs + (size_t)g * Ns, Cs + (size_t)g * Ns, (int64_t)G * Ns,
                      A[hd], D[hd], ys + (size_t)hd * P, (int64_t)nh * P, h);
        free(h);
    }
    return err ? ORACLE_ENOMEM : ORACLE_OK;
}

/* Gather rows of a (rows, width) table into a sequence: dst[i] = src[idx[i]]. */
static void gather_rows(const double *src, int64_t width, const int32_t *idx, int64_t n, double *dst)
{
    for (int64_t i = 0; i < n; ++i)
        memcpy(dst + i * width, src + (int64_t)idx[i] * width, sizeof(double) * (size_t)width);
}

/* The MA-branch token mix: bidirectional Mamba2 scan in Rotary Major Scan
 * order with optional review tokens ([Review] MA-Branch items 1-3, [QbitAI]
 * method section; readings R1-R4).
 *   x: (batch, T, H, W, nh, P)   dt: (batch, T, H, W, nh)   A, D: (nh)
 *   B, C: (batch, T, H, W, G, Ns)   out: (batch, T, H, W, nh, P)
 *   pool: {pt, ph, pw}; NULL or {0, 0, 0} = no review tokens.
 * For each batch element:
 *   1. unroll the grid into the scan sequence X of the mode;
 *   2. with review tokens, pool x, dt, B, C, unroll the pooled grid in the
 *      same mode into R and form the prefix [R, flip(R)];
 *   3. scan [prefix, X] and [prefix, flip(X)] from a zero state;
 *   4. drop the prefix outputs, flip the second result back, add the two and
 *      write each sum to the grid position of its token. */
int oracle_bissd(int batch, int T, int H, int W, int nh, int P, int Ns, int G,
                 const double *x, const double *dt, const double *A,
                 const double *B, const double *C, const double *D,
                 int mode, const int *pool, double *out)
{
    if (batch <= 0 || T <= 0 || H <= 0 || W <= 0 || nh <= 0 || P <= 0 || Ns <= 0 || G <= 0 ||
        nh % G || mode < 0 || mode > 4)
        return ORACLE_EINVAL;
    const int review = pool && (pool[0] || pool[1] || pool[2]);
    if (review && (pool[0] <= 0 || pool[1] <= 0 || pool[2] <= 0 ||
                   T % pool[0] || H % pool[1] || W % pool[2]))
        return ORACLE_EINVAL;

    const int64_t N = (int64_t)T * H * W;
    const int Tp = review ? T / pool[0] : 0, Hp = review ? H / pool[1] : 0, Wp = review ? W / pool[2] : 0;
    const int64_t Np = (int64_t)Tp * Hp * Wp;
    const int64_t Lp = 2 * Np;           /* prefix length */
    const int64_t L = Lp + N;            /* scanned sequence length */
    const int64_t wx = (int64_t)nh * P, wd = nh, wb = (int64_t)G * Ns;

    int32_t *order = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    int32_t *porder = review ? (int32_t *)malloc(sizeof(int32_t) * (size_t)Np) : NULL;
    double *sx = (double *)malloc(sizeof(double) * (size_t)(L * wx));
    double *sd = (double *)malloc(sizeof(double) * (size_t)(L * wd));
    double *sb = (double *)malloc(sizeof(double) * (size_t)(L * wb));
    double *sc = (double *)malloc(sizeof(double) * (size_t)(L * wb));
    double *yf = (double *)malloc(sizeof(double) * (size_t)(L * wx));
    double *yb = (double *)malloc(sizeof(double) * (size_t)(L * wx));
    double *px = review ? (double *)malloc(sizeof(double) * (size_t)(Np * wx)) : NULL;
    double *pd = review ? (double *)malloc(sizeof(double) * (size_t)(Np * wd)) : NULL;
    double *pb = review ? (double *)malloc(sizeof(double) * (size_t)(Np * wb)) : NULL;
    double *pc = review ? (double *)malloc(sizeof(double) * (size_t)(Np * wb)) : NULL;
    int rc = ORACLE_OK;
    if (!order || !sx || !sd || !sb || !sc || !yf || !yb ||
        (review && (!porder || !px || !pd || !pb || !pc))) {
        rc = ORACLE_ENOMEM;
        goto done;
    }
    oracle_rms_sequence(T, H, W, mode, 0, order);
    if (review) oracle_rms_sequence(Tp, Hp, Wp, mode, 0, porder);

    for (int b = 0; b < batch; ++b) {
        const double *xb = x + (size_t)b * N * wx, *db = dt + (size_t)b * N * wd;
        const double *Bb = B + (size_t)b * N * wb, *Cb = C + (size_t)b * N * wb;
        double *ob = out + (size_t)b * N * wx;

        /* step 2: the review prefix [R, flip(R)] */
        if (review) {
            oracle_avg_pool(xb, T, H, W, (int)wx, pool[0], pool[1], pool[2], px);
            oracle_avg_pool(db, T, H, W, (int)wd, pool[0], pool[1], pool[2], pd);
            oracle_avg_pool(Bb, T, H, W, (int)wb, pool[0], pool[1], pool[2], pb);
            oracle_avg_pool(Cb, T, H, W, (int)wb, pool[0], pool[1], pool[2], pc);
            for (int64_t i = 0; i < Np; ++i) {
                const int64_t lo = i, hi = Lp - 1 - i; /* R[i] sits at i and at its mirror */
                memcpy(sx + lo * wx, px + (int64_t)porder[i] * wx, sizeof(double) * (size_t)wx);
                memcpy(sx + hi * wx, px + (int64_t)porder[i] * wx, sizeof(double) * (size_t)wx);
                memcpy(sd + lo * wd, pd + (int64_t)porder[i] * wd, sizeof(double) * (size_t)wd);
                memcpy(sd + hi * wd, pd + (int64_t)porder[i] * wd, sizeof(double) * (size_t)wd);
                memcpy(sb + lo * wb, pb + (int64_t)porder[i] * wb, sizeof(double) * (size_t)wb);
                memcpy(sb + hi * wb, pb + (int64_t)porder[i] * wb, sizeof(double) * (size_t)wb);
                memcpy(sc + lo * wb, pc + (int64_t)porder[i] * wb, sizeof(double) * (size_t)wb);
                memcpy(sc + hi * wb, pc + (int64_t)porder[i] * wb, sizeof(double) * (size_t)wb);
            }
        }

        /* steps 1 and 3, forward: [prefix, X] */
        gather_rows(xb, wx, order, N, sx + Lp * wx);
        gather_rows(db, wd, order, N, sd + Lp * wd);
        gather_rows(Bb, wb, order, N, sb + Lp * wb);
        gather_rows(Cb, wb, order, N, sc + Lp * wb);
        rc = oracle_ssd_scan(L, nh, P, Ns, G, sx, sd, A, sb, sc, D, yf);
        if (rc) goto done;

        /* steps 1 and 3, flipped: [prefix, flip(X)] */
        for (int64_t i = 0; i < N; ++i) {
            const int64_t g = order[N - 1 - i];
            memcpy(sx + (Lp + i) * wx, xb + g * wx, sizeof(double) * (size_t)wx);
            memcpy(sd + (Lp + i) * wd, db + g * wd, sizeof(double) * (size_t)wd);
            memcpy(sb + (Lp + i) * wb, Bb + g * wb, sizeof(double) * (size_t)wb);
            memcpy(sc + (Lp + i) * wb, Cb + g * wb, sizeof(double) * (size_t)wb);
        }
        rc = oracle_ssd_scan(L, nh, P, Ns, G, sx, sd, A, sb, sc, D, yb);
        if (rc) goto done;

        /* step 4: drop the prefix, flip back, sum, scatter to grid order */
        for (int64_t n = 0; n < N; ++n) {
            const double *f = yf + (Lp + n) * wx;
            const double *r = yb + (Lp + (N - 1 - n)) * wx;
            double *o = ob + (int64_t)order[n] * wx;
            for (int64_t k = 0; k < wx; ++k) o[k] = f[k] + r[k];
        }
    }
done:
    free(order); free(porder); free(sx); free(sd); free(sb); free(sc); free(yf); free(yb);
    free(px); free(pd); free(pb); free(pc);
    return rc;
}

/* Window starts along one axis of length Lx for window size S and shift s
 * (reading R5). Returns the number of windows; starts[count] = Lx. */
static int axis_windows(int Lx, int S, int s, int *starts)
{
    int n = 0;
    if (s > 0) starts[n++] = 0; /* the partial window in front of the first boundary */
    for (int b = s; b < Lx; b += S) starts[n++] = b;
    starts[n] = Lx;
    return n;
}

static int valid_window_args(int T, int H, int W, int Tw, int Sw, const int *shift)
{
    if (T <= 0 || H <= 0 || W <= 0 || Tw <= 0 || Sw <= 0 || !shift) return 0;
    if (shift[0] < 0 || shift[0] >= Tw || shift[1] < 0 || shift[1] >= Sw || shift[2] < 0 || shift[2] >= Sw)
        return 0;
    return 1;
}

/* Window id of every grid token (grid order), windows numbered in
 * lexicographic (t, h, w) order of their first token. Returns the window
 * count, or a negative error. */
int oracle_tesa_window_ids(int T, int H, int W, int Tw, int Sw, const int *shift, int32_t *win)
{
    if (!valid_window_args(T, H, W, Tw, Sw, shift) || !win) return ORACLE_EINVAL;
    int *st = (int *)malloc(sizeof(int) * (size_t)(T + 2));
    int *sh = (int *)malloc(sizeof(int) * (size_t)(H + 2));
    int *sw = (int *)malloc(sizeof(int) * (size_t)(W + 2));
    if (!st || !sh || !sw) { free(st); free(sh); free(sw); return ORACLE_ENOMEM; }
    const int nt = axis_windows(T, Tw, shift[0], st);
    const int nhw = axis_windows(H, Sw, shift[1], sh);
    const int nww = axis_windows(W, Sw, shift[2], sw);
    int id = 0;
    for (int a = 0; a < nt; ++a)
        for (int bb = 0; bb < nhw; ++bb)
            for (int c = 0; c < nww; ++c, ++id)
                for (int t = st[a]; t < st[a + 1]; ++t)
                    for (int h = sh[bb]; h < sh[bb + 1]; ++h)
                        for (int w = sw[c]; w < sw[c + 1]; ++w)
                            win[((int64_t)t * H + h) * W + w] = id;
    free(st); free(sh); free(sw);
    return id;
}

/* TEmporal Swin Attention ([Review] TE-Branch; [QbitAI] method section:
 * attention only among tokens of the same T_w x S_w x S_w window, windows
 * shifting between layers; reading R5).
 *   q, k, v, out: (batch, T, H, W, nh, d). For every window and head:
 *   out_i = sum_j softmax_j(q_i . k_j / sqrt(d)) v_j over the window's tokens. */
int oracle_tesa(int batch, int T, int H, int W, int nh, int d,
                const double *q, const double *k, const double *v,
                int Tw, int Sw, const int *shift, double *out)
{
    if (batch <= 0 || nh <= 0 || d <= 0 || !valid_window_args(T, H, W, Tw, Sw, shift)) return ORACLE_EINVAL;
    const int64_t N = (int64_t)T * H * W;
    int32_t *win = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    if (!win) return ORACLE_ENOMEM;
    const int nwin = oracle_tesa_window_ids(T, H, W, Tw, Sw, shift, win);
    /* member lists: tokens of each window in grid order */
    int64_t *count = (int64_t *)calloc((size_t)nwin + 1, sizeof(int64_t));
    int32_t *members = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    int64_t *fill = (int64_t *)calloc((size_t)nwin + 1, sizeof(int64_t));
    if (!count || !members || !fill) { free(win); free(count); free(members); free(fill); return ORACLE_ENOMEM; }
    for (int64_t g = 0; g < N; ++g) count[win[g] + 1]++;
    for (int w = 0; w < nwin; ++w) count[w + 1] += count[w];
    for (int64_t g = 0; g < N; ++g) members[count[win[g]] + fill[win[g]]++] = (int32_t)g;

    const double scale = 1.0 / sqrt((double)d);
    const int64_t row = (int64_t)nh * d;
    int err = 0;
#pragma omp parallel for collapse(3) schedule(dynamic, 4)
    for (int b = 0; b < batch; ++b)
        for (int w = 0; w < nwin; ++w)
            for (int hd = 0; hd < nh; ++hd) {
                const int64_t m = count[w + 1] - count[w];
                const int32_t *tok = members + count[w];
                double *p = (double *)malloc(sizeof(double) * (size_t)m);
                if (!p) {
#pragma omp atomic write
                    err = 1;
                    continue;
                }
                const double *qb = q + (size_t)b * N * row, *kb = k + (size_t)b * N * row, *vb = v + (size_t)b * N * row;
                double *ob = out + (size_t)b * N * row;
                for (int64_t i = 0; i < m; ++i) {
                    const double *qi = qb + (int64_t)tok[i] * row + (int64_t)hd * d;
                    double mx = -INFINITY;
                    for (int64_t j = 0; j < m; ++j) {
                        const double *kj = kb + (int64_t)tok[j] * row + (int64_t)hd * d;
                        double s = 0.0;
                        for (int e = 0; e < d; ++e) s += qi[e] * kj[e];
                        p[j] = s * scale;
                        if (p[j] > mx) mx = p[j];
                    }
                    double den = 0.0;
                    for (int64_t j = 0; j < m; ++j) { p[j] = exp(p[j] - mx); den += p[j]; }
                    double *oi = ob + (int64_t)tok[i] * row + (int64_t)hd * d;
                    for (int e = 0; e < d; ++e) oi[e] = 0.0;
                    for (int64_t j = 0; j < m; ++j) {
                        const double *vj = vb + (int64_t)tok[j] * row + (int64_t)hd * d;
                        const double wgt = p[j] / den;
                        for (int e = 0; e < d; ++e) oi[e] += wgt * vj[e];
                    }
                }
                free(p);
            }
    free(win); free(count); free(members); free(fill);
    return err ? ORACLE_ENOMEM : nwin;
}

/* MATE composition ([Review] section 三, MATE: the MA-branch and the TE-branch
 * together replace self-attention; reading R7): the block output is the sum of
 * the two branches projected to the model width,
 *     out[i][n] = sum_k y1[i][k] w1[n][k] + sum_k y2[i][k] w2[n][k],
 * every row of y1 (M x K1) and y2 (M x K2) against every row of w1 (N x K1)
 * and w2 (N x K2), each sum in order of k, the two sums added last. */
int oracle_compose(int64_t M, int K1, int K2, int N, const double *y1, const double *y2, const double *w1,
                   const double *w2, double *out)
{
    if (M < 0 || K1 < 0 || K2 < 0 || N <= 0 || !out || (K1 && (!y1 || !w1)) || (K2 && (!y2 || !w2)))
        return ORACLE_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        for (int n = 0; n < N; ++n) {
            double s1 = 0.0, s2 = 0.0;
            for (int k = 0; k < K1; ++k) s1 += y1[i * K1 + k] * w1[(int64_t)n * K1 + k];
            for (int k = 0; k < K2; ++k) s2 += y2[i * K2 + k] * w2[(int64_t)n * K2 + k];
            out[i * N + n] = s1 + s2;
        }
    }
    return ORACLE_OK;
}


/*
 * MA-branch output side (paper review "LinGen ...", section 三, MA-Branch item 1:
 * the branch is a bidirectional Mamba2 block; reading R9): the bi-SSD output y
 * gated by the front-end's z and normalised, per row i and channel group g,
 *     v_k     = y_k z_k / (1 + exp(-z_k))                 (y times SiLU(z))
 *     out_k   = v_k w_k / sqrt(mean_{k in g} v_k^2 + eps)
 * y, z, out: (M, C) row-major; w: (C); C a multiple of group.
 */
int oracle_gate_norm(int64_t M, int C, int group, double eps, const double *y, const double *z, const double *w,
                     double *out)
{
    if (M < 0 || C <= 0 || group <= 0 || C % group || eps < 0.0 || !y || !z || !w || !out) return ORACLE_EINVAL;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        for (int g0 = 0; g0 < C; g0 += group) {
            double ss = 0.0;
            for (int k = g0; k < g0 + group; ++k) {
                const double zk = z[i * C + k];
                const double v = y[i * C + k] * zk / (1.0 + exp(-zk));
                out[i * C + k] = v;
                ss += v * v;
            }
            const double inv = 1.0 / sqrt(ss / group + eps);
            for (int k = g0; k < g0 + group; ++k) out[i * C + k] = out[i * C + k] * w[k] * inv;
        }
    }
    return ORACLE_OK;
}
