/*
 * monarch_oracle.c -- fp64 CPU oracle for the Monarch attention forward and
 * its gradients.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct
 * definition that the CUDA path is checked against.  Only the tests, the
 * package smoke check and the benchmark's CPU-baseline leg may load it; the
 * product path never does, and this file shares no code, header or constant
 * with the CUDA library.
 *
 * What it computes (MonarchRT: Efficient Attention for Real-Time Video
 * Generation; gist.science/nl/paper/2602.12271, section "Methodologie":
 * the attention matrix is factorised into a product of permutation and
 * block-diagonal matrices; gist.science/zh/paper/2602.12271, section 2.2
 * "Block Alignment": every video axis (f, h, w) lies inside one block
 * dimension; same page, "Tiled Monarch": blocks are subdivided into tiles):
 *
 *     out = M V,     M = P^T B2 P B1
 *
 * for every (batch, head) over the N = T*H*W tokens of a video latent,
 * token index n = (t*H + h)*W + w.
 *
 *   B1 (stage 1) is block diagonal.  FRAME factorisation: one block per
 *      frame t holding its m = H*W tokens.  TILED factorisation: one block
 *      per (frame t, spatial tile) holding tile_h*tile_w tokens.
 *   P  swaps the block index and the in-block index, so B2 acts on the
 *      groups of tokens that share a spatial position (h, w): the T tokens
 *      n = t*H*W + h*W + w, t = 0..T-1.
 *   B2 (stage 2) is block diagonal over those groups.
 *
 * Each diagonal block is a dense softmax attention over the block's own
 * tokens, with scale s = 1/sqrt(d):
 *     y_x = sum_y softmax_y( s <q_x, k_y> ) * val_y
 * Stage 1 uses values V; stage 2 uses the stage-1 outputs Y1 as values
 * (M V = P^T B2 P (B1 V)), with the same Q and K rows restricted to the
 * group.  Indices stay in the original token order throughout, so no final
 * permutation is applied.
 *
 * Readings where the pages say nothing:
 *   - scale d^-1/2 inside every softmax; no mask; no KV cache;
 *   - stage 2 reuses Q and K; its values are stage-1 outputs;
 *   - B1 acts first, then B2;
 *   - layout [B][heads][N][d], contiguous, token order (t, h, w);
 *   - the "refinement iterations" the pages mention are never defined
 *     there: this is the one-pass block-softmax form.
 *
 * Softmax is written the textbook way: subtract the row maximum, exponentiate,
 * divide by the sum.  All arithmetic is double precision.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_FACT_FRAME 0
#define ORACLE_FACT_TILED 1
#define ORACLE_FACT_ROW 2

enum { ORACLE_OK = 0, ORACLE_ERR_ARG = 1, ORACLE_ERR_NOMEM = 2 };

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static int check_shape(int B, int heads, int T, int H, int W, int d,
                       int fact, int tile_h, int tile_w) {
    if (B < 1 || heads < 1 || T < 1 || H < 1 || W < 1 || d < 1) return ORACLE_ERR_ARG;
    if (fact == ORACLE_FACT_TILED) {
        if (tile_h < 1 || tile_w < 1 || H % tile_h != 0 || W % tile_w != 0) return ORACLE_ERR_ARG;
    } else if (fact != ORACLE_FACT_FRAME && fact != ORACLE_FACT_ROW) {
        return ORACLE_ERR_ARG;
    }
    return ORACLE_OK;
}

/* Stage-2 groups: the tokens n = i * stride + g, i = 0 .. len-1, of group g
 * = 0 .. stride-1.  FRAME and TILED: stride H*W (one group per spatial
 * position, across the T frames).  ROW, the (f*h, w) split: stride W (one
 * group per column w, across all T*H frame rows). */
static long stage2_stride(int H, int W, int fact) {
    return fact == ORACLE_FACT_ROW ? (long)W : (long)H * W;
}

/* Number of stage-1 blocks per (batch, head) and tokens per block. */
static void stage1_geometry(int T, int H, int W, int fact, int tile_h, int tile_w,
                            long *nblocks, long *blocklen) {
    if (fact == ORACLE_FACT_TILED) {
        *nblocks = (long)T * (H / tile_h) * (W / tile_w);
        *blocklen = (long)tile_h * tile_w;
    } else if (fact == ORACLE_FACT_ROW) {
        *nblocks = (long)T * H;
        *blocklen = W;
    } else {
        *nblocks = T;
        *blocklen = (long)H * W;
    }
}

/* Token index of member i of stage-1 block b. */
static long stage1_token(long b, long i, int T, int H, int W, int fact,
                         int tile_h, int tile_w) {
    (void)T;
    if (fact == ORACLE_FACT_TILED) {
        long tiles_w = W / tile_w, tiles_h = H / tile_h;
        long per_frame = tiles_h * tiles_w;
        long t = b / per_frame;
        long tile = b % per_frame;
        long ti = tile / tiles_w, tj = tile % tiles_w;
        long hl = i / tile_w, wl = i % tile_w;
        long h = ti * tile_h + hl, w = tj * tile_w + wl;
        return (t * H + h) * (long)W + w;
    }
    if (fact == ORACLE_FACT_ROW) return b * (long)W + i;
    return b * (long)H * W + i;
}

/* Dense softmax attention of one query over a list of keys.
 *   q: the query row; krows/vrows: pointers to the key/value rows of the
 *   block; len keys; logit: scratch of len doubles; y: output row (d). */
static void attend_one(const double *q, const double *const *krows,
                       const double *const *vrows, long len, int d,
                       double scale, double *logit, double *y) {
    double mx = -INFINITY;
    for (long j = 0; j < len; ++j) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += q[c] * krows[j][c];
        logit[j] = scale * acc;
        if (logit[j] > mx) mx = logit[j];
    }
    double z = 0.0;
    for (long j = 0; j < len; ++j) {
        logit[j] = exp(logit[j] - mx);
        z += logit[j];
    }
    for (int c = 0; c < d; ++c) y[c] = 0.0;
    for (long j = 0; j < len; ++j) {
        double p = logit[j] / z;
        for (int c = 0; c < d; ++c) y[c] += p * vrows[j][c];
    }
}

/* Stage 1, y1 = B1 V: every token attends within its stage-1 block.
 * q,k,v,y1: [B*heads][N][d]. */
int oracle_monarch_stage1(const double *q, const double *k, const double *v, double *y1,
                          int B, int heads, int T, int H, int W, int d,
                          int fact, int tile_h, int tile_w) {
    int st = check_shape(B, heads, T, H, W, d, fact, tile_h, tile_w);
    if (st) return st;
    long N = (long)T * H * W;
    long nblocks, len;
    stage1_geometry(T, H, W, fact, tile_h, tile_w, &nblocks, &len);
    double scale = 1.0 / sqrt((double)d);
    long nwork = (long)B * heads * nblocks;
    int failed = 0;
#pragma omp parallel
    {
        const double **kr = (const double **)malloc(sizeof(double *) * len);
        const double **vr = (const double **)malloc(sizeof(double *) * len);
        double *logit = (double *)malloc(sizeof(double) * len);
        if (!kr || !vr || !logit) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long w = 0; w < nwork; ++w) {
                long bh = w / nblocks, b = w % nblocks;
                const double *qb = q + bh * N * d;
                const double *kb = k + bh * N * d;
                const double *vb = v + bh * N * d;
                double *yb = y1 + bh * N * d;
                for (long j = 0; j < len; ++j) {
                    long n = stage1_token(b, j, T, H, W, fact, tile_h, tile_w);
                    kr[j] = kb + n * d;
                    vr[j] = vb + n * d;
                }
                for (long i = 0; i < len; ++i) {
                    long n = stage1_token(b, i, T, H, W, fact, tile_h, tile_w);
                    attend_one(qb + n * d, kr, vr, len, d, scale, logit, yb + n * d);
                }
            }
        }
        free(kr); free(vr); free(logit);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* Stage 2 over the groups of stride `gs` (see stage2_stride): every token
 * attends, with its own Q and K, within its group; the values are the
 * stage-1 outputs. */
static int stage2_groups(const double *q, const double *k, const double *y1, double *out,
                         int B, int heads, long N, long gs, int d) {
    long gl = N / gs;
    double scale = 1.0 / sqrt((double)d);
    long nwork = (long)B * heads * gs;
    int failed = 0;
#pragma omp parallel
    {
        const double **kr = (const double **)malloc(sizeof(double *) * gl);
        const double **vr = (const double **)malloc(sizeof(double *) * gl);
        double *logit = (double *)malloc(sizeof(double) * gl);
        if (!kr || !vr || !logit) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long w = 0; w < nwork; ++w) {
                long bh = w / gs, g = w % gs;
                const double *qb = q + bh * N * d;
                const double *kb = k + bh * N * d;
                const double *yb = y1 + bh * N * d;
                double *ob = out + bh * N * d;
                for (long i = 0; i < gl; ++i) {
                    kr[i] = kb + (i * gs + g) * d;
                    vr[i] = yb + (i * gs + g) * d;
                }
                for (long i = 0; i < gl; ++i)
                    attend_one(qb + (i * gs + g) * d, kr, vr, gl, d, scale, logit, ob + (i * gs + g) * d);
            }
        }
        free(kr); free(vr); free(logit);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* Stage 2, out = P^T B2 P y1, for the frame and tiled splits: every token
 * attends, with its own Q and K, within the group of tokens at the same
 * spatial position across frames; the values are the stage-1 outputs. */
int oracle_monarch_stage2(const double *q, const double *k, const double *y1, double *out,
                          int B, int heads, int T, int H, int W, int d) {
    int st = check_shape(B, heads, T, H, W, d, ORACLE_FACT_FRAME, 0, 0);
    if (st) return st;
    long N = (long)T * H * W;
    return stage2_groups(q, k, y1, out, B, heads, N, stage2_stride(H, W, ORACLE_FACT_FRAME), d);
}

/* Full forward: out = P^T B2 P B1 V.  out must not alias q, k or v. */
int oracle_monarch_fwd(const double *q, const double *k, const double *v, double *out,
                       int B, int heads, int T, int H, int W, int d,
                       int fact, int tile_h, int tile_w) {
    int st = check_shape(B, heads, T, H, W, d, fact, tile_h, tile_w);
    if (st) return st;
    size_t n = (size_t)B * heads * T * H * W * d;
    double *y1 = (double *)malloc(sizeof(double) * n);
    if (!y1) return ORACLE_ERR_NOMEM;
    st = oracle_monarch_stage1(q, k, v, y1, B, heads, T, H, W, d, fact, tile_h, tile_w);
    if (!st) st = stage2_groups(q, k, y1, out, B, heads, (long)T * H * W, stage2_stride(H, W, fact), d);
    free(y1);
    return st;
}

/* Exact output rows for selected stage-2 groups only (for sizes where the
 * full oracle is too slow).  groups holds ngroups pairs (bh, pos), bh in
 * [0, B*heads), pos in [0, H*W).  For each group the T output rows
 * (t = 0..T-1) are written to out_rows[g][t][d].  Each needed stage-1 row
 * is computed exactly as in oracle_monarch_stage1 (same loops, same block). */
int oracle_monarch_fwd_groups(const double *q, const double *k, const double *v,
                              int B, int heads, int T, int H, int W, int d,
                              int fact, int tile_h, int tile_w,
                              const long *groups, int ngroups, double *out_rows) {
    int st = check_shape(B, heads, T, H, W, d, fact, tile_h, tile_w);
    if (st) return st;
    if (fact == ORACLE_FACT_ROW) return ORACLE_ERR_ARG; /* groups here are spatial positions */
    long HW = (long)H * W, N = (long)T * HW;
    long nblocks, len;
    stage1_geometry(T, H, W, fact, tile_h, tile_w, &nblocks, &len);
    long blocks_per_frame = nblocks / T;
    double scale = 1.0 / sqrt((double)d);
    for (int g = 0; g < ngroups; ++g) {
        long bh = groups[2 * g], pos = groups[2 * g + 1];
        if (bh < 0 || bh >= (long)B * heads || pos < 0 || pos >= HW) return ORACLE_ERR_ARG;
    }
    int failed = 0;
#pragma omp parallel
    {
        long cap = len > T ? len : T;
        const double **kr = (const double **)malloc(sizeof(double *) * cap);
        const double **vr = (const double **)malloc(sizeof(double *) * cap);
        double *logit = (double *)malloc(sizeof(double) * cap);
        double *y1 = (double *)malloc(sizeof(double) * (size_t)T * d);
        const double **yr = (const double **)malloc(sizeof(double *) * T);
        if (!kr || !vr || !logit || !y1 || !yr) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int g = 0; g < ngroups; ++g) {
                long bh = groups[2 * g], pos = groups[2 * g + 1];
                const double *qb = q + bh * N * d;
                const double *kb = k + bh * N * d;
                const double *vb = v + bh * N * d;
                long h = pos / W, w = pos % W;
                /* stage 1 for the token (t, pos) of every frame */
                for (int t = 0; t < T; ++t) {
                    long b;
                    if (fact == ORACLE_FACT_TILED) {
                        long tiles_w = W / tile_w;
                        b = (long)t * blocks_per_frame + (h / tile_h) * tiles_w + (w / tile_w);
                    } else {
                        b = t;
                    }
                    for (long j = 0; j < len; ++j) {
                        long n = stage1_token(b, j, T, H, W, fact, tile_h, tile_w);
                        kr[j] = kb + n * d;
                        vr[j] = vb + n * d;
                    }
                    attend_one(qb + (t * HW + pos) * d, kr, vr, len, d, scale, logit,
                               y1 + (size_t)t * d);
                }
                /* stage 2 over the group */
                for (int t = 0; t < T; ++t) {
                    kr[t] = kb + (t * HW + pos) * d;
                    yr[t] = y1 + (size_t)t * d;
                }
                for (int t = 0; t < T; ++t)
                    attend_one(qb + (t * HW + pos) * d, kr, yr, T, d, scale, logit,
                               out_rows + ((size_t)g * T + t) * d);
            }
        }
        free(kr); free(vr); free(logit); free(y1); free(yr);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* ------------------------------------------------------------------ gradients
 *
 * The pages state that their custom kernels run the backward pass as well
 * (gist.science/nl/paper/2602.12271, section "Methodologie";
 * gist.science/zh/paper/2602.12271, section 2.2).  The
 * gradient of the forward above follows from the chain rule alone, so it
 * needs no reading of the pages beyond the forward's.  For one dense block
 * with logits l_j = s <q_x, k_j>, weights p = softmax(l) and output
 * y_x = sum_j p_j val_j, an upstream gradient dy_x gives
 *     dp_j  = <dy_x, val_j>
 *     dl_j  = p_j (dp_j - sum_i p_i dp_i)          (softmax Jacobian)
 *     dq_x += s sum_j dl_j k_j,   dk_j += s dl_j q_x,   dval_j += p_j dy_x.
 * For out = A2(Q, K) Y1 with Y1 = A1(Q, K) V: stage 2's backward takes dy =
 * dout and yields dY1 (its value gradient) and stage-2 parts of dQ and dK;
 * stage 1's backward takes dy = dY1 and yields dV and the stage-1 parts. */

/* Backward of one query of one block: accumulates into dq (the query's row),
 * dkrows[j] and dvrows[j].  logit and dp are scratch of len doubles. */
static void attend_one_bwd(const double *q, const double *const *krows,
                           const double *const *vrows, long len, int d, double scale,
                           const double *dy, double *logit, double *dp, double *dq,
                           double *const *dkrows, double *const *dvrows) {
    double mx = -INFINITY;
    for (long j = 0; j < len; ++j) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += q[c] * krows[j][c];
        logit[j] = scale * acc;
        if (logit[j] > mx) mx = logit[j];
    }
    double z = 0.0;
    for (long j = 0; j < len; ++j) {
        logit[j] = exp(logit[j] - mx);
        z += logit[j];
    }
    double pdp = 0.0;
    for (long j = 0; j < len; ++j) {
        logit[j] /= z; /* now p_j */
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += dy[c] * vrows[j][c];
        dp[j] = acc;
        pdp += logit[j] * acc;
    }
    for (long j = 0; j < len; ++j) {
        double dl = logit[j] * (dp[j] - pdp);
        for (int c = 0; c < d; ++c) {
            dq[c] += scale * dl * krows[j][c];
            dkrows[j][c] += scale * dl * q[c];
            dvrows[j][c] += logit[j] * dy[c];
        }
    }
}

/* Gradients of out = P^T B2 P B1 V with respect to q, k and v for an upstream
 * gradient dout.  All arrays [B*heads][N][d]; dq, dk, dv are overwritten and
 * must not alias the inputs or each other. */
int oracle_monarch_bwd(const double *q, const double *k, const double *v, const double *dout,
                       double *dq, double *dk, double *dv,
                       int B, int heads, int T, int H, int W, int d,
                       int fact, int tile_h, int tile_w) {
    int st = check_shape(B, heads, T, H, W, d, fact, tile_h, tile_w);
    if (st) return st;
    long HW = (long)H * W, N = (long)T * HW;
    size_t n = (size_t)B * heads * N * d;
    double *y1 = (double *)malloc(sizeof(double) * n);
    double *dy1 = (double *)calloc(n, sizeof(double));
    if (!y1 || !dy1) { free(y1); free(dy1); return ORACLE_ERR_NOMEM; }
    memset(dq, 0, sizeof(double) * n);
    memset(dk, 0, sizeof(double) * n);
    memset(dv, 0, sizeof(double) * n);
    st = oracle_monarch_stage1(q, k, v, y1, B, heads, T, H, W, d, fact, tile_h, tile_w);
    if (st) { free(y1); free(dy1); return st; }
    double scale = 1.0 / sqrt((double)d);
    int failed = 0;
    long nblocks, len;
    stage1_geometry(T, H, W, fact, tile_h, tile_w, &nblocks, &len);
    long gs = stage2_stride(H, W, fact), gl = N / gs;
    long maxlen = len > gl ? len : gl;
#pragma omp parallel
    {
        const double **kr = (const double **)malloc(sizeof(double *) * maxlen);
        const double **vr = (const double **)malloc(sizeof(double *) * maxlen);
        double **dkr = (double **)malloc(sizeof(double *) * maxlen);
        double **dvr = (double **)malloc(sizeof(double *) * maxlen);
        double *logit = (double *)malloc(sizeof(double) * maxlen);
        double *dp = (double *)malloc(sizeof(double) * maxlen);
        if (!kr || !vr || !dkr || !dvr || !logit || !dp) {
#pragma omp atomic write
            failed = 1;
        } else {
            /* stage 2: the groups of stride gs (gl tokens each); values Y1 */
#pragma omp for schedule(dynamic, 16)
            for (long w = 0; w < (long)B * heads * gs; ++w) {
                long bh = w / gs, g = w % gs;
                long off = bh * N * d;
                for (long i = 0; i < gl; ++i) {
                    long row = off + (i * gs + g) * d;
                    kr[i] = k + row;
                    vr[i] = y1 + row;
                    dkr[i] = dk + row;
                    dvr[i] = dy1 + row;
                }
                for (long i = 0; i < gl; ++i) {
                    long row = off + (i * gs + g) * d;
                    attend_one_bwd(q + row, kr, vr, gl, d, scale, dout + row, logit, dp, dq + row,
                                   dkr, dvr);
                }
            }
            /* stage 1: blocks; upstream gradient dY1, values V */
#pragma omp for schedule(dynamic, 1)
            for (long w = 0; w < (long)B * heads * nblocks; ++w) {
                long bh = w / nblocks, b = w % nblocks;
                long off = bh * N * d;
                for (long j = 0; j < len; ++j) {
                    long row = off + stage1_token(b, j, T, H, W, fact, tile_h, tile_w) * d;
                    kr[j] = k + row;
                    vr[j] = v + row;
                    dkr[j] = dk + row;
                    dvr[j] = dv + row;
                }
                for (long i = 0; i < len; ++i) {
                    long row = off + stage1_token(b, i, T, H, W, fact, tile_h, tile_w) * d;
                    attend_one_bwd(q + row, kr, vr, len, d, scale, dy1 + row, logit, dp, dq + row,
                                   dkr, dvr);
                }
            }
        }
        free(kr); free(vr); free(dkr); free(dvr); free(logit); free(dp);
    }
    free(y1);
    free(dy1);
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* ------------------------------------------------------------------ autoregressive chunks
 *
 * The pages' main workload is an autoregressive few-step video model
 * (gist.science/it/paper/2602.12271, problem statement: autoregressive
 * generation), and their kernels process the query frames in chunks
 * ("mini-sequence", gist.science/zh/paper/2602.12271, section 2.2).  Reading:
 * a chunk of new frames is generated with the earlier frames as context.
 * With the frame or tiled split, stage-1 blocks never cross frames, so the
 * new chunk's stage 1 needs only its own frames; its stage 2 (the group of a
 * spatial position) attends over the keys and stage-1 outputs of every frame
 * so far.  So the context kept from earlier frames is their K and Y1 (their
 * V is no longer needed).  For the last chunk this gives exactly the full
 * forward's rows for those frames.
 *
 * q, k, v, out, y1_new: [B*heads][T_new*H*W][d] (the new frames);
 * k_cache, y1_cache:    [B*heads][T_old*H*W][d] (may be NULL when T_old = 0). */
int oracle_monarch_fwd_chunk(const double *q, const double *k, const double *v,
                             const double *k_cache, const double *y1_cache,
                             double *out, double *y1_new,
                             int B, int heads, int T_old, int T_new, int H, int W, int d,
                             int fact, int tile_h, int tile_w) {
    if (fact == ORACLE_FACT_ROW || T_old < 0) return ORACLE_ERR_ARG; /* (f*h, w) groups are not per position */
    int st = check_shape(B, heads, T_new, H, W, d, fact, tile_h, tile_w);
    if (st) return st;
    if (T_old > 0 && (!k_cache || !y1_cache)) return ORACLE_ERR_ARG;
    st = oracle_monarch_stage1(q, k, v, y1_new, B, heads, T_new, H, W, d, fact, tile_h, tile_w);
    if (st) return st;
    long HW = (long)H * W, Nn = (long)T_new * HW, No = (long)T_old * HW;
    long tot = (long)T_old + T_new;
    double scale = 1.0 / sqrt((double)d);
    int failed = 0;
#pragma omp parallel
    {
        const double **kr = (const double **)malloc(sizeof(double *) * tot);
        const double **vr = (const double **)malloc(sizeof(double *) * tot);
        double *logit = (double *)malloc(sizeof(double) * tot);
        if (!kr || !vr || !logit) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long w = 0; w < (long)B * heads * HW; ++w) {
                long bh = w / HW, pos = w % HW;
                for (long t = 0; t < T_old; ++t) {
                    kr[t] = k_cache + (bh * No + t * HW + pos) * d;
                    vr[t] = y1_cache + (bh * No + t * HW + pos) * d;
                }
                for (long t = 0; t < T_new; ++t) {
                    kr[T_old + t] = k + (bh * Nn + t * HW + pos) * d;
                    vr[T_old + t] = y1_new + (bh * Nn + t * HW + pos) * d;
                }
                for (long t = 0; t < T_new; ++t) {
                    long row = (bh * Nn + t * HW + pos) * d;
                    attend_one(q + row, kr, vr, tot, d, scale, logit, out + row);
                }
            }
        }
        free(kr); free(vr); free(logit);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}
