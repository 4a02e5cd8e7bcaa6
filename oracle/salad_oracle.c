/*
 * CPU oracle for the SALAD hybrid attention layer.  TEST INFRASTRUCTURE ONLY:
 * only the tests, the smoke check and the benchmark's CPU-baseline leg may load
 * this library.  It shares no code with the CUDA path.
 *
 * Plain fp64 C, written from the definitions in the SALAD pages:
 *   - the parallel dual-branch layer and the shared Q/K/V
 *     (SALAD technical summary, section 2.1 "Architecture design");
 *   - the sparse branch as static spatio-temporal sliding-window attention
 *     (ST-SWA, a baseline in Figure 1 of the sciencestack SALAD page; the
 *     summary's section 5 names sliding windows as the static kind of sparse
 *     attention the method applies to);
 *   - the ReLU-based O(N) linear branch (summary section 2.1);
 *   - the static projection on the linear output (summary section 2.2, LWSS);
 *   - a scalar gate in (0,1) that depends on the input and scales the linear
 *     branch (summary section 2.2, ITADS; the sciencestack TL;DR);
 *   - dropping the linear branch when the gate is 0 (summary section 2.3).
 * The pages give no formula; the readings taken where they are silent are:
 *   token n <-> (t, y, x) with n = (t*H + y)*W + x; key/query block I holds
 *   tokens [I*blk, min(N, (I+1)*blk)); block pair (I, J) is kept when some real
 *   token pair i in I, j in J has |dt| <= wt, |dy| <= wh, |dx| <= ww; softmax
 *   scale tau (1/sqrt(d) by default); phi = ReLU on q and k; denominator
 *   phi(q).z + eps; y = o_lin W (row vector times W[c][e]); out = o_sp + g*y,
 *   with out = o_sp exactly when g == 0.
 *
 * Parity pins (tests/test_oracle_*.py): token-pair brute force for the mask,
 * dense element-masked attention, torch SDPA for the full window, the naive
 * O(N^2) linear attention, and the closed-form limits.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Block mask.  For every head h and query block I: visit every real token i of
 * I, every grid point j inside i's window box, and mark the key block holding
 * j.  The x-extent of the box on one (t, y) row is a contiguous token range, so
 * the blocks that range touches are marked directly.
 *
 * windows: int32 [Hh][3] = (wt, wh, ww).  row_ptr: int32 [Hh*nb + 1], global
 * offsets into col_idx.  col_idx: int32 [cap] (may be NULL when cap == 0).
 * Returns the total number of kept block pairs; col_idx is only written when
 * it fits (the caller compares the return value with cap).
 */
int64_t oracle_block_mask(int T, int H, int W, int blk, int Hh, const int32_t *windows,
                          int32_t *row_ptr, int32_t *col_idx, int64_t cap) {
    const int64_t N = (int64_t)T * H * W;
    const int64_t nb = (N + blk - 1) / blk;
    unsigned char *mark = (unsigned char *)malloc((size_t)(nb * nb));
    int64_t total = 0;
    for (int h = 0; h < Hh; ++h) {
        const int wt = windows[3 * h + 0], wh = windows[3 * h + 1], ww = windows[3 * h + 2];
        memset(mark, 0, (size_t)(nb * nb));
#pragma omp parallel for schedule(dynamic)
        for (int64_t I = 0; I < nb; ++I) {
            unsigned char *row = mark + I * nb;
            const int64_t i_end = (I + 1) * blk < N ? (I + 1) * blk : N;
            for (int64_t i = I * blk; i < i_end; ++i) {
                const int x = (int)(i % W), y = (int)((i / W) % H), t = (int)(i / ((int64_t)W * H));
                for (int t2 = t - wt; t2 <= t + wt; ++t2) {
                    if (t2 < 0 || t2 >= T) continue;
                    for (int y2 = y - wh; y2 <= y + wh; ++y2) {
                        if (y2 < 0 || y2 >= H) continue;
                        const int x_lo = x - ww < 0 ? 0 : x - ww;
                        const int x_hi = x + ww > W - 1 ? W - 1 : x + ww;
                        const int64_t base = ((int64_t)t2 * H + y2) * W;
                        for (int64_t J = (base + x_lo) / blk; J <= (base + x_hi) / blk; ++J)
                            row[J] = 1;
                    }
                }
            }
        }
        for (int64_t I = 0; I < nb; ++I) {
            row_ptr[h * nb + I] = (int32_t)total;
            for (int64_t J = 0; J < nb; ++J) {
                if (mark[I * nb + J]) {
                    if (col_idx && total < cap) col_idx[total] = (int32_t)J;
                    ++total;
                }
            }
        }
    }
    row_ptr[Hh * nb] = (int32_t)total;
    free(mark);
    return total;
}

/*
 * 3-D tile blocks (the SPADE explainer, section 1, puts attention on a 3-D grid
 * of video blocks).  Reading taken: the T x H x W grid is cut into bt x bh x bw
 * boxes (bt divides T; boxes at the H and W edges may stick out of the grid),
 * numbered in raster order over (box t, box y, box x).  Box I has bt*bh*bw
 * slots, slot s = (tt*bh + yy)*bw + xx for the point (t0 + tt, y0 + yy, x0 + xx);
 * a slot outside the grid holds no token.  geom = {T, H, W, bt, bh, bw}.
 * Writes the token of every slot of block I (-1 for a slot without one) and
 * returns the slot count; without geom a block is `blk` raster tokens.
 */
static int block_tokens(const int32_t *geom, int64_t N, int blk, int64_t I, int64_t *tok) {
    if (!geom) {
        for (int s = 0; s < blk; ++s) tok[s] = I * blk + s < N ? I * blk + s : -1;
        return blk;
    }
    const int T = geom[0], H = geom[1], W = geom[2], bt = geom[3], bh = geom[4], bw = geom[5];
    const int nh = (H + bh - 1) / bh, nw = (W + bw - 1) / bw;
    const int ti = (int)(I / ((int64_t)nh * nw)), yi = (int)((I / nw) % nh), xi = (int)(I % nw);
    int s = 0;
    for (int tt = 0; tt < bt; ++tt)
        for (int yy = 0; yy < bh; ++yy)
            for (int xx = 0; xx < bw; ++xx, ++s) {
                const int t = ti * bt + tt, y = yi * bh + yy, x = xi * bw + xx;
                tok[s] = (t < T && y < H && x < W) ? ((int64_t)t * H + y) * W + x : -1;
            }
    return s;
}

/*
 * Window mask over 3-D tile blocks (geometry as for block_tokens): box pair
 * (I, J) is kept when some real token of I and some real token of J lie within
 * the window, found by brute force over the token pairs.  row_ptr: int32
 * [Hh*nb + 1], col_idx as for oracle_block_mask; returns the kept pair count.
 */
int64_t oracle_tile_mask(const int32_t *geom, int Hh, const int32_t *windows, int32_t *row_ptr, int32_t *col_idx,
                         int64_t cap) {
    const int T = geom[0], H = geom[1], W = geom[2], bt = geom[3], bh = geom[4], bw = geom[5];
    const int nb = (T / bt) * ((H + bh - 1) / bh) * ((W + bw - 1) / bw), slots = bt * bh * bw;
    const int64_t N = (int64_t)T * H * W;
    unsigned char *mark = (unsigned char *)calloc((size_t)nb * nb, 1);
    int64_t total = 0;
    for (int h = 0; h < Hh; ++h) {
        const int wt = windows[3 * h + 0], wh = windows[3 * h + 1], ww = windows[3 * h + 2];
        memset(mark, 0, (size_t)nb * nb);
#pragma omp parallel for schedule(dynamic)
        for (int I = 0; I < nb; ++I) {
            int64_t *ti = (int64_t *)malloc(sizeof(int64_t) * slots), *tj = (int64_t *)malloc(sizeof(int64_t) * slots);
            block_tokens(geom, N, 0, I, ti);
            for (int J = 0; J < nb; ++J) {
                block_tokens(geom, N, 0, J, tj);
                int kept = 0;
                for (int a = 0; a < slots && !kept; ++a) {
                    if (ti[a] < 0) continue;
                    const int64_t x = ti[a] % W, y = (ti[a] / W) % H, t = ti[a] / ((int64_t)W * H);
                    for (int c = 0; c < slots; ++c) {
                        if (tj[c] < 0) continue;
                        const int64_t x2 = tj[c] % W, y2 = (tj[c] / W) % H, t2 = tj[c] / ((int64_t)W * H);
                        if (llabs(t - t2) <= wt && llabs(y - y2) <= wh && llabs(x - x2) <= ww) {
                            kept = 1;
                            break;
                        }
                    }
                }
                mark[(int64_t)I * nb + J] = (unsigned char)kept;
            }
            free(ti);
            free(tj);
        }
        for (int I = 0; I < nb; ++I) {
            row_ptr[h * nb + I] = (int32_t)total;
            for (int J = 0; J < nb; ++J)
                if (mark[(int64_t)I * nb + J]) {
                    if (col_idx && total < cap) col_idx[total] = J;
                    ++total;
                }
        }
    }
    row_ptr[Hh * nb] = (int32_t)total;
    free(mark);
    return total;
}

/*
 * Linear-branch state of every (b, h), over all N real tokens (global and
 * non-causal: the summary's section 2.1 gives the linear branch the job of
 * interactions between all tokens):
 *   z[c]    = sum_j relu(k_j[c])
 *   S[c][e] = sum_j relu(k_j[c]) * v_j[e]
 * q/k/v are bf16 bits [B][N][Hh][d].  S: fp64 [B*Hh][d][d], z: fp64 [B*Hh][d].
 */
void oracle_linear_state(const uint16_t *k, const uint16_t *v, int B, int N, int Hh, int d,
                         double *S, double *z) {
#pragma omp parallel for schedule(static)
    for (int bh = 0; bh < B * Hh; ++bh) {
        const int b = bh / Hh, h = bh % Hh;
        double *Sb = S + (int64_t)bh * d * d;
        double *zb = z + (int64_t)bh * d;
        double *pk = (double *)malloc(sizeof(double) * d);
        double *pv = (double *)malloc(sizeof(double) * d);
        for (int64_t i = 0; i < (int64_t)d * d; ++i) Sb[i] = 0.0;
        for (int c = 0; c < d; ++c) zb[c] = 0.0;
        for (int64_t j = 0; j < N; ++j) {
            const int64_t off = (((int64_t)b * N + j) * Hh + h) * d;
            for (int c = 0; c < d; ++c) {
                const double kv = bf16_to_double(k[off + c]);
                pk[c] = kv > 0.0 ? kv : 0.0;
                pv[c] = bf16_to_double(v[off + c]);
            }
            for (int c = 0; c < d; ++c) {
                if (pk[c] == 0.0) continue; /* relu(k) = 0 adds exact zeros */
                zb[c] += pk[c];
                for (int e = 0; e < d; ++e) Sb[(int64_t)c * d + e] += pk[c] * pv[e];
            }
        }
        free(pk);
        free(pv);
    }
}

/*
 * Forward pass for a list of (bh, I) query blocks.
 *   pairs:   int32 [npairs][2] = (b*Hh + h, I)
 *   S, z:    from oracle_linear_state (may be NULL when every gate of the listed
 *            pairs is 0)
 *   w_proj:  bf16 bits [d][d];  gate: float [B][Hh]
 *   out:     fp64 [npairs][blk][d]; rows past N are left untouched.
 *   o_sp, o_lin (nullable): same layout, the sparse branch and the normalised
 *            linear branch before the projection.
 * For each real query i of the block:
 *   s_j  = tau * q_i . k_j over all real tokens j of the kept key blocks
 *   o_sp = sum_j exp(s_j - max s) v_j / sum_j exp(s_j - max s)
 *   if g == 0: out = o_sp (linear branch dropped)
 *   else:      u = relu(q_i)^T S, den = relu(q_i) . z, o_lin = u / (den + eps),
 *              y = o_lin W, out = o_sp + g * y
 */
void oracle_forward_blocks(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int N,
                           int Hh, int d, int blk, const int32_t *row_ptr, const int32_t *col_idx,
                           const uint16_t *w_proj, const float *gate, double tau, double eps,
                           const double *S, const double *z, const int32_t *pairs, int npairs,
                           double *out, double *o_sp, double *o_lin, int mask_per_bh, const int32_t *geom) {
    /* geom: 3-D tile blocks (see block_tokens; then blk = bt*bh*bw), or NULL */
    const int nb = geom ? (geom[0] / geom[3]) * ((geom[1] + geom[4] - 1) / geom[4]) *
                              ((geom[2] + geom[5] - 1) / geom[5])
                        : (N + blk - 1) / blk;
    double *W = (double *)malloc(sizeof(double) * d * d);
    for (int i = 0; i < d * d; ++i) W[i] = bf16_to_double(w_proj[i]);
#pragma omp parallel for schedule(dynamic)
    for (int p = 0; p < npairs; ++p) {
        const int bh = pairs[2 * p], I = pairs[2 * p + 1];
        const int b = bh / Hh, h = bh % Hh;
        const double g = (double)gate[bh];
        const int mrow = (mask_per_bh ? bh : h) * nb + I; /* the mask has rows per head or per (b, h) */
        const int32_t r0 = row_ptr[mrow], r1 = row_ptr[mrow + 1];
        /* gather the real key tokens of the kept key blocks, in CSR order */
        int64_t *slot_tok = (int64_t *)malloc(sizeof(int64_t) * blk);
        const int64_t nkeys = (int64_t)(r1 - r0) * blk;
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (nkeys > 0 ? nkeys : 1));
        double *s = (double *)malloc(sizeof(double) * (nkeys > 0 ? nkeys : 1));
        double *qi = (double *)malloc(sizeof(double) * d);
        double *acc = (double *)malloc(sizeof(double) * d);
        double *lin = (double *)malloc(sizeof(double) * d);
        int64_t nk = 0;
        for (int32_t r = r0; r < r1; ++r) {
            block_tokens(geom, N, blk, col_idx[r], slot_tok);
            for (int sl = 0; sl < blk; ++sl)
                if (slot_tok[sl] >= 0) keys[nk++] = slot_tok[sl];
        }
        int64_t *qtok = (int64_t *)malloc(sizeof(int64_t) * blk);
        block_tokens(geom, N, blk, I, qtok);
        for (int qs = 0; qs < blk; ++qs) {
            if (qtok[qs] < 0) continue;
            const int64_t i = qtok[qs];
            const int64_t qoff = (((int64_t)b * N + i) * Hh + h) * d;
            for (int c = 0; c < d; ++c) qi[c] = bf16_to_double(q[qoff + c]);
            /* sparse branch: exact softmax over the kept keys */
            double m = -INFINITY;
            for (int64_t t = 0; t < nk; ++t) {
                const int64_t koff = (((int64_t)b * N + keys[t]) * Hh + h) * d;
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += qi[c] * bf16_to_double(k[koff + c]);
                s[t] = tau * dot;
                if (s[t] > m) m = s[t];
            }
            double den = 0.0;
            for (int c = 0; c < d; ++c) acc[c] = 0.0;
            for (int64_t t = 0; t < nk; ++t) {
                const double pexp = exp(s[t] - m);
                const int64_t voff = (((int64_t)b * N + keys[t]) * Hh + h) * d;
                den += pexp;
                for (int c = 0; c < d; ++c) acc[c] += pexp * bf16_to_double(v[voff + c]);
            }
            const int64_t ooff = ((int64_t)p * blk + qs) * d;
            for (int c = 0; c < d; ++c) {
                acc[c] /= den;
                if (o_sp) o_sp[ooff + c] = acc[c];
            }
            /* linear branch, projection and gate */
            if (g != 0.0 || o_lin) {
                const double *Sb = S + (int64_t)bh * d * d;
                const double *zb = z + (int64_t)bh * d;
                double dn = 0.0;
                for (int c = 0; c < d; ++c) {
                    const double pq = qi[c] > 0.0 ? qi[c] : 0.0;
                    dn += pq * zb[c];
                }
                for (int e = 0; e < d; ++e) {
                    double u = 0.0;
                    for (int c = 0; c < d; ++c) {
                        const double pq = qi[c] > 0.0 ? qi[c] : 0.0;
                        u += pq * Sb[(int64_t)c * d + e];
                    }
                    lin[e] = u / (dn + eps);
                    if (o_lin) o_lin[ooff + e] = lin[e];
                }
            }
            if (g == 0.0) {
                for (int c = 0; c < d; ++c) out[ooff + c] = acc[c];
            } else {
                for (int e = 0; e < d; ++e) {
                    double y = 0.0;
                    for (int c = 0; c < d; ++c) y += lin[c] * W[c * d + e];
                    out[ooff + e] = acc[e] + g * y;
                }
            }
        }
        free(keys);
        free(slot_tok);
        free(qtok);
        free(s);
        free(qi);
        free(acc);
        free(lin);
    }
    free(W);
}

/*
 * Backward pass of the layer (the gradients the fine-tuning of the SALAD summary,
 * section 3, needs: the sparse branch, the linear branch, the static projection
 * and the gate), for raster blocks, given dout = dL/dout fp64 [B][N][Hh][d].
 * Written from the forward above by the chain rule, in the forward's notation:
 *   sparse:  p_ij = softmax_j(s_ij), s_ij = tau q_i.k_j over the kept keys;
 *            dp_ij = dout_i.v_j, D_i = sum_j p_ij dp_ij, ds_ij = p_ij (dp_ij - D_i);
 *            dq_i += tau sum_j ds_ij k_j, dk_j += tau sum_i ds_ij q_i,
 *            dv_j += sum_i p_ij dout_i
 *   linear:  a_i = relu(q_i), den_i = a_i.z + eps, u_i = a_i^T S,
 *            o_i = u_i / den_i, y_i = o_i W;
 *            dgate[b][h] = sum_i dout_i.y_i   (also where g = 0);
 *            dy_i = g dout_i, dW += sum_i o_i^T dy_i (over every (b, h));
 *            do_i = dy_i W^T, du_i = do_i / den_i, dden_i = -(do_i.o_i) / den_i;
 *            dS = sum_i a_i du_i^T, dz = sum_i dden_i a_i;
 *            dq_i += [q_i > 0] (S du_i + dden_i z);
 *            dk_j += [k_j > 0] (dS v_j + dz), dv_j += dS^T relu(k_j)
 * (the derivative of relu at 0 is taken as 0).  Outputs fp64: dq, dk, dv
 * [B][N][Hh][d], dw [d][d], dgate [B][Hh].  mask_per_bh as in the forward.
 */
static int row_has(const int32_t *cols, int32_t n, int32_t J) {
    int32_t lo = 0, hi = n; /* columns ascending */
    while (lo < hi) {
        const int32_t mid = (lo + hi) / 2;
        if (cols[mid] < J) lo = mid + 1;
        else hi = mid;
    }
    return lo < n && cols[lo] == J;
}

void oracle_backward(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int N, int Hh, int d,
                     int blk, const int32_t *row_ptr, const int32_t *col_idx, const uint16_t *w_proj,
                     const float *gate, double tau, double eps, const double *dout, int mask_per_bh, double *dq,
                     double *dk, double *dv, double *dw, double *dgate) {
    const int nb = (N + blk - 1) / blk;
    const int BH = B * Hh;
    const int64_t rows = (int64_t)BH * N; /* per-row scratch, indexed (bh * N + i) */
    double *W = (double *)malloc(sizeof(double) * d * d);
    double *S = (double *)malloc(sizeof(double) * BH * d * d);
    double *z = (double *)malloc(sizeof(double) * BH * d);
    double *dS = (double *)calloc((size_t)BH * d * d, sizeof(double));
    double *dz = (double *)calloc((size_t)BH * d, sizeof(double));
    double *dWbh = (double *)calloc((size_t)BH * d * d, sizeof(double));
    double *lse = (double *)malloc(sizeof(double) * rows);
    double *Dr = (double *)malloc(sizeof(double) * rows);
    double *du = (double *)malloc(sizeof(double) * rows * d);
    double *dden = (double *)malloc(sizeof(double) * rows);
    double *orow = (double *)malloc(sizeof(double) * rows * d);
    double *yg = (double *)malloc(sizeof(double) * rows);
    for (int i = 0; i < d * d; ++i) W[i] = bf16_to_double(w_proj[i]);
    oracle_linear_state(k, v, B, N, Hh, d, S, z);

    /* queries: softmax statistics, D_i, dq_i and the linear branch's per-row terms */
#pragma omp parallel for schedule(dynamic)
    for (int64_t task = 0; task < (int64_t)BH * nb; ++task) {
        const int bh = (int)(task / nb), I = (int)(task % nb), b = bh / Hh, h = bh % Hh;
        const double g = (double)gate[bh];
        const int mrow = (mask_per_bh ? bh : h) * nb + I;
        const int32_t r0 = row_ptr[mrow], r1 = row_ptr[mrow + 1];
        const int64_t nkeys = (int64_t)(r1 - r0) * blk;
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (nkeys > 0 ? nkeys : 1));
        double *sc = (double *)malloc(sizeof(double) * (nkeys > 0 ? nkeys : 1));
        double *qi = (double *)malloc(sizeof(double) * d);
        double *gi = (double *)malloc(sizeof(double) * d);
        double *acc = (double *)malloc(sizeof(double) * d);
        double *y = (double *)malloc(sizeof(double) * d);
        double *dov = (double *)malloc(sizeof(double) * d);
        int64_t nk = 0;
        for (int32_t r = r0; r < r1; ++r)
            for (int64_t j = (int64_t)col_idx[r] * blk; j < (int64_t)(col_idx[r] + 1) * blk && j < N; ++j)
                keys[nk++] = j;
        for (int64_t i = (int64_t)I * blk; i < (int64_t)(I + 1) * blk && i < N; ++i) {
            const int64_t off = (((int64_t)b * N + i) * Hh + h) * d;
            const int64_t ri = (int64_t)bh * N + i;
            for (int c = 0; c < d; ++c) {
                qi[c] = bf16_to_double(q[off + c]);
                gi[c] = dout[off + c];
                acc[c] = 0.0;
            }
            /* sparse branch: the probabilities, then D_i and dq_i */
            double m = -INFINITY, l = 0.0;
            for (int64_t t = 0; t < nk; ++t) {
                const int64_t koff = (((int64_t)b * N + keys[t]) * Hh + h) * d;
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += qi[c] * bf16_to_double(k[koff + c]);
                sc[t] = tau * dot;
                if (sc[t] > m) m = sc[t];
            }
            for (int64_t t = 0; t < nk; ++t) l += exp(sc[t] - m);
            lse[ri] = m + log(l);
            double D = 0.0;
            for (int64_t t = 0; t < nk; ++t) {
                const int64_t voff = (((int64_t)b * N + keys[t]) * Hh + h) * d;
                double dp = 0.0;
                for (int c = 0; c < d; ++c) dp += gi[c] * bf16_to_double(v[voff + c]);
                sc[t] = exp(sc[t] - lse[ri]); /* p_ij */
                D += sc[t] * dp;
            }
            Dr[ri] = D;
            for (int64_t t = 0; t < nk; ++t) {
                const int64_t kvoff = (((int64_t)b * N + keys[t]) * Hh + h) * d;
                double dp = 0.0;
                for (int c = 0; c < d; ++c) dp += gi[c] * bf16_to_double(v[kvoff + c]);
                const double ds = sc[t] * (dp - D);
                for (int c = 0; c < d; ++c) acc[c] += tau * ds * bf16_to_double(k[kvoff + c]);
            }
            /* linear branch */
            const double *Sb = S + (int64_t)bh * d * d;
            const double *zb = z + (int64_t)bh * d;
            double den = eps;
            for (int c = 0; c < d; ++c) den += (qi[c] > 0.0 ? qi[c] : 0.0) * zb[c];
            double *o = orow + ri * d;
            for (int e = 0; e < d; ++e) {
                double u = 0.0;
                for (int c = 0; c < d; ++c) u += (qi[c] > 0.0 ? qi[c] : 0.0) * Sb[(int64_t)c * d + e];
                o[e] = u / den;
            }
            double ygi = 0.0;
            for (int f = 0; f < d; ++f) {
                y[f] = 0.0;
                for (int e = 0; e < d; ++e) y[f] += o[e] * W[e * d + f];
                ygi += gi[f] * y[f];
            }
            yg[ri] = ygi;
            double od = 0.0;
            for (int e = 0; e < d; ++e) {
                dov[e] = 0.0;
                for (int f = 0; f < d; ++f) dov[e] += W[e * d + f] * g * gi[f]; /* do = (g dout) W^T */
                od += dov[e] * o[e];
            }
            dden[ri] = -od / den;
            for (int e = 0; e < d; ++e) du[ri * d + e] = dov[e] / den;
            for (int c = 0; c < d; ++c) {
                if (!(qi[c] > 0.0)) continue;
                double da = dden[ri] * zb[c];
                for (int e = 0; e < d; ++e) da += Sb[(int64_t)c * d + e] * du[ri * d + e];
                acc[c] += da;
            }
            for (int c = 0; c < d; ++c) dq[off + c] = acc[c];
        }
        free(keys);
        free(sc);
        free(qi);
        free(gi);
        free(acc);
        free(y);
        free(dov);
    }

    /* per (b, h): dS, dz, the gate's gradient and this (b, h)'s share of dW */
#pragma omp parallel for schedule(static)
    for (int bh = 0; bh < BH; ++bh) {
        const int b = bh / Hh, h = bh % Hh;
        const double g = (double)gate[bh];
        double dg = 0.0;
        for (int64_t i = 0; i < N; ++i) {
            const int64_t off = (((int64_t)b * N + i) * Hh + h) * d;
            const int64_t ri = (int64_t)bh * N + i;
            dg += yg[ri];
            for (int c = 0; c < d; ++c) {
                const double a = bf16_to_double(q[off + c]);
                if (a > 0.0) {
                    dz[(int64_t)bh * d + c] += dden[ri] * a;
                    for (int e = 0; e < d; ++e) dS[((int64_t)bh * d + c) * d + e] += a * du[ri * d + e];
                }
            }
            for (int e = 0; e < d; ++e)
                for (int f = 0; f < d; ++f)
                    dWbh[((int64_t)bh * d + e) * d + f] += orow[ri * d + e] * g * dout[off + f];
        }
        dgate[bh] = dg;
    }
    for (int i = 0; i < d * d; ++i) {
        double sum = 0.0;
        for (int bh = 0; bh < BH; ++bh) sum += dWbh[(int64_t)bh * d * d + i];
        dw[i] = sum;
    }

    /* keys: every query of every query block whose row keeps the key's block */
#pragma omp parallel for schedule(dynamic)
    for (int64_t task = 0; task < (int64_t)BH * nb; ++task) {
        const int bh = (int)(task / nb), J = (int)(task % nb), b = bh / Hh, h = bh % Hh;
        const double *dSb = dS + (int64_t)bh * d * d;
        const double *dzb = dz + (int64_t)bh * d;
        double *kj = (double *)malloc(sizeof(double) * d);
        double *vj = (double *)malloc(sizeof(double) * d);
        double *ak = (double *)malloc(sizeof(double) * d);
        double *av = (double *)malloc(sizeof(double) * d);
        for (int64_t j = (int64_t)J * blk; j < (int64_t)(J + 1) * blk && j < N; ++j) {
            const int64_t off = (((int64_t)b * N + j) * Hh + h) * d;
            for (int c = 0; c < d; ++c) {
                kj[c] = bf16_to_double(k[off + c]);
                vj[c] = bf16_to_double(v[off + c]);
                ak[c] = 0.0;
                av[c] = 0.0;
            }
            for (int I = 0; I < nb; ++I) {
                const int mrow = (mask_per_bh ? bh : h) * nb + I;
                if (!row_has(col_idx + row_ptr[mrow], row_ptr[mrow + 1] - row_ptr[mrow], J)) continue;
                for (int64_t i = (int64_t)I * blk; i < (int64_t)(I + 1) * blk && i < N; ++i) {
                    const int64_t qoff = (((int64_t)b * N + i) * Hh + h) * d;
                    const int64_t ri = (int64_t)bh * N + i;
                    double dot = 0.0, dp = 0.0;
                    for (int c = 0; c < d; ++c) {
                        dot += bf16_to_double(q[qoff + c]) * kj[c];
                        dp += dout[qoff + c] * vj[c];
                    }
                    const double p = exp(tau * dot - lse[ri]);
                    const double ds = p * (dp - Dr[ri]);
                    for (int c = 0; c < d; ++c) {
                        ak[c] += tau * ds * bf16_to_double(q[qoff + c]);
                        av[c] += p * dout[qoff + c];
                    }
                }
            }
            /* linear branch through S and z */
            for (int c = 0; c < d; ++c) {
                if (kj[c] > 0.0) {
                    double t = dzb[c];
                    for (int e = 0; e < d; ++e) t += dSb[(int64_t)c * d + e] * vj[e];
                    ak[c] += t;
                }
            }
            for (int e = 0; e < d; ++e) {
                double t = 0.0;
                for (int c = 0; c < d; ++c)
                    if (kj[c] > 0.0) t += dSb[(int64_t)c * d + e] * kj[c];
                av[e] += t;
            }
            for (int c = 0; c < d; ++c) {
                dk[off + c] = ak[c];
                dv[off + c] = av[c];
            }
        }
        free(kj);
        free(vj);
        free(ak);
        free(av);
    }
    free(W);
    free(S);
    free(z);
    free(dS);
    free(dz);
    free(dWbh);
    free(lse);
    free(Dr);
    free(du);
    free(dden);
    free(orow);
    free(yg);
}

/*
 * Log-sum-exp of the sparse branch's softmax for every query row (the quantity
 * a training forward keeps for the backward pass):
 *   lse[b][h][i] = log sum_j exp(tau q_i . k_j) over the real tokens j of the
 *   key blocks kept for i's block (raster blocks); -inf for a row with no keys.
 * fp64, natural log; lse is [B][Hh][N].  mask_per_bh as in the forward.
 */
void oracle_lse(const uint16_t *q, const uint16_t *k, int B, int N, int Hh, int d, int blk,
                const int32_t *row_ptr, const int32_t *col_idx, double tau, int mask_per_bh, double *lse) {
    const int nb = (N + blk - 1) / blk;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int bh = 0; bh < B * Hh; ++bh) {
        for (int I = 0; I < nb; ++I) {
            const int b = bh / Hh, h = bh % Hh;
            const int mrow = (mask_per_bh ? bh : h) * nb + I;
            for (int64_t i = (int64_t)I * blk; i < (int64_t)(I + 1) * blk && i < N; ++i) {
                const int64_t qoff = (((int64_t)b * N + i) * Hh + h) * d;
                double m = -INFINITY;
                for (int pass = 0; pass < 2; ++pass) {
                    double l = 0.0;
                    for (int32_t r = row_ptr[mrow]; r < row_ptr[mrow + 1]; ++r) {
                        for (int64_t j = (int64_t)col_idx[r] * blk; j < (int64_t)(col_idx[r] + 1) * blk && j < N; ++j) {
                            const int64_t koff = (((int64_t)b * N + j) * Hh + h) * d;
                            double dot = 0.0;
                            for (int c = 0; c < d; ++c)
                                dot += bf16_to_double(q[qoff + c]) * bf16_to_double(k[koff + c]);
                            if (pass == 0) {
                                if (tau * dot > m) m = tau * dot;
                            } else {
                                l += exp(tau * dot - m);
                            }
                        }
                    }
                    if (pass == 1) lse[(int64_t)bh * N + i] = l > 0.0 ? m + log(l) : -INFINITY;
                }
            }
        }
    }
}

/* Threads the OpenMP runtime will use (reported next to the CPU timings). */
/*
 * Top-K dynamic block mask.  The SALAD summary (section 5) names Top-K dynamic
 * sparse attention among the kinds of sparse attention the method applies to,
 * and gives no scoring rule.  Reading taken here: per (b, h), the mean of q
 * over the real tokens of each block and the same for k; the score of block
 * pair (I, J) is the dot product of the two means; row (b, h, I) keeps the
 * `keep` highest scores (ties: the smaller J), listed in ascending J.  The
 * arithmetic is fixed, in fp32, so that another implementation reproduces the
 * scores bit for bit and takes the same integer decisions: each mean is the
 * sum over the block's tokens in token order, then one division by the token
 * count; each score is a chain of fused multiply-adds in feature order,
 * starting from 0.
 *
 * q, k: bf16 [B][N][Hh][d].  kk = min(keep, nb) (keep >= 1).  row_ptr: int32
 * [B*Hh*nb + 1] = r * kk for row r = (b*Hh + h)*nb + I; col_idx: int32
 * [B*Hh*nb*kk].  Returns kk (0 for keep < 1).
 */
typedef struct {
    float score;
    int32_t j;
} scored_block;

static int by_score_desc_then_j(const void *a, const void *b) {
    const scored_block *x = (const scored_block *)a, *y = (const scored_block *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

static int by_int_asc(const void *a, const void *b) {
    const int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

static float bf16_to_float(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

int oracle_topk_mask(const uint16_t *q, const uint16_t *k, int B, int N, int Hh, int d, int blk, int keep,
                     int32_t *row_ptr, int32_t *col_idx) {
    if (keep < 1) return 0;
    const int nb = (N + blk - 1) / blk;
    const int kk = keep < nb ? keep : nb;
    const int64_t rows = (int64_t)B * Hh * nb;
    for (int64_t r = 0; r <= rows; ++r) row_ptr[r] = (int32_t)(r * kk);
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < B * Hh; ++bh) {
        const int b = bh / Hh, h = bh % Hh;
        float *qm = (float *)malloc(sizeof(float) * nb * d);
        float *km = (float *)malloc(sizeof(float) * nb * d);
        scored_block *sc = (scored_block *)malloc(sizeof(scored_block) * nb);
        int32_t *kept = (int32_t *)malloc(sizeof(int32_t) * kk);
        for (int I = 0; I < nb; ++I) {
            const int t0 = I * blk, t1 = (I + 1) * blk < N ? (I + 1) * blk : N;
            for (int c = 0; c < d; ++c) {
                float sq = 0.f, sk = 0.f;
                for (int t = t0; t < t1; ++t) {
                    const int64_t off = (((int64_t)b * N + t) * Hh + h) * d + c;
                    sq += bf16_to_float(q[off]);
                    sk += bf16_to_float(k[off]);
                }
                qm[(int64_t)I * d + c] = sq / (float)(t1 - t0);
                km[(int64_t)I * d + c] = sk / (float)(t1 - t0);
            }
        }
        for (int I = 0; I < nb; ++I) {
            for (int J = 0; J < nb; ++J) {
                float a = 0.f;
                for (int c = 0; c < d; ++c) a = fmaf(qm[(int64_t)I * d + c], km[(int64_t)J * d + c], a);
                sc[J].score = a;
                sc[J].j = J;
            }
            qsort(sc, (size_t)nb, sizeof(scored_block), by_score_desc_then_j);
            for (int t = 0; t < kk; ++t) kept[t] = sc[t].j;
            qsort(kept, (size_t)kk, sizeof(int32_t), by_int_asc);
            const int64_t r = (int64_t)bh * nb + I;
            memcpy(col_idx + r * kk, kept, sizeof(int32_t) * kk);
        }
        free(qm);
        free(km);
        free(sc);
        free(kept);
    }
    return kk;
}

/*
 * The dynamic gate and branch dropping (SALAD technical summary, section 2.2
 * ITADS: a lightweight module maps the denoising timestep and the hidden state
 * to a global factor squashed by a sigmoid into (0, 1); section 2.3: at
 * inference the linear branch is dropped where that factor is very low).  The
 * pages give neither the module nor the threshold; the reading taken: per
 * (b, h), with the layer's queries as the hidden state,
 *   pooled[f] = (1/N) sum_n q[b][n][h][f]
 *   s         = sigmoid(sum_e w_t[h][e] t_emb[b][e] + sum_f w_x[h][f] pooled[f] + beta[h])
 *   gate      = 0 where s < threshold (the branch is dropped), s otherwise.
 * In fp64; writes s (before dropping) and the gate, both [B][Hh].
 */
void oracle_gate(const uint16_t *q, int B, int N, int Hh, int d, const double *t_emb, int E,
                 const double *w_t, const double *w_x, const double *beta, double threshold,
                 double *s_out, double *gate_out) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hh; ++h) {
            double logit = beta[h];
            for (int e = 0; e < E; ++e) logit += w_t[(size_t)h * E + e] * t_emb[(size_t)b * E + e];
            for (int f = 0; f < d; ++f) {
                double sum = 0.0;
                for (int n = 0; n < N; ++n) sum += bf16_to_double(q[(((size_t)b * N + n) * Hh + h) * d + f]);
                logit += w_x[(size_t)h * d + f] * (sum / N);
            }
            const double sv = 1.0 / (1.0 + exp(-logit));
            s_out[b * Hh + h] = sv;
            gate_out[b * Hh + h] = sv < threshold ? 0.0 : sv;
        }
    }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
