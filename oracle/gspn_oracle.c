/*
 * gspn_oracle.c -- float64, single-threaded CPU reference of the GSPN 4-direction
 * line-scan propagation (forward and backward).
 *
 * TEST INFRASTRUCTURE ONLY. This file is the oracle that the CUDA library is checked
 * against. Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
 * legs may load it. It shares no code, header or table with the CUDA library.
 *
 * What it computes (citations are page title + section):
 *  - "GSPN-2: Efficient Parallel Sequence Modeling" (paper notes), section
 *    "2D spatial propagation review": the map is propagated line by line; the
 *    per-line propagation matrix w_{i,c} is W x W, tridiagonal and row-stochastic
 *    (rows sum to 1), lambda_{i,:,c} is a per-channel scaling of the input, and the
 *    scan is run in four directions (top->bottom, bottom->top, left->right,
 *    right->left).
 *  - "Parallel Sequence Modeling via Generalized Spatial Propagation Network"
 *    (summary), section "Approach": the weights are made row-stochastic by a sigmoid
 *    followed by a row normalisation over the three neighbours j-1, j, j+1.
 *  - "GSPN-2 ..." (paper notes), section "Optimisation 2: compact channel
 *    propagation": in the channel-shared mode one matrix w_i is used by every channel
 *    and only lambda stays per channel.
 *  The display equation that followed "GSPN propagates row by row" was lost in the
 *  page extraction. The rule implemented here is the plainest reading consistent with
 *  the surviving text:
 *      h_{-1} = 0,   h_i = w_i h_{i-1} + lambda_i (.) x_i,
 *      y = u (.) sum_{d in mask} h^d          (h^d mapped back to image coordinates).
 *  Edge rows of w have two in-range neighbours; the normalisation runs over the
 *  in-range neighbours only, so every row sums to exactly one.
 *
 * Conventions (shared with the CUDA library by specification, not by code):
 *  - x, lam, u, y, dy, dx, dlam, du: N x C x H x W, contiguous.
 *  - a, da: D x N x Cw x 3 x H x W, D = popcount(mask), slots in the order TB, BT, LR,
 *    RL keeping the directions set in mask; Cw = C (per-channel) or 1 (shared).
 *  - Scan coordinates: step i along the scan axis, lane j across it.
 *      TB: r = i,       c = j      (L = H, M = W)
 *      BT: r = H-1-i,   c = j      (L = H, M = W)
 *      LR: r = j,       c = i      (L = W, M = H)
 *      RL: r = j,       c = W-1-i  (L = W, M = H)
 *  - Neighbour k in {0,1,2} is lane j+k-1, i.e. ordered by increasing image coordinate
 *    on the axis across the scan. The 3 logits of hidden pixel (r,c) are stored at
 *    image position (r,c).
 *
 * Local (chunked) propagation. The pages contrast local and global GSPN ("Parallel
 * Sequence Modeling via Generalized Spatial Propagation Network" summary, section
 * "Measured effects": a hybrid of local and global layers beats all-local ones) and give
 * the fused kernel a chunk grid axis ("GSPN-2 ..." paper notes, "Optimisation 1"), but do
 * not spell the local rule out. Reading used here: with chunk length K > 0 the image is cut
 * along each direction's scan axis into chunks of K lines aligned to line 0 (rows for
 * TB/BT, columns for LR/RL) and propagation does not cross a chunk boundary: the scan
 * restarts from h = 0 at the first line of every chunk in scan order. K = 0 is the global
 * scan. The *_chunked entry points take K; the plain ones are K = 0.
 *
 * Per-direction lambda and u (the *_ex entry points with per_dir = 1): the pages' models merge
 * the four directions with a learnable merge ("Parallel Sequence Modeling via Generalized
 * Spatial Propagation Network" summary, section "Measured effects"). Reading: lambda and u carry
 * a direction axis (D x N x C x H x W, slots ordered as the logits), h^d is driven by
 * lambda_d (.) x, and y = sum_d u_d (.) h^d, i.e. a per-pixel, per-channel learnable weighting
 * of the directions. per_dir = 0 is the shared lambda / u above.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define DIR_TB 1u
#define DIR_BT 2u
#define DIR_LR 4u
#define DIR_RL 8u

/* scan length L and lane count M of direction d */
static void geom(unsigned d, int H, int W, int *L, int *M) {
    if (d == DIR_TB || d == DIR_BT) { *L = H; *M = W; }
    else                            { *L = W; *M = H; }
}

/* image offset r*W + c of scan position (i, j) in direction d */
static long pix(unsigned d, int H, int W, int i, int j) {
    int r, c;
    switch (d) {
    case DIR_TB: r = i;         c = j;         break;
    case DIR_BT: r = H - 1 - i; c = j;         break;
    case DIR_LR: r = j;         c = i;         break;
    default:     r = j;         c = W - 1 - i; break; /* RL */
    }
    return (long)r * W + c;
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* Weights of hidden lane j (of M) from its three logits a_k: sigmoid, then division by
 * the sum over in-range neighbours. Out-of-range neighbours get weight 0. Also returns
 * s_k and the normaliser S for the backward. */
static void row_weights(const double av[3], int j, int M, double w[3], double s[3], double *S) {
    double sum = 0.0;
    for (int k = 0; k < 3; ++k) {
        int jj = j + k - 1;
        if (jj >= 0 && jj < M) { s[k] = sigmoid(av[k]); sum += s[k]; }
        else                   { s[k] = 0.0; }
    }
    for (int k = 0; k < 3; ++k) w[k] = s[k] / sum;
    *S = sum;
}

/* Whether scan step i of direction d starts a chunk (h restarts from 0 there). */
static int chunk_start(unsigned d, int H, int W, int chunk, int i) {
    if (i == 0) return 1;
    if (chunk <= 0) return 0;
    int line; /* image row (TB, BT) or column (LR, RL) of step i */
    switch (d) {
    case DIR_TB: line = i;         break;
    case DIR_BT: line = H - 1 - i; break;
    case DIR_LR: line = i;         break;
    default:     line = W - 1 - i; break; /* RL */
    }
    if (d == DIR_TB || d == DIR_LR) return line % chunk == 0;  /* first line of its chunk */
    return (line + 1) % chunk == 0;                            /* last line of its chunk */
}

static int popcount4(unsigned m) { int n = 0; for (int b = 0; b < 4; ++b) n += (m >> b) & 1u; return n; }

static int check_args(int N, int C, int H, int W, int wmode, unsigned mask, int chunk) {
    if (N < 1 || C < 1 || H < 1 || W < 1 || chunk < 0) return 1;
    if (wmode != 0 && wmode != 1) return 1;
    if (mask < 1u || mask > 15u) return 1;
    return 0;
}

/* Forward scan of one (n, c, d): fills hbuf[i*M + j] (scan coordinates). */
static void scan_forward(unsigned d, int H, int W, int chunk, const double *x, const double *lam,
                         const double *a3 /* 3 planes of H*W */, double *hbuf) {
    int L, M;
    geom(d, H, W, &L, &M);
    const long HW = (long)H * W;
    for (int i = 0; i < L; ++i) {
        for (int j = 0; j < M; ++j) {
            long p = pix(d, H, W, i, j);
            double z = lam[p] * x[p];
            double acc = z;
            if (!chunk_start(d, H, W, chunk, i)) {
                double av[3] = {a3[p], a3[HW + p], a3[2 * HW + p]}, w[3], s[3], S;
                row_weights(av, j, M, w, s, &S);
                for (int k = 0; k < 3; ++k) {
                    int jj = j + k - 1;
                    if (jj >= 0 && jj < M) acc += w[k] * hbuf[(long)(i - 1) * M + jj];
                }
            }
            hbuf[(long)i * M + j] = acc;
        }
    }
}

static long logit_base(int slot, int n, int cw, int N, int Cw, long HW) {
    return (((long)slot * N + n) * Cw + cw) * 3 * HW;
}

int gspn_ref_forward_ex(int N, int C, int H, int W, int wmode, unsigned mask, int chunk, int per_dir,
                        const double *x, const double *a, const double *lam, const double *u, double *y) {
    if (check_args(N, C, H, W, wmode, mask, chunk) || (per_dir != 0 && per_dir != 1)) return 1;
    const long HW = (long)H * W;
    const long U = (long)N * C * HW; /* elements of one N x C x H x W tensor */
    const int Cw = wmode ? 1 : C;
    const int Lmax = H > W ? H : W;
    double *hbuf = (double *)malloc(sizeof(double) * (size_t)Lmax * (size_t)Lmax);
    double *acc = (double *)malloc(sizeof(double) * (size_t)HW);
    if (!hbuf || !acc) { free(hbuf); free(acc); return 2; }
    for (int n = 0; n < N; ++n) {
        for (int c = 0; c < C; ++c) {
            const long off = ((long)n * C + c) * HW;
            memset(acc, 0, sizeof(double) * (size_t)HW);
            int slot = 0;
            for (unsigned d = DIR_TB; d <= DIR_RL; d <<= 1) {
                if (!(mask & d)) continue;
                const double *a3 = a + logit_base(slot, n, wmode ? 0 : c, N, Cw, HW);
                const double *lam_d = lam + (per_dir ? slot * U : 0) + off;
                const double *u_d = u + (per_dir ? slot * U : 0) + off;
                scan_forward(d, H, W, chunk, x + off, lam_d, a3, hbuf);
                int L, M;
                geom(d, H, W, &L, &M);
                for (int i = 0; i < L; ++i)
                    for (int j = 0; j < M; ++j) {
                        const long p = pix(d, H, W, i, j);
                        /* per-direction u weights h^d here; the shared u is applied once below */
                        acc[p] += (per_dir ? u_d[p] : 1.0) * hbuf[(long)i * M + j];
                    }
                ++slot;
            }
            for (long p = 0; p < HW; ++p) y[off + p] = per_dir ? acc[p] : u[off + p] * acc[p];
        }
    }
    free(hbuf);
    free(acc);
    return 0;
}

int gspn_ref_forward_chunked(int N, int C, int H, int W, int wmode, unsigned mask, int chunk,
                             const double *x, const double *a, const double *lam, const double *u,
                             double *y) {
    return gspn_ref_forward_ex(N, C, H, W, wmode, mask, chunk, 0, x, a, lam, u, y);
}

int gspn_ref_forward(int N, int C, int H, int W, int wmode, unsigned mask,
                     const double *x, const double *a, const double *lam, const double *u,
                     double *y) {
    return gspn_ref_forward_ex(N, C, H, W, wmode, mask, 0, 0, x, a, lam, u, y);
}

/*
 * Backward (the adjoint of the forward above, written from the chain rule):
 *   acc = sum_d h^d,  du = dy (.) acc,  g = dy (.) u.
 *   Per direction, in scan coordinates: delta_{L-1} = g_{L-1},
 *     delta_i = g_i + w_{i+1}^T delta_{i+1},
 *     (w^T delta)[j] = w[j-1][2] delta[j-1] + w[j][1] delta[j] + w[j+1][0] delta[j+1]
 *     (in-range terms only).
 *   dz = sum_d delta^d (image coordinates), dx = lam (.) dz, dlam = x (.) dz.
 *   dw_i[j][k] = delta_i[j] h_{i-1}[j+k-1]  (0 on step 0, where h_{-1} = 0).
 *   w_k = s_k / S with s_k = sigmoid(a_k):
 *     da_k = s_k (1 - s_k) (dw_k - sum_{k' in range} w_k' dw_k') / S  for in-range k,
 *     da_k = 0 for out-of-range k. In the shared mode da is summed over channels.
 *   With chunks, a step that starts a chunk behaves like step 0: its weights multiply
 *   h = 0 (zero logit gradient) and no delta flows back through them.
 *   Per-direction lambda / u: g^d = dy (.) u_d, du_d = dy (.) h^d, dlam_d = x (.) delta^d,
 *   dx = sum_d lam_d (.) delta^d.
 */
int gspn_ref_backward_ex(int N, int C, int H, int W, int wmode, unsigned mask, int chunk, int per_dir,
                         const double *x, const double *a, const double *lam, const double *u,
                         const double *dy, double *dx, double *da, double *dlam, double *du) {
    if (check_args(N, C, H, W, wmode, mask, chunk) || (per_dir != 0 && per_dir != 1)) return 1;
    const long HW = (long)H * W;
    const long U = (long)N * C * HW;
    const int Cw = wmode ? 1 : C;
    const int D = popcount4(mask);
    const int Lmax = H > W ? H : W;
    double *hbuf = (double *)malloc(sizeof(double) * (size_t)Lmax * (size_t)Lmax);
    double *acc = (double *)malloc(sizeof(double) * (size_t)HW);
    double *dz = (double *)malloc(sizeof(double) * (size_t)HW);
    double *dcur = (double *)malloc(sizeof(double) * (size_t)Lmax);
    double *dnext = (double *)malloc(sizeof(double) * (size_t)Lmax);
    double *wnext = (double *)malloc(sizeof(double) * 3 * (size_t)Lmax);
    double *dd = (double *)malloc(sizeof(double) * (size_t)HW); /* delta^d, image coordinates */
    if (!hbuf || !acc || !dz || !dcur || !dnext || !wnext || !dd) {
        free(hbuf); free(acc); free(dz); free(dcur); free(dnext); free(wnext); free(dd);
        return 2;
    }
    memset(da, 0, sizeof(double) * (size_t)D * N * Cw * 3 * HW);
    for (int n = 0; n < N; ++n) {
        for (int c = 0; c < C; ++c) {
            const long off = ((long)n * C + c) * HW;
            const double *xp = x + off, *lp = lam + off, *up = u + off, *dyp = dy + off;
            /* acc = sum_d h^d, needed for du */
            memset(acc, 0, sizeof(double) * (size_t)HW);
            memset(dz, 0, sizeof(double) * (size_t)HW);
            int slot = 0;
            for (unsigned d = DIR_TB; d <= DIR_RL; d <<= 1) {
                if (!(mask & d)) continue;
                const long ab = logit_base(slot, n, wmode ? 0 : c, N, Cw, HW);
                const double *a3 = a + ab;
                double *da3 = da + ab;
                const long so = per_dir ? slot * U : 0;   /* this direction's lambda / u */
                const double *lp_d = lam + so + off, *up_d = u + so + off;
                int L, M;
                geom(d, H, W, &L, &M);
                scan_forward(d, H, W, chunk, xp, lp_d, a3, hbuf);
                for (int i = 0; i < L; ++i)
                    for (int j = 0; j < M; ++j) {
                        const long p = pix(d, H, W, i, j);
                        if (per_dir) du[so + off + p] = dyp[p] * hbuf[(long)i * M + j];
                        else acc[p] += hbuf[(long)i * M + j];
                    }
                memset(dd, 0, sizeof(double) * (size_t)HW);
                /* reverse scan */
                for (int i = L - 1; i >= 0; --i) {
                    for (int j = 0; j < M; ++j) {
                        long p = pix(d, H, W, i, j);
                        double del = dyp[p] * up_d[p];
                        if (i < L - 1) {
                            /* w_{i+1}^T delta_{i+1}: row j' of w_{i+1} touches lane j through k = j - j' + 1 */
                            for (int jp = j - 1; jp <= j + 1; ++jp) {
                                if (jp < 0 || jp >= M) continue;
                                int k = j - jp + 1;
                                del += wnext[3 * (long)jp + k] * dnext[jp];
                            }
                        }
                        dcur[j] = del;
                        dd[p] = del;
                    }
                    /* weights of step i (used by step i-1's transpose product) and da_i */
                    for (int j = 0; j < M; ++j) {
                        long p = pix(d, H, W, i, j);
                        double av[3] = {a3[p], a3[HW + p], a3[2 * HW + p]}, w[3], s[3], S;
                        row_weights(av, j, M, w, s, &S);
                        if (!chunk_start(d, H, W, chunk, i)) {
                            double dw[3] = {0.0, 0.0, 0.0}, wdw = 0.0;
                            for (int k = 0; k < 3; ++k) {
                                int jj = j + k - 1;
                                if (jj >= 0 && jj < M) {
                                    dw[k] = dcur[j] * hbuf[(long)(i - 1) * M + jj];
                                    wdw += w[k] * dw[k];
                                }
                            }
                            for (int k = 0; k < 3; ++k) {
                                int jj = j + k - 1;
                                if (jj >= 0 && jj < M)
                                    da3[k * HW + p] += s[k] * (1.0 - s[k]) * (dw[k] - wdw) / S;
                            }
                        } else {
                            /* w_0 (and a chunk's first w) multiplies h = 0: no effect on the output */
                            for (int k = 0; k < 3; ++k) w[k] = 0.0;
                        }
                        for (int k = 0; k < 3; ++k) wnext[3 * (long)j + k] = w[k];
                    }
                    for (int j = 0; j < M; ++j) dnext[j] = dcur[j];
                }
                for (long p = 0; p < HW; ++p) {
                    if (per_dir) {
                        dlam[so + off + p] = xp[p] * dd[p];
                        dz[p] += lp_d[p] * dd[p];   /* dz accumulates dx directly */
                    } else {
                        dz[p] += dd[p];
                    }
                }
                ++slot;
            }
            for (long p = 0; p < HW; ++p) {
                if (per_dir) {
                    dx[off + p] = dz[p];
                } else {
                    du[off + p] = dyp[p] * acc[p];
                    dx[off + p] = lp[p] * dz[p];
                    dlam[off + p] = xp[p] * dz[p];
                }
            }
        }
    }
    free(hbuf); free(acc); free(dz); free(dcur); free(dnext); free(wnext); free(dd);
    return 0;
}

int gspn_ref_backward_chunked(int N, int C, int H, int W, int wmode, unsigned mask, int chunk,
                              const double *x, const double *a, const double *lam, const double *u,
                              const double *dy, double *dx, double *da, double *dlam, double *du) {
    return gspn_ref_backward_ex(N, C, H, W, wmode, mask, chunk, 0, x, a, lam, u, dy, dx, da, dlam, du);
}

int gspn_ref_backward(int N, int C, int H, int W, int wmode, unsigned mask,
                      const double *x, const double *a, const double *lam, const double *u,
                      const double *dy, double *dx, double *da, double *dlam, double *du) {
    return gspn_ref_backward_ex(N, C, H, W, wmode, mask, 0, 0, x, a, lam, u, dy, dx, da, dlam, du);
}

/* Version tag so that a loader can check it got this file's build. */
int gspn_ref_abi_version(void) { return 3; }
