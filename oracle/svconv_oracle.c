/*
 * CPU oracle for SparseConv2D on frame-wise pruned ViT tokens.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header, table or constant with the CUDA library.
 *
 * Plain, single-threaded, obviously-correct restatements of the definitions on
 * the SV-TAD page (papernotes.org, "SV-TAD: Native Sparse Convolutions for
 * Efficient Temporal Action Detection"):
 *   - Key Design 1 ("Static Neighbor Index Table"): the lookup map M (H x W per
 *     frame, filled with -1, then M[y_k, x_k] = k) and the neighbour table
 *     N[k, j] = M[y_k + dy_j, x_k + dx_j], or -1 if pruned or out of bounds.
 *   - Key Design 2 ("Native Sparse 2D Convolution Kernels"), the convolution
 *     equation y_k = sum_j W_j x[N[k, j]] with N = -1 read as zero padding.
 *   - The backward pass is named on that page but not written out; it is the
 *     adjoint of the forward, written here in SCATTER form (every forward term
 *     W_j x[N[k,j]] sends W_j^T dy_k back to token N[k,j]), which is independent
 *     of the mirrored-offset gather the GPU uses.
 *   - The bottleneck adapter ("lightweight bottleneck adapters", Overall
 *     Architecture and Key Design 3 "down-projected"): Linear D->R, SparseConv2D
 *     R->R, GELU (erf form), Linear R->D, residual add; bf16 storage between the
 *     stages.
 *
 * Readings taken where the page is silent (listed in the design notes too):
 *   - taps j = 0..8 are row-major over (dy, dx) in {-1,0,1}^2: j = (dy+1)*3+(dx+1),
 *     so j = 4 is the token itself and 8-j is the point reflection of j;
 *   - cross-correlation (W_j multiplies the neighbour at +delta_j), as torch conv2d;
 *   - an optional bias b is added to every output row;
 *   - N holds GLOBAL packed row indices, so one table serves all frames;
 *   - neighbours never cross frames (the convolution is spatial, per frame).
 *
 * All floating point is double.  bf16 rounding (adapter only) is round to
 * nearest even onto an 8-bit significand.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Status bits reported by orc_build_index (same meaning as the library's). */
#define ORC_BAD_COORD 1     /* y or x outside the frame */
#define ORC_DUPLICATE 2     /* two tokens at the same (t, y, x) */
#define ORC_BAD_FRAME 4     /* coords[k].t disagrees with the frame segment holding k */
#define ORC_BAD_OFFSETS 8   /* frame_off not 0 .. n and non-decreasing */

/* Tap j -> spatial offset. */
static int tap_dy(int j) { return j / 3 - 1; }
static int tap_dx(int j) { return j % 3 - 1; }

/* Key Design 1, step 1 and step 2. Returns a bitwise OR of ORC_* flags (0 = OK).
 * M (may be NULL) is [T][H][W]; nbr is [n][9]. */
int orc_build_index(const int32_t *coords, const int32_t *frame_off, int T, int H, int W, int n,
                    int32_t *nbr, int32_t *M)
{
    int status = 0;
    int32_t *map = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1) * H * W);
    if (!map) return -1;
    for (size_t c = 0; c < (size_t)T * H * W; ++c) map[c] = -1;
    for (int k = 0; k < n; ++k)
        for (int j = 0; j < 9; ++j) nbr[(size_t)k * 9 + j] = -1;

    int offsets_ok = (frame_off[0] == 0) && (frame_off[T] == n);
    for (int t = 0; t < T; ++t)
        if (frame_off[t + 1] < frame_off[t]) offsets_ok = 0;
    if (!offsets_ok) {
        status |= ORC_BAD_OFFSETS;
    } else {
        /* step 1: M[t][y_k][x_k] = k */
        for (int t = 0; t < T; ++t) {
            for (int k = frame_off[t]; k < frame_off[t + 1]; ++k) {
                int tt = coords[3 * k], y = coords[3 * k + 1], x = coords[3 * k + 2];
                if (tt != t) { status |= ORC_BAD_FRAME; continue; }
                if (y < 0 || y >= H || x < 0 || x >= W) { status |= ORC_BAD_COORD; continue; }
                int32_t *cell = &map[((size_t)t * H + y) * W + x];
                if (*cell != -1) status |= ORC_DUPLICATE;
                *cell = k;
            }
        }
        /* step 2: N[k][j] = M[t][y_k + dy_j][x_k + dx_j], or -1 */
        for (int t = 0; t < T; ++t) {
            for (int k = frame_off[t]; k < frame_off[t + 1]; ++k) {
                int tt = coords[3 * k], y = coords[3 * k + 1], x = coords[3 * k + 2];
                if (tt != t || y < 0 || y >= H || x < 0 || x >= W) continue;
                for (int j = 0; j < 9; ++j) {
                    int yy = y + tap_dy(j), xx = x + tap_dx(j);
                    int32_t v = -1;
                    if (yy >= 0 && yy < H && xx >= 0 && xx < W) v = map[((size_t)t * H + yy) * W + xx];
                    nbr[(size_t)k * 9 + j] = v;
                }
            }
        }
    }
    if (M) memcpy(M, map, sizeof(int32_t) * (size_t)T * H * W);
    free(map);
    return status;
}

/* Key Design 2: y_k = sum_j W_j x[N[k,j]] (+ b).  W is [Cout][9][Cin].
 * rows == NULL computes every row k into Y[k]; otherwise Y[r] = y_{rows[r]}. */
void orc_fwd(const double *X, const int32_t *nbr, int n, int Cin, int Cout, const double *Wt,
             const double *bias, const int64_t *rows, int nrows, double *Y)
{
    int count = rows ? nrows : n;
    for (int r = 0; r < count; ++r) {
        int64_t k = rows ? rows[r] : r;
        for (int o = 0; o < Cout; ++o) {
            double acc = bias ? bias[o] : 0.0;
            for (int j = 0; j < 9; ++j) {
                int32_t m = nbr[k * 9 + j];
                if (m < 0) continue; /* -1 is zero padding */
                const double *w = Wt + ((size_t)o * 9 + j) * Cin;
                const double *x = X + (size_t)m * Cin;
                for (int i = 0; i < Cin; ++i) acc += w[i] * x[i];
            }
            Y[(size_t)r * Cout + o] = acc;
        }
    }
}

/* Adjoint of orc_fwd with respect to X, scatter form:
 *   for every (k, j) with m = N[k,j] >= 0:  dX[m] += W_j^T dY[k].
 * rows == NULL produces all of dX; otherwise dX[r] is the row rows[r], found by
 * scanning N for every entry equal to rows[r] (still the scatter definition). */
void orc_bwd_data(const double *dY, const int32_t *nbr, int n, int Cin, int Cout, const double *Wt,
                  const int64_t *rows, int nrows, double *dX)
{
    if (!rows) {
        memset(dX, 0, sizeof(double) * (size_t)n * Cin);
        for (int k = 0; k < n; ++k)
            for (int j = 0; j < 9; ++j) {
                int32_t m = nbr[(size_t)k * 9 + j];
                if (m < 0) continue;
                for (int i = 0; i < Cin; ++i) {
                    double acc = 0.0;
                    for (int o = 0; o < Cout; ++o)
                        acc += Wt[((size_t)o * 9 + j) * Cin + i] * dY[(size_t)k * Cout + o];
                    dX[(size_t)m * Cin + i] += acc;
                }
            }
        return;
    }
    memset(dX, 0, sizeof(double) * (size_t)nrows * Cin);
    for (int r = 0; r < nrows; ++r) {
        int64_t target = rows[r];
        for (int k = 0; k < n; ++k)
            for (int j = 0; j < 9; ++j) {
                if (nbr[(size_t)k * 9 + j] != target) continue;
                for (int i = 0; i < Cin; ++i) {
                    double acc = 0.0;
                    for (int o = 0; o < Cout; ++o)
                        acc += Wt[((size_t)o * 9 + j) * Cin + i] * dY[(size_t)k * Cout + o];
                    dX[(size_t)r * Cin + i] += acc;
                }
            }
    }
}

/* Adjoint of orc_fwd with respect to W and b:
 *   dW[o][j][i] = sum_k dY[k][o] * x[N[k,j]][i],   db[o] = sum_k dY[k][o]. */
void orc_bwd_weight(const double *dY, const double *X, const int32_t *nbr, int n, int Cin, int Cout,
                    double *dW, double *db)
{
    memset(dW, 0, sizeof(double) * (size_t)Cout * 9 * Cin);
    if (db) memset(db, 0, sizeof(double) * (size_t)Cout);
    for (int k = 0; k < n; ++k) {
        for (int o = 0; o < Cout; ++o) {
            double g = dY[(size_t)k * Cout + o];
            if (db) db[o] += g;
            for (int j = 0; j < 9; ++j) {
                int32_t m = nbr[(size_t)k * 9 + j];
                if (m < 0) continue;
                double *w = dW + ((size_t)o * 9 + j) * Cin;
                const double *x = X + (size_t)m * Cin;
                for (int i = 0; i < Cin; ++i) w[i] += g * x[i];
            }
        }
    }
}

/* Selected entries of dW: ent is [m][3] = (o, j, i); out[e] = dW[o][j][i]. */
void orc_bwd_weight_entries(const double *dY, const double *X, const int32_t *nbr, int n, int Cin,
                            int Cout, const int32_t *ent, int m_ent, double *out)
{
    for (int e = 0; e < m_ent; ++e) {
        int o = ent[3 * e], j = ent[3 * e + 1], i = ent[3 * e + 2];
        double acc = 0.0;
        for (int k = 0; k < n; ++k) {
            int32_t m = nbr[(size_t)k * 9 + j];
            if (m < 0) continue;
            acc += dY[(size_t)k * Cout + o] * X[(size_t)m * Cin + i];
        }
        out[e] = acc;
    }
}

/* Round a double to the nearest bf16 value, ties to even (8-bit significand). */
double orc_round_bf16(double v)
{
    if (v == 0.0 || !isfinite(v)) return v;
    int e;
    double m = frexp(v, &e);          /* v = m * 2^e, 0.5 <= |m| < 1 */
    double s = ldexp(m, 8);           /* 8 significant bits -> integer part */
    double r = nearbyint(s);          /* default rounding mode: nearest, ties to even */
    return ldexp(r, e - 8);
}

static double gelu_erf(double v) { return 0.5 * v * (1.0 + erf(v / sqrt(2.0))); }

/* Bottleneck adapter on packed rows r0 .. r1-1, which must be whole frames
 * (neighbours never leave a frame).  X is [n][D] (all rows, bf16 values), nbr the
 * global table.  Out is [r1-r0][D]:
 *   H1 = bf16(X Wd^T)                       Wd [R][D]
 *   H2 = bf16(GELU(SparseConv(H1) + bc))    Wc [R][9][R], bc [R] or NULL
 *   Out = bf16(X + H2 Wu^T)                 Wu [D][R]                       */
void orc_adapter_fwd(const double *X, const int32_t *nbr, int r0, int r1, int D, int R,
                     const double *Wd, const double *Wc, const double *bc, const double *Wu,
                     double *Out)
{
    int rows = r1 - r0;
    double *H1 = (double *)malloc(sizeof(double) * (size_t)rows * R);
    double *H2 = (double *)malloc(sizeof(double) * (size_t)rows * R);
    for (int r = 0; r < rows; ++r)
        for (int q = 0; q < R; ++q) {
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += X[(size_t)(r0 + r) * D + d] * Wd[(size_t)q * D + d];
            H1[(size_t)r * R + q] = orc_round_bf16(acc);
        }
    for (int r = 0; r < rows; ++r)
        for (int o = 0; o < R; ++o) {
            double acc = bc ? bc[o] : 0.0;
            for (int j = 0; j < 9; ++j) {
                int32_t m = nbr[(size_t)(r0 + r) * 9 + j];
                if (m < 0) continue;
                const double *h = H1 + (size_t)(m - r0) * R;
                const double *w = Wc + ((size_t)o * 9 + j) * R;
                for (int i = 0; i < R; ++i) acc += w[i] * h[i];
            }
            H2[(size_t)r * R + o] = orc_round_bf16(gelu_erf(acc));
        }
    for (int r = 0; r < rows; ++r)
        for (int d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int q = 0; q < R; ++q) acc += H2[(size_t)r * R + q] * Wu[(size_t)d * R + q];
            Out[(size_t)r * D + d] = orc_round_bf16(X[(size_t)(r0 + r) * D + d] + acc);
        }
    free(H1);
    free(H2);
}

/* Dense zero-padded 3x3 cross-correlation on one [H][W][Cin] grid, written out
 * directly (no neighbour table).  Used only to pin the sparse oracle:
 * Y[y][x][o] = sum_{dy,dx,i} W[o][(dy+1)*3+(dx+1)][i] * G[y+dy][x+dx][i]. */
void orc_dense_conv(const double *G, int H, int W, int Cin, int Cout, const double *Wt,
                    const double *bias, double *Y)
{
    for (int y = 0; y < H; ++y)
        for (int x = 0; x < W; ++x)
            for (int o = 0; o < Cout; ++o) {
                double acc = bias ? bias[o] : 0.0;
                for (int dy = -1; dy <= 1; ++dy)
                    for (int dx = -1; dx <= 1; ++dx) {
                        int yy = y + dy, xx = x + dx;
                        if (yy < 0 || yy >= H || xx < 0 || xx >= W) continue;
                        const double *w = Wt + ((size_t)o * 9 + (dy + 1) * 3 + (dx + 1)) * Cin;
                        const double *g = G + ((size_t)yy * W + xx) * Cin;
                        for (int i = 0; i < Cin; ++i) acc += w[i] * g[i];
                    }
                Y[((size_t)y * W + x) * Cout + o] = acc;
            }
}

/* Bias gradient alone: db[o] = sum_k dY[k][o]. */
void orc_bwd_bias(const double *dY, int n, int Cout, double *db)
{
    for (int o = 0; o < Cout; ++o) db[o] = 0.0;
    for (int k = 0; k < n; ++k)
        for (int o = 0; o < Cout; ++o) db[o] += dY[(size_t)k * Cout + o];
}

/* Asymmetric cross-attention of auxiliary tokens over the sparse tokens (SV-TAD page, Key
 * Design 3, "Asymmetric Cross-Attention for Temporal Recombination"): the auxiliary tokens
 * (e.g. a CLS token) are the queries, the down-projected sparse visual features are the keys
 * and the values, and only the auxiliary tokens are updated.
 * Readings where the page gives only the name: scaled dot-product attention with softmax,
 * no extra projections (the page names the down-projected features themselves as keys and
 * values), the R channels split into `heads` heads of R / heads channels each scaled by
 * 1 / sqrt(R / heads), and the result added to the auxiliary token (residual).  Group g
 * (a video) owns sparse rows goff[g] .. goff[g+1]-1 and auxiliary tokens g*A .. g*A+A-1;
 * a group without rows leaves its auxiliary tokens unchanged.
 *   Hf [n][R], goff [G+1], aux [G][A][R], out [G][A][R]. */
void orc_xattn_aux(const double *Hf, const int32_t *goff, int G, int R, int heads, const double *aux, int A,
                   double *out)
{
    const int d = R / heads;
    const double scale = 1.0 / sqrt((double)d);
    for (int g = 0; g < G; ++g) {
        const int r0 = goff[g], r1 = goff[g + 1];
        for (int a = 0; a < A; ++a) {
            const double *q = aux + ((size_t)g * A + a) * R;
            double *o = out + ((size_t)g * A + a) * R;
            for (int c = 0; c < R; ++c) o[c] = q[c];
            if (r1 <= r0) continue;
            for (int h = 0; h < heads; ++h) {
                const int c0 = h * d;
                /* softmax over the group's rows of the scaled scores, shifted by their maximum */
                double m = -INFINITY;
                for (int r = r0; r < r1; ++r) {
                    double s = 0.0;
                    for (int c = 0; c < d; ++c) s += q[c0 + c] * Hf[(size_t)r * R + c0 + c];
                    s *= scale;
                    if (s > m) m = s;
                }
                double den = 0.0;
                for (int c = 0; c < d; ++c) o[c0 + c] = 0.0;
                for (int r = r0; r < r1; ++r) {
                    double s = 0.0;
                    for (int c = 0; c < d; ++c) s += q[c0 + c] * Hf[(size_t)r * R + c0 + c];
                    const double p = exp(s * scale - m);
                    den += p;
                    for (int c = 0; c < d; ++c) o[c0 + c] += p * Hf[(size_t)r * R + c0 + c];
                }
                for (int c = 0; c < d; ++c) o[c0 + c] = q[c0 + c] + o[c0 + c] / den;
            }
        }
    }
}

/* The adapter's down-projection on its own: H1 = bf16(X Wd^T) for rows 0 .. n-1, the
 * same first stage as orc_adapter_fwd (the features the auxiliary tokens attend over).
 *   X [n][D], Wd [R][D], H1 [n][R]. */
void orc_down_proj(const double *X, int n, int D, int R, const double *Wd, double *H1)
{
    for (int r = 0; r < n; ++r)
        for (int q = 0; q < R; ++q) {
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += X[(size_t)r * D + d] * Wd[(size_t)q * D + d];
            H1[(size_t)r * R + q] = orc_round_bf16(acc);
        }
}
