/*
 * ss2d_oracle.c -- CPU oracle for the SS2D forward core.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py may load this library.  The CUDA library in
 * selective_scan_02_b200/ shares no code, header, table or helper with it.
 *
 * Plain, sequential restatement of what the SS2D core computes, written from
 * these sources:
 *   [VM]  "Deep dive into the SS2D module of VMamba, from theory to code"
 *         section 2.2 (A_log), 3.1 (cross scan), 3.2 (projections and the
 *         selective_scan call), 3.3 (cross merge), 4 (direction table).
 *   [DA]  DAMamba article, section 2.1: discrete SSM h_t = A h_{t-1} + B x_t,
 *         y_t = C h_t + D x_t.
 *   [VS]  VSSD article, section 2.1 (continuous SSM x' = Ax + Bu, y = Cx + Du).
 *   and the scan definition of the hot path: delta = softplus(dt + dt_bias),
 *   dA = exp(delta * A) with A = -exp(A_log), h_l = dA h_{l-1} + delta B_l u_l,
 *   y_l = C_l . h_l + D u_l.
 *
 * Readings where the pages are silent:
 *   - the state starts at zero (h_{-1} = 0) unless an explicit h0 is passed;
 *   - softplus(z) = log(1 + e^z), evaluated as max(z,0) + log1p(exp(-|z|));
 *   - channel c = k*D + d uses B/C group c / (C/G) (k outer, as in
 *     xs.view(B, -1, L) of [VM] 3.2);
 *   - the merge adds the four terms left to right in the order the page's
 *     expression lists them: y0 + flip(y2) + untranspose(y1) + untranspose(flip(y3)).
 *
 * All arrays are dense row-major, of element type `real`: fp64 (the parity
 * oracle, liboracle.so) unless the file is compiled with -DORACLE_REAL=float
 * (liboracle_f32.so, used only to time an fp32 CPU baseline).  <tgmath.h> makes
 * exp/log1p/fabs follow that type.  No function keeps state.
 */
#include <stdlib.h>
#include <string.h>
#include <tgmath.h>

#ifndef ORACLE_REAL
#define ORACLE_REAL double
#endif
typedef ORACLE_REAL real;

#define IDX4(a, b, c, d, nb, nc, nd) ((((size_t)(a) * (nb) + (b)) * (nc) + (c)) * (nd) + (d))

static real softplus_r(real z)
{
    /* log(1 + e^z); the two branches are the same function written so that
       exp() never overflows. */
    return z > 0 ? z + log1p(exp(-z)) : log1p(exp(z));
}

/* [VM] 3.1: x_hwwh = stack([x.view(B,-1,L), transpose(x,2,3).view(B,-1,L)]),
 *           xs = cat([x_hwwh, flip(x_hwwh, -1)], dim=1)       -> (B, 4, D, L)
 * x is (B, D, H, W). */
void oracle_cross_scan(const real *x, real *xs, int B, int D, int H, int W)
{
    const int L = H * W;
    for (int b = 0; b < B; ++b)
        for (int d = 0; d < D; ++d) {
            const real *plane = x + ((size_t)b * D + d) * L;
            real *s0 = xs + IDX4(b, 0, d, 0, 4, D, L);
            real *s1 = xs + IDX4(b, 1, d, 0, 4, D, L);
            real *s2 = xs + IDX4(b, 2, d, 0, 4, D, L);
            real *s3 = xs + IDX4(b, 3, d, 0, 4, D, L);
            /* direction 0: row-major flatten (the view) */
            for (int l = 0; l < L; ++l)
                s0[l] = plane[l];
            /* direction 1: the transposed (W, H) plane flattened row-major,
               so element (w, h) lands at w*H + h */
            for (int w = 0; w < W; ++w)
                for (int h = 0; h < H; ++h)
                    s1[(size_t)w * H + h] = plane[(size_t)h * W + w];
            /* directions 2 and 3: flip of 0 and 1 along the sequence */
            for (int l = 0; l < L; ++l) {
                s2[l] = s0[L - 1 - l];
                s3[l] = s1[L - 1 - l];
            }
        }
}

/* [VM] 3.3: inv_y = flip(out_y[:, 2:4], -1)
 *           wh_y = transpose(out_y[:, 1].view(B,-1,W,H), 2, 3).view(B,-1,L)
 *           invwh_y = transpose(inv_y[:, 1].view(B,-1,W,H), 2, 3).view(B,-1,L)
 *           y = out_y[:, 0] + inv_y[:, 0] + wh_y + invwh_y
 * out_y is (B, 4, D, L); y is (B, D, L) = (B, D, H, W). */
void oracle_cross_merge(const real *out_y, real *y, int B, int D, int H, int W)
{
    const int L = H * W;
    real *inv0 = (real *)malloc(sizeof(real) * (size_t)L);
    real *inv1 = (real *)malloc(sizeof(real) * (size_t)L);
    for (int b = 0; b < B; ++b)
        for (int d = 0; d < D; ++d) {
            const real *y0 = out_y + IDX4(b, 0, d, 0, 4, D, L);
            const real *y1 = out_y + IDX4(b, 1, d, 0, 4, D, L);
            const real *y2 = out_y + IDX4(b, 2, d, 0, 4, D, L);
            const real *y3 = out_y + IDX4(b, 3, d, 0, 4, D, L);
            for (int l = 0; l < L; ++l) {
                inv0[l] = y2[L - 1 - l];
                inv1[l] = y3[L - 1 - l];
            }
            real *dst = y + ((size_t)b * D + d) * L;
            for (int h = 0; h < H; ++h)
                for (int w = 0; w < W; ++w) {
                    /* the (W, H) view's element (w, h) sits at w*H + h; after
                       the transpose it is element (h, w) of the (H, W) plane */
                    const real wh = y1[(size_t)w * H + h];
                    const real invwh = inv1[(size_t)w * H + h];
                    const size_t p = (size_t)h * W + w;
                    dst[p] = y0[p] + inv0[p] + wh + invwh;
                }
        }
    free(inv0);
    free(inv1);
}

/* [VM] 3.2: x_dbl = einsum("b k d l, k c d -> b k c l", xs, x_proj_weight)
 * xs (B,4,D,L), weight (4,Cp,D), x_dbl (B,4,Cp,L). */
void oracle_x_proj(const real *xs, const real *weight, real *x_dbl, int B, int D, int L, int Cp)
{
    for (int b = 0; b < B; ++b)
        for (int k = 0; k < 4; ++k)
            for (int c = 0; c < Cp; ++c) {
                real *dst = x_dbl + IDX4(b, k, c, 0, 4, Cp, L);
                for (int l = 0; l < L; ++l)
                    dst[l] = 0.0;
                for (int d = 0; d < D; ++d) {
                    const real wv = weight[((size_t)k * Cp + c) * D + d];
                    const real *src = xs + IDX4(b, k, d, 0, 4, D, L);
                    for (int l = 0; l < L; ++l)
                        dst[l] += wv * src[l];
                }
            }
}

/* [VM] 3.2: dts, Bs, Cs = split(x_dbl, [R, N, N], dim=2)
 *           dts = einsum("b k r l, k d r -> b k d l", dts, dt_projs_weight)
 * x_dbl (B,4,R+2N,L) supplies the first R rows; weight (4,D,R); out (B,4,D,L). */
void oracle_dt_proj(const real *x_dbl, const real *weight, real *dts, int B, int D, int L, int R, int N)
{
    const int Cp = R + 2 * N;
    for (int b = 0; b < B; ++b)
        for (int k = 0; k < 4; ++k)
            for (int d = 0; d < D; ++d) {
                real *dst = dts + IDX4(b, k, d, 0, 4, D, L);
                for (int l = 0; l < L; ++l) {
                    real acc = 0.0;
                    for (int r = 0; r < R; ++r)
                        acc += weight[((size_t)k * D + d) * R + r] * x_dbl[IDX4(b, k, r, l, 4, Cp, L)];
                    dst[l] = acc;
                }
            }
}

/* The selective scan over (B, C, L) with G groups of B/C:
 *   delta = softplus(dt + delta_bias)       (or dt + delta_bias when softplus_on == 0)
 *   A     = -exp(A_log)                      ([VM] 2.2 keeps A in log space)
 *   h_l   = exp(delta A) h_{l-1} + delta B_l u_l      ([DA] 2.1 with the
 *                                                       zero-order-hold dA)
 *   y_l   = sum_n C_l[n] h_l[n] + D u_l
 * u, delta (B,C,L); A_log (C,N); Bm, Cm (B,G,N,L); Dv (C) or NULL;
 * delta_bias (C) or NULL; y (B,C,L).
 * h0 (B,C,N) or NULL: initial state (NULL means zero).
 * h_last (B,C,N) or NULL: receives the state after the last step.
 * every > 0, ckpt (B,C,ceil(L/every),N): receives the state before every
 * every-th step, ckpt[b,c,j] = h_{j*every-1} (the initial state for j = 0). */
static void selective_scan_impl(const real *u, const real *delta, const real *A_log,
                                const real *Bm, const real *Cm, const real *Dv,
                                const real *delta_bias, int softplus_on, real *y,
                                int B, int C, int G, int N, int L,
                                const real *h0, real *h_last, int every, real *ckpt)
{
    const int per_group = C / G;
    real *h = (real *)malloc(sizeof(real) * (size_t)N);
    real *A = (real *)malloc(sizeof(real) * (size_t)N);
    for (int b = 0; b < B; ++b)
        for (int c = 0; c < C; ++c) {
            const int g = c / per_group;
            for (int n = 0; n < N; ++n) {
                A[n] = -exp(A_log[(size_t)c * N + n]);
                h[n] = h0 ? h0[((size_t)b * C + c) * N + n] : 0.0;
            }
            const real dskip = Dv ? Dv[c] : 0.0;
            const real bias = delta_bias ? delta_bias[c] : 0.0;
            const real *uc = u + ((size_t)b * C + c) * L;
            const real *dc = delta + ((size_t)b * C + c) * L;
            real *yc = y + ((size_t)b * C + c) * L;
            for (int l = 0; l < L; ++l) {
                if (ckpt && l % every == 0)
                    for (int n = 0; n < N; ++n)
                        ckpt[(((size_t)b * C + c) * ((L + every - 1) / every) + l / every) * N + n] = h[n];
                real dt = dc[l] + bias;
                if (softplus_on)
                    dt = softplus_r(dt);
                real acc = 0.0;
                for (int n = 0; n < N; ++n) {
                    const real Bv = Bm[IDX4(b, g, n, l, G, N, L)];
                    const real Cv = Cm[IDX4(b, g, n, l, G, N, L)];
                    h[n] = exp(dt * A[n]) * h[n] + dt * Bv * uc[l];
                    acc += Cv * h[n];
                }
                yc[l] = acc + dskip * uc[l];
            }
            if (h_last)
                for (int n = 0; n < N; ++n)
                    h_last[((size_t)b * C + c) * N + n] = h[n];
        }
    free(h);
    free(A);
}

void oracle_selective_scan(const real *u, const real *delta, const real *A_log,
                           const real *Bm, const real *Cm, const real *Dv,
                           const real *delta_bias, int softplus_on, real *y,
                           int B, int C, int G, int N, int L,
                           const real *h0, real *h_last)
{
    selective_scan_impl(u, delta, A_log, Bm, Cm, Dv, delta_bias, softplus_on, y, B, C, G, N, L, h0, h_last, 0,
                        NULL);
}

/* oracle_selective_scan from a zero state that also records the state before
 * every every-th step (see selective_scan_impl). */
void oracle_selective_scan_ckpt(const real *u, const real *delta, const real *A_log,
                                const real *Bm, const real *Cm, const real *Dv,
                                const real *delta_bias, int softplus_on, real *y,
                                int B, int C, int G, int N, int L, int every, real *ckpt)
{
    selective_scan_impl(u, delta, A_log, Bm, Cm, Dv, delta_bias, softplus_on, y, B, C, G, N, L, NULL, NULL,
                        every, ckpt);
}

/* forward_corev0 of [VM] section 3, channel-first input:
 *   xs = cross_scan(x)
 *   if the projection weights are given:
 *       x_dbl = x_proj(xs); dts, Bs, Cs = split; dts = dt_proj(dts)
 *   out_y = selective_scan(xs.view(B,-1,L), dts.view(B,-1,L), -exp(A_logs),
 *                          Bs, Cs, Ds, delta_bias=dt_bias, delta_softplus)
 *   y = cross_merge(out_y)                                   -> (B, D, H, W)
 * dts (B,4,D,L), Bs/Cs (B,4,N,L) are used when x_proj_weight is NULL.
 * x_proj_weight (4,R+2N,D), dt_projs_weight (4,D,R). */
void oracle_forward_core(const real *x, const real *dts, const real *A_logs,
                         const real *Bs, const real *Cs, const real *Ds,
                         const real *dt_bias, int softplus_on,
                         const real *x_proj_weight, const real *dt_projs_weight,
                         real *y, int B, int D, int H, int W, int N, int R)
{
    const int L = H * W;
    const size_t n_xs = (size_t)B * 4 * D * L;
    real *xs = (real *)malloc(sizeof(real) * n_xs);
    real *out_y = (real *)malloc(sizeof(real) * n_xs);
    real *dts_own = NULL, *Bs_own = NULL, *Cs_own = NULL, *x_dbl = NULL;
    oracle_cross_scan(x, xs, B, D, H, W);
    if (x_proj_weight) {
        const int Cp = R + 2 * N;
        x_dbl = (real *)malloc(sizeof(real) * (size_t)B * 4 * Cp * L);
        oracle_x_proj(xs, x_proj_weight, x_dbl, B, D, L, Cp);
        dts_own = (real *)malloc(sizeof(real) * n_xs);
        oracle_dt_proj(x_dbl, dt_projs_weight, dts_own, B, D, L, R, N);
        Bs_own = (real *)malloc(sizeof(real) * (size_t)B * 4 * N * L);
        Cs_own = (real *)malloc(sizeof(real) * (size_t)B * 4 * N * L);
        for (int b = 0; b < B; ++b)
            for (int k = 0; k < 4; ++k)
                for (int n = 0; n < N; ++n) {
                    memcpy(Bs_own + IDX4(b, k, n, 0, 4, N, L), x_dbl + IDX4(b, k, R + n, 0, 4, Cp, L), sizeof(real) * L);
                    memcpy(Cs_own + IDX4(b, k, n, 0, 4, N, L), x_dbl + IDX4(b, k, R + N + n, 0, 4, Cp, L), sizeof(real) * L);
                }
        dts = dts_own;
        Bs = Bs_own;
        Cs = Cs_own;
    }
    oracle_selective_scan(xs, dts, A_logs, Bs, Cs, Ds, dt_bias, softplus_on, out_y,
                          B, 4 * D, 4, N, L, NULL, NULL);
    oracle_cross_merge(out_y, y, B, D, H, W);
    free(xs);
    free(out_y);
    free(dts_own);
    free(Bs_own);
    free(Cs_own);
    free(x_dbl);
}

/* Reverse-mode derivative of oracle_selective_scan (zero initial state) for a loss
 * whose gradient with respect to y is dy, by the chain rule applied to the
 * recurrence of [DA] 2.1 with the discretisation of [VM] 3.2.  With
 * z_l = delta_l + bias, dt_l = softplus(z_l) (or z_l), dA_l[n] = exp(dt_l A[n]) and the
 * forward states h_l[n] (h_{-1} = 0), the adjoint g_l[n] = dLoss/dh_l[n] obeys
 *     g_{L-1} = C_{L-1} dy_{L-1},   g_l = C_l dy_l + dA_{l+1} g_{l+1},
 * and the gradients are
 *     du_l      = D dy_l + dt_l sum_n g_l[n] B_l[n]
 *     ddt_l     = sum_n g_l[n] (B_l[n] u_l + A[n] dA_l[n] h_{l-1}[n])
 *     ddelta_l  = ddt_l * sigmoid(z_l) with softplus, else ddt_l
 *     dA[n]     = sum_l g_l[n] dt_l dA_l[n] h_{l-1}[n],   dA_log[n] = dA[n] * A[n]
 *     dB_l[n]   = sum over the group's channels of g_l[n] dt_l u_l
 *     dC_l[n]   = sum over the group's channels of dy_l h_l[n]
 *     dD        = sum_l dy_l u_l,   dbias = sum_l ddelta_l
 * Shapes as oracle_selective_scan; dy, du, ddelta (B,C,L); dA_log (C,N); dBm, dCm
 * (B,G,N,L); dDv, ddelta_bias (C).  Parameter gradients are summed over the batch.
 * Every output is overwritten. */
void oracle_selective_scan_bwd(const real *u, const real *delta, const real *A_log,
                               const real *Bm, const real *Cm, const real *Dv,
                               const real *delta_bias, int softplus_on, const real *dy,
                               real *du, real *ddelta, real *dA_log, real *dBm, real *dCm,
                               real *dDv, real *ddelta_bias, int B, int C, int G, int N, int L)
{
    const int per_group = C / G;
    real *A = (real *)malloc(sizeof(real) * (size_t)N);
    real *g = (real *)malloc(sizeof(real) * (size_t)N);
    real *dAacc = (real *)malloc(sizeof(real) * (size_t)N);
    real *hs = (real *)malloc(sizeof(real) * (size_t)(L + 1) * N); /* hs[(l+1)*N + n] = h_l[n] */
    real *dts = (real *)malloc(sizeof(real) * (size_t)L);
    memset(dA_log, 0, sizeof(real) * (size_t)C * N);
    memset(dBm, 0, sizeof(real) * (size_t)B * G * N * L);
    memset(dCm, 0, sizeof(real) * (size_t)B * G * N * L);
    memset(dDv, 0, sizeof(real) * (size_t)C);
    memset(ddelta_bias, 0, sizeof(real) * (size_t)C);
    for (int b = 0; b < B; ++b)
        for (int c = 0; c < C; ++c) {
            const int grp = c / per_group;
            const real dskip = Dv ? Dv[c] : 0.0;
            const real bias = delta_bias ? delta_bias[c] : 0.0;
            const real *uc = u + ((size_t)b * C + c) * L;
            const real *dc = delta + ((size_t)b * C + c) * L;
            const real *dyc = dy + ((size_t)b * C + c) * L;
            real *duc = du + ((size_t)b * C + c) * L;
            real *ddc = ddelta + ((size_t)b * C + c) * L;
            for (int n = 0; n < N; ++n) {
                A[n] = -exp(A_log[(size_t)c * N + n]);
                hs[n] = 0.0;
                g[n] = 0.0;
                dAacc[n] = 0.0;
            }
            /* forward: every state of the sequence */
            for (int l = 0; l < L; ++l) {
                const real z = dc[l] + bias;
                dts[l] = softplus_on ? softplus_r(z) : z;
                for (int n = 0; n < N; ++n) {
                    const real Bv = Bm[IDX4(b, grp, n, l, G, N, L)];
                    hs[(size_t)(l + 1) * N + n] = exp(dts[l] * A[n]) * hs[(size_t)l * N + n] + dts[l] * Bv * uc[l];
                }
            }
            /* backward: l = L-1 .. 0; g holds dA_{l+1} g_{l+1} on entry */
            for (int l = L - 1; l >= 0; --l) {
                const real dt = dts[l];
                real su = 0.0, sdt = 0.0;
                for (int n = 0; n < N; ++n) {
                    const real Bv = Bm[IDX4(b, grp, n, l, G, N, L)];
                    const real Cv = Cm[IDX4(b, grp, n, l, G, N, L)];
                    const real hprev = hs[(size_t)l * N + n];
                    const real hcur = hs[(size_t)(l + 1) * N + n];
                    const real dA = exp(dt * A[n]);
                    const real gl = Cv * dyc[l] + g[n];
                    dCm[IDX4(b, grp, n, l, G, N, L)] += dyc[l] * hcur;
                    dBm[IDX4(b, grp, n, l, G, N, L)] += gl * dt * uc[l];
                    su += gl * Bv;
                    sdt += gl * (Bv * uc[l] + A[n] * dA * hprev);
                    dAacc[n] += gl * dt * dA * hprev;
                    g[n] = dA * gl; /* becomes dA_l g_l for step l-1 */
                }
                duc[l] = dskip * dyc[l] + dt * su;
                const real z = dc[l] + bias;
                real sig = 1.0;
                if (softplus_on)
                    sig = z >= 0.0 ? 1.0 / (1.0 + exp(-z)) : exp(z) / (1.0 + exp(z));
                ddc[l] = sdt * sig;
                ddelta_bias[c] += ddc[l];
                dDv[c] += dyc[l] * uc[l];
            }
            for (int n = 0; n < N; ++n)
                dA_log[(size_t)c * N + n] += dAacc[n] * A[n];
        }
    free(A);
    free(g);
    free(dAacc);
    free(hs);
    free(dts);
}

/* Reverse-mode derivative of oracle_forward_core, dts/Bs/Cs form.  CrossMerge's
 * adjoint is CrossScan (the gradient of out_y is cross_scan(dy)) and CrossScan's
 * adjoint is CrossMerge (dx = cross_merge(dxs)); the scan in between is
 * oracle_selective_scan_bwd with 4D channels in 4 groups.
 * dy, dx (B,D,H,W); ddts (B,4,D,L); dA_logs (4D,N); dBs, dCs (B,4,N,L);
 * dDs, ddt_bias (4D).  Every output is overwritten. */
void oracle_forward_core_bwd(const real *x, const real *dts, const real *A_logs,
                             const real *Bs, const real *Cs, const real *Ds,
                             const real *dt_bias, int softplus_on, const real *dy,
                             real *dx, real *ddts, real *dA_logs, real *dBs, real *dCs,
                             real *dDs, real *ddt_bias, int B, int D, int H, int W, int N)
{
    const int L = H * W;
    const size_t n_xs = (size_t)B * 4 * D * L;
    real *xs = (real *)malloc(sizeof(real) * n_xs);
    real *dys = (real *)malloc(sizeof(real) * n_xs);
    real *dxs = (real *)malloc(sizeof(real) * n_xs);
    oracle_cross_scan(x, xs, B, D, H, W);
    oracle_cross_scan(dy, dys, B, D, H, W);
    oracle_selective_scan_bwd(xs, dts, A_logs, Bs, Cs, Ds, dt_bias, softplus_on, dys,
                              dxs, ddts, dA_logs, dBs, dCs, dDs, ddt_bias, B, 4 * D, 4, N, L);
    oracle_cross_merge(dxs, dx, B, D, H, W);
    free(xs);
    free(dys);
    free(dxs);
}
