// api.cu -- the C ABI of libss2d: argument checks on the host, then launches.
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include "api_internal.h"
#include "kernels.h"
#include "scan.cuh"
#include "ss2d.h"
#include "xproj.h"

namespace {

thread_local char g_err[512] = "";

int fail(int status, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return status;
}

int cuda_fail(cudaError_t e, const char *what)
{
    return fail(SS2D_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool valid_dtype(int d) { return d == SS2D_F32 || d == SS2D_BF16; }
bool valid_n(int n) { return n == 1 || n == 2 || n == 4 || n == 8 || n == 16; }
size_t esize(int dtype) { return dtype == SS2D_BF16 ? 2 : 4; }

struct Span {
    const void *p;
    size_t bytes;
};

bool overlaps(Span a, Span b)
{
    if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0)
        return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
    return a0 < b0 + b.bytes && b0 < a0 + a.bytes;
}

// Largest sequence length the kernels index with 32-bit steps and the exact
// float-reciprocal division of the column-major orders.
constexpr long long kMaxL = 1LL << 24;

}  // namespace

extern "C" const char *ss2d_status_string(int status)
{
    switch (status) {
    case SS2D_OK: return "SS2D_OK";
    case SS2D_ERR_INVALID_ARG: return "SS2D_ERR_INVALID_ARG";
    case SS2D_ERR_UNSUPPORTED: return "SS2D_ERR_UNSUPPORTED";
    case SS2D_ERR_MISALIGNED: return "SS2D_ERR_MISALIGNED";
    case SS2D_ERR_WORKSPACE: return "SS2D_ERR_WORKSPACE";
    case SS2D_ERR_CUDA: return "SS2D_ERR_CUDA";
    default: return "SS2D_ERR_UNKNOWN";
    }
}

extern "C" const char *ss2d_last_error(void) { return g_err; }

extern "C" int ss2d_version(void) { return 100; }

extern "C" int ss2d_cross_scan(const void *x, int dtype, void *xs, int B, int D, int H, int W, void *stream)
{
    g_err[0] = 0;
    if (!x || !xs)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_cross_scan: x and xs must be non-null");
    if (B <= 0 || D <= 0 || H <= 0 || W <= 0)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_cross_scan: sizes must be positive (B=%d D=%d H=%d W=%d)", B, D, H, W);
    if (!valid_dtype(dtype))
        return fail(SS2D_ERR_UNSUPPORTED, "ss2d_cross_scan: dtype code %d is not SS2D_F32 or SS2D_BF16", dtype);
    if ((long long)H * W > kMaxL || (long long)B * D > 0x7fffffffLL ||
        (long long)((H + 31) / 32) * ((W + 31) / 32) > 65535)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_cross_scan: problem too large");
    if (!aligned16(x) || !aligned16(xs))
        return fail(SS2D_ERR_MISALIGNED, "ss2d_cross_scan: x and xs must be 16-byte aligned");
    const size_t n = (size_t)B * D * H * W * esize(dtype);
    if (overlaps({x, n}, {xs, 4 * n}))
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_cross_scan: xs overlaps x");
    cudaError_t e = ss2d::launch_cross_scan(x, dtype == SS2D_BF16, xs, B, D, H, W, (cudaStream_t)stream);
    return e == cudaSuccess ? SS2D_OK : cuda_fail(e, "ss2d_cross_scan launch");
}

extern "C" int ss2d_cross_merge(const float *ys, float *y, int B, int D, int H, int W, void *stream)
{
    g_err[0] = 0;
    if (!ys || !y)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_cross_merge: ys and y must be non-null");
    if (B <= 0 || D <= 0 || H <= 0 || W <= 0)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_cross_merge: sizes must be positive (B=%d D=%d H=%d W=%d)", B, D, H, W);
    if ((long long)H * W > kMaxL || (long long)B * D > 0x7fffffffLL ||
        (long long)((H + 31) / 32) * ((W + 31) / 32) > 65535)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_cross_merge: problem too large");
    if (!aligned16(ys) || !aligned16(y))
        return fail(SS2D_ERR_MISALIGNED, "ss2d_cross_merge: ys and y must be 16-byte aligned");
    const size_t n = (size_t)B * D * H * W * sizeof(float);
    if (overlaps({ys, 4 * n}, {y, n}))
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_cross_merge: y overlaps ys");
    cudaError_t e = ss2d::launch_cross_merge(ys, y, B, D, H, W, (cudaStream_t)stream);
    return e == cudaSuccess ? SS2D_OK : cuda_fail(e, "ss2d_cross_merge launch");
}

extern "C" int ss2d_selective_scan(const void *u, int u_dtype, const void *delta, int delta_dtype,
                                   const float *A_log, const float *Bm, const float *Cm, const float *Dv,
                                   const float *delta_bias, int delta_softplus, float *y, int B, int C, int G,
                                   int N, int L, void *stream)
{
    g_err[0] = 0;
    if (!u || !delta || !A_log || !Bm || !Cm || !y)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_selective_scan: u, delta, A_log, Bm, Cm and y must be non-null");
    if (B <= 0 || C <= 0 || G <= 0 || N <= 0 || L <= 0)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_selective_scan: sizes must be positive (B=%d C=%d G=%d N=%d L=%d)",
                    B, C, G, N, L);
    if (C % G != 0)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_selective_scan: C=%d is not a multiple of G=%d", C, G);
    if (!valid_dtype(u_dtype) || !valid_dtype(delta_dtype))
        return fail(SS2D_ERR_UNSUPPORTED, "ss2d_selective_scan: dtype codes (%d, %d) must be SS2D_F32 or SS2D_BF16",
                    u_dtype, delta_dtype);
    if (!valid_n(N))
        return fail(SS2D_ERR_UNSUPPORTED, "ss2d_selective_scan: N=%d is not one of 1, 2, 4, 8, 16", N);
    if ((long long)L > kMaxL || (long long)B * C > 0x7fffffffLL)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_selective_scan: problem too large");
    const void *ptrs[] = {u, delta, A_log, Bm, Cm, Dv, delta_bias, y};
    for (const void *p : ptrs)
        if (p && !aligned16(p))
            return fail(SS2D_ERR_MISALIGNED, "ss2d_selective_scan: every tensor must be 16-byte aligned");
    const size_t nY = (size_t)B * C * L * 4;
    const Span ins[] = {{u, (size_t)B * C * L * esize(u_dtype)},
                        {delta, (size_t)B * C * L * esize(delta_dtype)},
                        {A_log, (size_t)C * N * 4},
                        {Bm, (size_t)B * G * N * L * 4},
                        {Cm, (size_t)B * G * N * L * 4},
                        {Dv, Dv ? (size_t)C * 4 : 0},
                        {delta_bias, delta_bias ? (size_t)C * 4 : 0}};
    for (const Span &s : ins)
        if (overlaps(s, {y, nY}))
            return fail(SS2D_ERR_INVALID_ARG, "ss2d_selective_scan: y overlaps an input");

    ss2d::ScanArgs a{};
    a.u = u;
    a.delta = delta;
    a.A_log = A_log;
    a.Bm = Bm;
    a.Cm = Cm;
    a.gs = (long long)N * L;
    a.Dv = Dv;
    a.bias = delta_bias;
    a.y = y;
    a.B = B;
    a.C = C;
    a.G = G;
    a.L = L;
    a.per_group = C / G;
    a.W = 1;
    a.divH = {1, 1.0f};
    a.u_bf16 = u_dtype == SS2D_BF16;
    a.delta_bf16 = delta_dtype == SS2D_BF16;
    a.softplus = delta_softplus != 0;
    a.delta_bytes = (size_t)B * C * L * esize(delta_dtype);
    cudaError_t e = ss2d::launch_scan(a, N, ss2d::kStandalone, (cudaStream_t)stream);
    return e == cudaSuccess ? SS2D_OK : cuda_fail(e, "ss2d_selective_scan launch");
}

namespace {

// Checks shared by the workspace query and the call; returns SS2D_OK or a status.
int check_core(const ss2d_core_args *a)
{
    if (!a)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: args is null");
    if (a->struct_size != sizeof(ss2d_core_args))
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: struct_size %zu != %zu", a->struct_size,
                    sizeof(ss2d_core_args));
    if (a->B <= 0 || a->D <= 0 || a->H <= 0 || a->W <= 0 || a->N <= 0)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: sizes must be positive (B=%d D=%d H=%d W=%d N=%d)",
                    a->B, a->D, a->H, a->W, a->N);
    if (!a->x || !a->A_logs || !a->y)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: x, A_logs and y must be non-null");
    if (!valid_n(a->N))
        return fail(SS2D_ERR_UNSUPPORTED, "ss2d_forward_core: N=%d is not one of 1, 2, 4, 8, 16", a->N);
    if (!valid_dtype(a->x_dtype))
        return fail(SS2D_ERR_UNSUPPORTED, "ss2d_forward_core: x_dtype %d is not SS2D_F32 or SS2D_BF16", a->x_dtype);
    const long long L = (long long)a->H * a->W;
    if (L > kMaxL || (long long)a->B * 4 * a->D > 0x7fffffffLL)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: problem too large");
    const bool direct = a->dts || a->Bs || a->Cs;
    const bool proj = a->x_proj_weight || a->dt_projs_weight;
    if (direct == proj)
        return fail(SS2D_ERR_INVALID_ARG,
                    "ss2d_forward_core: give either (dts, Bs, Cs) or (x_proj_weight, dt_projs_weight)");
    if (direct) {
        if (!a->dts || !a->Bs || !a->Cs)
            return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: dts, Bs and Cs must all be set");
        if (!valid_dtype(a->dts_dtype))
            return fail(SS2D_ERR_UNSUPPORTED, "ss2d_forward_core: dts_dtype %d is not SS2D_F32 or SS2D_BF16",
                        a->dts_dtype);
    } else {
        if (!a->x_proj_weight || !a->dt_projs_weight)
            return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: x_proj_weight and dt_projs_weight must both be set");
        if (a->R <= 0)
            return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: R=%d must be positive with projections", a->R);
        if (a->x_dtype != SS2D_BF16)
            return fail(SS2D_ERR_UNSUPPORTED, "ss2d_forward_core: the projection path takes bf16 x");
        int why = ss2d::xproj_supported(a->B, a->D, a->H, a->W, a->N, a->R);
        if (why != 0)
            return fail(SS2D_ERR_UNSUPPORTED, "ss2d_forward_core: projection shape not supported (code %d)", why);
    }
    const void *ptrs[] = {a->x, a->dts, a->Bs, a->Cs, a->A_logs, a->Ds, a->dt_bias,
                          a->x_proj_weight, a->dt_projs_weight, a->y};
    for (const void *p : ptrs)
        if (p && !aligned16(p))
            return fail(SS2D_ERR_MISALIGNED, "ss2d_forward_core: every tensor must be 16-byte aligned");
    const size_t B = a->B, D = a->D, N = a->N, R = a->R;
    const Span y{a->y, B * D * L * 4};
    const Span ins[] = {{a->x, B * D * L * esize(a->x_dtype)},
                        {a->dts, a->dts ? B * 4 * D * L * esize(a->dts_dtype) : 0},
                        {a->Bs, a->Bs ? B * 4 * N * L * 4 : 0},
                        {a->Cs, a->Cs ? B * 4 * N * L * 4 : 0},
                        {a->A_logs, 4 * D * N * 4},
                        {a->Ds, a->Ds ? 4 * D * 4 : 0},
                        {a->dt_bias, a->dt_bias ? 4 * D * 4 : 0},
                        {a->x_proj_weight, a->x_proj_weight ? 4 * (R + 2 * N) * D * 2 : 0},
                        {a->dt_projs_weight, a->dt_projs_weight ? 4 * D * R * 4 : 0}};
    for (const Span &s : ins)
        if (overlaps(s, y))
            return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: y overlaps an input");
    return SS2D_OK;
}

}  // namespace

int ss2d::validate_core_args(const ss2d_core_args *a)
{
    return check_core(a);
}

int ss2d::set_last_error(int status, const char *msg)
{
    return fail(status, "%s", msg);
}

namespace {

// Segments of the direct form (long sequences with few channels run as a segmented scan).
void core_segments(const ss2d_core_args *a, int *nseg, int *seg_len)
{
    ss2d::plan_segments(a->B, 4, a->D, a->H * a->W, a->N, ss2d::kFused, a->x_dtype == SS2D_BF16,
                        a->dts_dtype == SS2D_BF16, a->delta_softplus != 0, nseg, seg_len);
}

// Bytes of the transposed copy of x the direct form reads for the column-major orders (0 if unused).
size_t core_transposed_bytes(const ss2d_core_args *a)
{
    const int L = a->H * a->W;
    if (!ss2d::scan_reads_transposed_u(a->N, ss2d::kFused, a->x_dtype == SS2D_BF16, a->dts_dtype == SS2D_BF16,
                                       a->delta_softplus != 0, L))
        return 0;
    return (size_t)a->B * a->D * L * esize(a->x_dtype);
}

// Workspace of the direct form: the segment states of a segmented scan (if any), then the
// transposed copy of x (if used).
size_t core_workspace(const ss2d_core_args *a)
{
    if (a->x_proj_weight)
        return ss2d::xproj_workspace_bytes(a->B, a->D, a->H, a->W, a->N, a->R);
    int nseg, seg_len;
    core_segments(a, &nseg, &seg_len);
    return ss2d::segment_workspace_bytes(a->B, 4 * a->D, nseg, a->N) + core_transposed_bytes(a);
}

}  // namespace

extern "C" size_t ss2d_forward_core_workspace(const ss2d_core_args *args)
{
    g_err[0] = 0;
    if (check_core(args) != SS2D_OK)
        return (size_t)-1;
    return core_workspace(args);
}

extern "C" int ss2d_forward_core(const ss2d_core_args *args, void *workspace, size_t workspace_bytes, void *stream)
{
    g_err[0] = 0;
    int st = check_core(args);
    if (st != SS2D_OK)
        return st;
    const ss2d_core_args &a = *args;
    const size_t need = core_workspace(args);
    if (need > 0) {
        if (!workspace || workspace_bytes < need)
            return fail(SS2D_ERR_WORKSPACE, "ss2d_forward_core: workspace of %zu bytes needed, %zu given", need,
                        workspace_bytes);
        if (!aligned16(workspace))
            return fail(SS2D_ERR_MISALIGNED, "ss2d_forward_core: workspace must be 16-byte aligned");
        if (overlaps({workspace, need}, {a.y, (size_t)a.B * a.D * a.H * a.W * 4}))
            return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: workspace overlaps y");
    }
    cudaStream_t s = (cudaStream_t)stream;
    const int L = a.H * a.W;
    cudaError_t e = ss2d::launch_fill_zero(a.y, (size_t)a.B * a.D * L, s);
    if (e != cudaSuccess)
        return cuda_fail(e, "ss2d_forward_core zero-fill launch");
    if (a.x_proj_weight) {
        e = ss2d::launch_core_with_projections(a.x, a.x_proj_weight, a.dt_projs_weight, a.A_logs, a.Ds, a.dt_bias,
                                               a.delta_softplus != 0, a.y, workspace, a.B, a.D, a.H, a.W, a.N, a.R,
                                               s);
        return e == cudaSuccess ? SS2D_OK : cuda_fail(e, "ss2d_forward_core (projections) launch");
    }
    ss2d::ScanArgs sa{};
    sa.u = a.x;
    sa.delta = a.dts;
    sa.A_log = a.A_logs;
    sa.Bm = a.Bs;
    sa.Cm = a.Cs;
    sa.gs = (long long)a.N * L;
    sa.Dv = a.Ds;
    sa.bias = a.dt_bias;
    sa.y = a.y;
    sa.B = a.B;
    sa.C = 4 * a.D;
    sa.G = 4;
    sa.L = L;
    sa.per_group = a.D;
    sa.W = a.W;
    sa.divH = {a.H, 1.0f / (float)a.H};
    sa.u_bf16 = a.x_dtype == SS2D_BF16;
    sa.delta_bf16 = a.dts_dtype == SS2D_BF16;
    sa.softplus = a.delta_softplus != 0;
    sa.delta_bytes = (size_t)a.B * 4 * a.D * L * esize(a.dts_dtype);
    int nseg, seg_len;
    core_segments(args, &nseg, &seg_len);
    const size_t seg_bytes = ss2d::segment_workspace_bytes(a.B, 4 * a.D, nseg, a.N);
    if (core_transposed_bytes(args) > 0) {
        void *xT = static_cast<char *>(workspace) + seg_bytes;
        e = ss2d::launch_transpose_planes(a.x, a.x_dtype == SS2D_BF16, xT, a.B * a.D, a.H, a.W, s);
        if (e != cudaSuccess)
            return cuda_fail(e, "ss2d_forward_core transpose launch");
        sa.uT = xT;
    }
    if (nseg > 1) {
        sa.nseg = nseg;
        sa.seg_len = seg_len;
        e = ss2d::launch_scan_segmented(sa, a.N, static_cast<float *>(workspace), s);
        return e == cudaSuccess ? SS2D_OK : cuda_fail(e, "ss2d_forward_core (segmented) launch");
    }
    e = ss2d::launch_scan(sa, a.N, ss2d::kFused, s);
    return e == cudaSuccess ? SS2D_OK : cuda_fail(e, "ss2d_forward_core launch");
}
