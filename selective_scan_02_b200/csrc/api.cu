// api.cu -- the C ABI of libss2d: argument checks on the host, then launches.
#include <stdarg.h>
#include <stddef.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "api_internal.h"
#include "kernels.h"
#include "proj_bwd.h"
#include "scan.cuh"
#include "scan_bwd.cuh"
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
    case SS2D_ERR_DEVICE: return "SS2D_ERR_DEVICE";
    default: return "SS2D_ERR_UNKNOWN";
    }
}

extern "C" const char *ss2d_last_error(void) { return g_err; }

extern "C" int ss2d_version(void) { return 107; }

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

namespace {

// The standalone scan, optionally from an initial state h0 and returning the final state.
int selective_scan_impl(const char *name, const void *u, int u_dtype, const void *delta, int delta_dtype,
                        const float *A_log, const float *Bm, const float *Cm, const float *Dv,
                        const float *delta_bias, int delta_softplus, const float *h0, float *h_last, float *y,
                        int B, int C, int G, int N, int L, void *stream)
{
    g_err[0] = 0;
    if (!u || !delta || !A_log || !Bm || !Cm || !y)
        return fail(SS2D_ERR_INVALID_ARG, "%s: u, delta, A_log, Bm, Cm and y must be non-null", name);
    if (B <= 0 || C <= 0 || G <= 0 || N <= 0 || L <= 0)
        return fail(SS2D_ERR_INVALID_ARG, "%s: sizes must be positive (B=%d C=%d G=%d N=%d L=%d)",
                    name, B, C, G, N, L);
    if (C % G != 0)
        return fail(SS2D_ERR_INVALID_ARG, "%s: C=%d is not a multiple of G=%d", name, C, G);
    if (!valid_dtype(u_dtype) || !valid_dtype(delta_dtype))
        return fail(SS2D_ERR_UNSUPPORTED, "%s: dtype codes (%d, %d) must be SS2D_F32 or SS2D_BF16",
                    name, u_dtype, delta_dtype);
    if (!valid_n(N))
        return fail(SS2D_ERR_UNSUPPORTED, "%s: N=%d is not one of 1, 2, 4, 8, 16", name, N);
    if ((long long)L > kMaxL || (long long)B * C > 0x7fffffffLL)
        return fail(SS2D_ERR_INVALID_ARG, "%s: problem too large", name);
    const void *ptrs[] = {u, delta, A_log, Bm, Cm, Dv, delta_bias, h0, h_last, y};
    for (const void *p : ptrs)
        if (p && !aligned16(p))
            return fail(SS2D_ERR_MISALIGNED, "%s: every tensor must be 16-byte aligned", name);
    const size_t nY = (size_t)B * C * L * 4;
    const Span ins[] = {{u, (size_t)B * C * L * esize(u_dtype)},
                        {delta, (size_t)B * C * L * esize(delta_dtype)},
                        {A_log, (size_t)C * N * 4},
                        {Bm, (size_t)B * G * N * L * 4},
                        {Cm, (size_t)B * G * N * L * 4},
                        {Dv, Dv ? (size_t)C * 4 : 0},
                        {delta_bias, delta_bias ? (size_t)C * 4 : 0},
                        {h0, h0 ? (size_t)B * C * N * 4 : 0}};
    const Span hl{h_last, h_last ? (size_t)B * C * N * 4 : 0};
    for (const Span &s : ins)
        if (overlaps(s, {y, nY}) || overlaps(s, hl))
            return fail(SS2D_ERR_INVALID_ARG, "%s: an output (y or h_last) overlaps an input", name);
    if (overlaps({y, nY}, hl))
        return fail(SS2D_ERR_INVALID_ARG, "%s: y overlaps h_last", name);

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
    a.h0 = h0;
    a.hlast = h_last;
    cudaError_t e = ss2d::launch_scan(a, N, ss2d::kStandalone, (cudaStream_t)stream);
    return e == cudaSuccess ? SS2D_OK : cuda_fail(e, name);
}

}  // namespace

extern "C" int ss2d_selective_scan(const void *u, int u_dtype, const void *delta, int delta_dtype,
                                   const float *A_log, const float *Bm, const float *Cm, const float *Dv,
                                   const float *delta_bias, int delta_softplus, float *y, int B, int C, int G,
                                   int N, int L, void *stream)
{
    return selective_scan_impl("ss2d_selective_scan", u, u_dtype, delta, delta_dtype, A_log, Bm, Cm, Dv,
                               delta_bias, delta_softplus, nullptr, nullptr, y, B, C, G, N, L, stream);
}

extern "C" int ss2d_selective_scan_state(const void *u, int u_dtype, const void *delta, int delta_dtype,
                                         const float *A_log, const float *Bm, const float *Cm, const float *Dv,
                                         const float *delta_bias, int delta_softplus, const float *h0,
                                         float *h_last, float *y, int B, int C, int G, int N, int L, void *stream)
{
    return selective_scan_impl("ss2d_selective_scan_state", u, u_dtype, delta, delta_dtype, A_log, Bm, Cm, Dv,
                               delta_bias, delta_softplus, h0, h_last, y, B, C, G, N, L, stream);
}

namespace {

// The layout of x and y; callers built against the struct without `layout` get channels-first.
int core_layout(const ss2d_core_args *a)
{
    return a->struct_size >= offsetof(ss2d_core_args, layout) + sizeof(int) ? a->layout : SS2D_CHANNELS_FIRST;
}

// The element type of y; callers built against the struct without `y_dtype` get fp32.
int core_y_dtype(const ss2d_core_args *a)
{
    return a->struct_size >= offsetof(ss2d_core_args, y_dtype) + sizeof(int) ? a->y_dtype : SS2D_F32;
}

float *core_ckpt(const ss2d_core_args *a)
{
    return a->struct_size >= offsetof(ss2d_core_args, ckpt) + sizeof(float *) ? a->ckpt : nullptr;
}

// The merge order; callers built against the struct without `merge_order` get atomic adds.
int core_merge_order(const ss2d_core_args *a)
{
    return a->struct_size >= offsetof(ss2d_core_args, merge_order) + sizeof(int) ? a->merge_order
                                                                                  : SS2D_MERGE_ATOMIC;
}

// Bytes of the checkpoint buffer: (B, 4D, ceil(L/16), 16) fp32.
size_t ckpt_bytes(const ss2d_core_args *a)
{
    const size_t L = (size_t)a->H * a->W;
    return (size_t)a->B * 4 * a->D * ((L + 15) / 16) * 16 * sizeof(float);
}

// Tiles of the per-image (H*W, D) transpose that channels-last x takes where a channels-first
// copy is needed (the x_proj GEMM, the backward); one launch covers at most 65535 of them.
long long channels_last_transpose_tiles(const ss2d_core_args *a)
{
    const long long L = (long long)a->H * a->W;
    return ((L + 31) / 32) * (((long long)a->D + 31) / 32);
}

bool channels_last_transpose_fits(const ss2d_core_args *a) { return channels_last_transpose_tiles(a) <= 65535; }

// Checks shared by the workspace query and the call; returns SS2D_OK or a status.
// check_y = false skips the checks of y's address (the workspace queries, the backward and
// ss2d_device_status, none of which writes y).
int check_core(const ss2d_core_args *a, bool check_y = true)
{
    if (!a)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: args is null");
    if (a->struct_size != sizeof(ss2d_core_args) && a->struct_size != offsetof(ss2d_core_args, merge_order) &&
        a->struct_size != offsetof(ss2d_core_args, ckpt) && a->struct_size != offsetof(ss2d_core_args, y_dtype) &&
        a->struct_size != offsetof(ss2d_core_args, layout))
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: struct_size %zu is not %zu, %zu, %zu, %zu or %zu",
                    a->struct_size, sizeof(ss2d_core_args), offsetof(ss2d_core_args, merge_order),
                    offsetof(ss2d_core_args, ckpt), offsetof(ss2d_core_args, y_dtype),
                    offsetof(ss2d_core_args, layout));
    if (a->B <= 0 || a->D <= 0 || a->H <= 0 || a->W <= 0 || a->N <= 0)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: sizes must be positive (B=%d D=%d H=%d W=%d N=%d)",
                    a->B, a->D, a->H, a->W, a->N);
    if (!a->x || !a->A_logs || (check_y && !a->y))
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
    if (!valid_dtype(core_y_dtype(a)))
        return fail(SS2D_ERR_UNSUPPORTED, "ss2d_forward_core: y_dtype %d is not SS2D_F32 or SS2D_BF16",
                    core_y_dtype(a));
    const int layout = core_layout(a);
    if (layout != SS2D_CHANNELS_FIRST && layout != SS2D_CHANNELS_LAST)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: layout %d is not SS2D_CHANNELS_FIRST or "
                    "SS2D_CHANNELS_LAST", layout);
    if (layout == SS2D_CHANNELS_LAST) {
        if (proj && !ss2d::xproj_dt_fused(a->R))
            return fail(SS2D_ERR_UNSUPPORTED,
                        "ss2d_forward_core: channels-last x/y with projections needs R <= 16 (dt_proj fused into "
                        "the scan); R=%d", a->R);
        const bool ok = a->N == 16 && a->delta_softplus && (!direct || a->x_dtype == a->dts_dtype) &&
                        ((size_t)a->D * esize(a->x_dtype)) % 16 == 0;
        if (!ok)
            return fail(SS2D_ERR_UNSUPPORTED,
                        "ss2d_forward_core: channels-last x/y needs N = 16, softplus on, x and dts of one type and "
                        "D * sizeof(x) a multiple of 16 bytes");
        if (proj && !channels_last_transpose_fits(a))
            return fail(SS2D_ERR_UNSUPPORTED,
                        "ss2d_forward_core: channels-last x with projections is transposed per image in 32x32 "
                        "tiles, at most 65535 of them: ceil(H*W/32) * ceil(D/32) is %lld",
                        channels_last_transpose_tiles(a));
    }
    if (layout == SS2D_CHANNELS_FIRST &&
        ss2d::scan_reads_transposed_u(a->N, proj ? ss2d::kFusedProj : ss2d::kFused, a->x_dtype == SS2D_BF16,
                                      proj ? 0 : a->dts_dtype == SS2D_BF16, a->delta_softplus != 0, (int)L) &&
        (long long)((a->H + 31) / 32) * ((a->W + 31) / 32) > 65535)
        return fail(SS2D_ERR_UNSUPPORTED,
                    "ss2d_forward_core: the column-major scan orders read x with its planes transposed, one launch "
                    "of at most 65535 tiles of 32x32: ceil(H/32) * ceil(W/32) is %lld",
                    (long long)((a->H + 31) / 32) * ((a->W + 31) / 32));
    const int mo = core_merge_order(a);
    if (mo != SS2D_MERGE_ATOMIC && mo != SS2D_MERGE_PAGE_ORDER)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: merge_order %d is not SS2D_MERGE_ATOMIC or "
                    "SS2D_MERGE_PAGE_ORDER", mo);
    if (mo == SS2D_MERGE_PAGE_ORDER) {
        const bool ok = direct && a->N == 16 && a->delta_softplus && a->x_dtype == a->dts_dtype;
        if (!ok)
            return fail(SS2D_ERR_UNSUPPORTED,
                        "ss2d_forward_core: SS2D_MERGE_PAGE_ORDER needs the dts/Bs/Cs form with N = 16, softplus "
                        "on, and x and dts of one type");
        // channel-first y is merged by one CrossMerge launch of 32x32 tiles per plane
        if (layout == SS2D_CHANNELS_FIRST && (long long)((a->H + 31) / 32) * ((a->W + 31) / 32) > 65535)
            return fail(SS2D_ERR_UNSUPPORTED,
                        "ss2d_forward_core: SS2D_MERGE_PAGE_ORDER merges channel-first y in one launch of at most "
                        "65535 tiles of 32x32 per plane: ceil(H/32) * ceil(W/32) is %lld",
                        (long long)((a->H + 31) / 32) * ((a->W + 31) / 32));
    }
    float *ck = core_ckpt(a);
    if (ck) {
        const bool ok = direct && a->N == 16 && a->delta_softplus && a->x_dtype == a->dts_dtype;
        if (!ok)
            return fail(SS2D_ERR_UNSUPPORTED,
                        "ss2d_forward_core: checkpoints are kept for the dts/Bs/Cs form with N = 16, softplus on, "
                        "and x and dts of one type");
    }
    const void *ptrs[] = {a->x, a->dts, a->Bs, a->Cs, a->A_logs, a->Ds, a->dt_bias,
                          a->x_proj_weight, a->dt_projs_weight, a->y, ck};
    for (const void *p : ptrs)
        if (p && !aligned16(p))
            return fail(SS2D_ERR_MISALIGNED, "ss2d_forward_core: every tensor must be 16-byte aligned");
    const size_t B = a->B, D = a->D, N = a->N, R = a->R;
    const Span y{a->y, B * D * L * esize(core_y_dtype(a))};
    const Span ins[] = {{a->x, B * D * L * esize(a->x_dtype)},
                        {a->dts, a->dts ? B * 4 * D * L * esize(a->dts_dtype) : 0},
                        {a->Bs, a->Bs ? B * 4 * N * L * 4 : 0},
                        {a->Cs, a->Cs ? B * 4 * N * L * 4 : 0},
                        {a->A_logs, 4 * D * N * 4},
                        {a->Ds, a->Ds ? 4 * D * 4 : 0},
                        {a->dt_bias, a->dt_bias ? 4 * D * 4 : 0},
                        {a->x_proj_weight, a->x_proj_weight ? 4 * (R + 2 * N) * D * 2 : 0},
                        {a->dt_projs_weight, a->dt_projs_weight ? 4 * D * R * 4 : 0}};
    if (check_y)
        for (const Span &s : ins)
            if (overlaps(s, y))
                return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: y overlaps an input");
    if (ck) {
        const Span c{ck, ckpt_bytes(a)};
        if (check_y && overlaps(c, y))
            return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: ckpt overlaps y");
        for (const Span &s : ins)
            if (overlaps(s, c))
                return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: ckpt overlaps an input");
    }
    return SS2D_OK;
}

}  // namespace

int ss2d::validate_core_args(const ss2d_core_args *a, bool check_y)
{
    return check_core(a, check_y);
}

bool ss2d::core_channels_last(const ss2d_core_args *a)
{
    return core_layout(a) == SS2D_CHANNELS_LAST;
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
    if (core_layout(a) == SS2D_CHANNELS_LAST)
        return 0;  // channels-last u of every scan order is read per pixel
    const int L = a->H * a->W;
    if (!ss2d::scan_reads_transposed_u(a->N, ss2d::kFused, a->x_dtype == SS2D_BF16, a->dts_dtype == SS2D_BF16,
                                       a->delta_softplus != 0, L))
        return 0;
    return (size_t)a->B * a->D * L * esize(a->x_dtype);
}

// Bytes of one fp32 copy of y.
size_t core_y_f32_bytes(const ss2d_core_args *a) { return (size_t)a->B * a->D * a->H * a->W * sizeof(float); }

// Offset of the page-order merge's outputs: with channel-first y the four directions' outputs
// in scan order, (B, 4D, L) fp32 as the standalone scan writes them, for a CrossMerge pass; with
// channels-last y three per-direction copies of y (directions 1, 2, 3; direction 0 writes y
// itself) for an element-wise sum.  After the segment states and the transposed copy of x.
size_t core_page_buffers_offset(const ss2d_core_args *a)
{
    int nseg, seg_len;
    core_segments(a, &nseg, &seg_len);
    return (ss2d::segment_workspace_bytes(a->B, 4 * a->D, nseg, a->N) + core_transposed_bytes(a) + 255) &
           ~(size_t)255;
}

// Workspace before the fp32 accumulation buffer of a bf16 y: for the direct form the segment
// states of a segmented scan (if any), then the transposed copy of x (if used), then (page-order
// merge) three fp32 copies of y; for the projection form the projection path's workspace.
size_t core_workspace_base(const ss2d_core_args *a)
{
    if (a->x_proj_weight)
        return ss2d::xproj_workspace_bytes(a->B, a->D, a->H, a->W, a->N, a->R,
                                           core_layout(a) == SS2D_CHANNELS_LAST);
    int nseg, seg_len;
    core_segments(a, &nseg, &seg_len);
    if (core_merge_order(a) == SS2D_MERGE_PAGE_ORDER)
        return core_page_buffers_offset(a) + (core_layout(a) == SS2D_CHANNELS_LAST
                                                  ? 3 * ((core_y_f32_bytes(a) + 255) & ~(size_t)255)
                                                  : 4 * core_y_f32_bytes(a));
    return ss2d::segment_workspace_bytes(a->B, 4 * a->D, nseg, a->N) + core_transposed_bytes(a);
}

// The whole workspace: the base, then (bf16 y only) y in fp32, where the four directions add up.
size_t core_workspace(const ss2d_core_args *a)
{
    const size_t base = (core_workspace_base(a) + 255) & ~(size_t)255;
    const size_t y32 = (size_t)a->B * a->D * a->H * a->W * sizeof(float);
    return core_y_dtype(a) == SS2D_BF16 ? base + y32 : core_workspace_base(a);
}

}  // namespace

extern "C" size_t ss2d_forward_core_workspace(const ss2d_core_args *args)
{
    g_err[0] = 0;
    if (check_core(args, false) != SS2D_OK)  // the size does not depend on y's address
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
    const bool ybf = core_y_dtype(args) == SS2D_BF16;
    const size_t y_bytes = (size_t)a.B * a.D * a.H * a.W * esize(core_y_dtype(args));
    if (need > 0) {
        if (!workspace || workspace_bytes < need)
            return fail(SS2D_ERR_WORKSPACE, "ss2d_forward_core: workspace of %zu bytes needed, %zu given", need,
                        workspace_bytes);
        if (!aligned16(workspace))
            return fail(SS2D_ERR_MISALIGNED, "ss2d_forward_core: workspace must be 16-byte aligned");
        if (overlaps({workspace, need}, {a.y, y_bytes}))
            return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core: workspace overlaps y");
    }
    cudaStream_t s = (cudaStream_t)stream;
    const int L = a.H * a.W;
    const size_t n_y = (size_t)a.B * a.D * L;
    // the four directions add up in fp32: in y itself, or for a bf16 y in the workspace
    float *y32 = ybf ? reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                                 ((core_workspace_base(args) + 255) & ~(size_t)255))
                     : static_cast<float *>(a.y);
    // the direct form's plane transpose of bf16 x also zeroes y; the projection form's launcher
    // zeroes y itself
    const bool page_order = core_merge_order(args) == SS2D_MERGE_PAGE_ORDER;
    const bool zero_in_transpose = !a.x_proj_weight && core_transposed_bytes(args) > 0 &&
                                   ss2d::transpose_planes_can_zero(a.x_dtype == SS2D_BF16, a.H, a.W);
    cudaError_t e = cudaSuccess;
    if (!a.x_proj_weight && !zero_in_transpose && !page_order) {  // the page-order merge stores every element
        e = ss2d::launch_fill_zero(y32, n_y, s);
        if (e != cudaSuccess)
            return cuda_fail(e, "ss2d_forward_core zero-fill launch");
    }
    if (a.x_proj_weight) {
        e = ss2d::launch_core_with_projections(a.x, a.x_proj_weight, a.dt_projs_weight, a.A_logs, a.Ds, a.dt_bias,
                                               a.delta_softplus != 0, y32, workspace, a.B, a.D, a.H, a.W, a.N, a.R,
                                               core_layout(args) == SS2D_CHANNELS_LAST, true, s);
        if (e != cudaSuccess)
            return cuda_fail(e, "ss2d_forward_core (projections) launch");
    } else {
        ss2d::ScanArgs sa{};
        sa.u = a.x;
        sa.delta = a.dts;
        sa.A_log = a.A_logs;
        sa.Bm = a.Bs;
        sa.Cm = a.Cs;
        sa.gs = (long long)a.N * L;
        sa.Dv = a.Ds;
        sa.bias = a.dt_bias;
        sa.y = y32;
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
        sa.ch_last = core_layout(args) == SS2D_CHANNELS_LAST;
        sa.ckpt = core_ckpt(args);  // kept for the backward when given
        int nseg, seg_len;
        core_segments(args, &nseg, &seg_len);
        const size_t seg_bytes = ss2d::segment_workspace_bytes(a.B, 4 * a.D, nseg, a.N);
        if (core_transposed_bytes(args) > 0) {
            void *xT = static_cast<char *>(workspace) + seg_bytes;
            e = zero_in_transpose && !page_order
                    ? ss2d::launch_transpose_planes_zero(a.x, xT, y32, a.B * a.D, a.H, a.W, s)
                                  : ss2d::launch_transpose_planes(a.x, a.x_dtype == SS2D_BF16, xT, a.B * a.D, a.H,
                                                                  a.W, s);
            if (e != cudaSuccess)
                return cuda_fail(e, "ss2d_forward_core transpose launch");
            sa.uT = xT;
        }
        // page order: every direction stores its output once, without atomics, and the four
        // are then added in the order of the article's sum ((y0 + inv_y0) + wh_y) + invwh_y:
        // channel-first y by CrossMerge from scan-order outputs, channels-last y element-wise
        // from direction 0's output in y and the others' in the workspace
        const bool cl = core_layout(args) == SS2D_CHANNELS_LAST;
        float *yd[3] = {nullptr, nullptr, nullptr};
        char *pb = static_cast<char *>(workspace) + (page_order ? core_page_buffers_offset(args) : 0);
        if (page_order && cl) {
            const size_t step = (core_y_f32_bytes(args) + 255) & ~(size_t)255;
            for (int k = 0; k < 3; ++k)
                yd[k] = reinterpret_cast<float *>(pb + k * step);
            sa.ydir[0] = y32;
            sa.ydir[1] = yd[0];
            sa.ydir[2] = yd[1];
            sa.ydir[3] = yd[2];
        } else if (page_order) {
            sa.ydir[0] = reinterpret_cast<float *>(pb);  // ys (B, 4D, L)
        }
        if (nseg > 1) {
            sa.nseg = nseg;
            sa.seg_len = seg_len;
            e = ss2d::launch_scan_segmented(sa, a.N, ss2d::kFused, static_cast<float *>(workspace), s);
            if (e != cudaSuccess)
                return cuda_fail(e, "ss2d_forward_core (segmented) launch");
        } else {
            e = ss2d::launch_scan(sa, a.N, ss2d::kFused, s);
            if (e != cudaSuccess)
                return cuda_fail(e, "ss2d_forward_core launch");
        }
        if (page_order) {
            e = cl ? ss2d::launch_page_order_sum(y32, yd[0], yd[1], yd[2], n_y, s)
                   : ss2d::launch_cross_merge(reinterpret_cast<const float *>(pb), y32, a.B, a.D, a.H, a.W, s);
            if (e != cudaSuccess)
                return cuda_fail(e, "ss2d_forward_core page-order merge launch");
        }
    }
    if (ybf) {
        e = ss2d::launch_f32_to_bf16(y32, a.y, n_y, s);
        if (e != cudaSuccess)
            return cuda_fail(e, "ss2d_forward_core bf16 output launch");
    }
    return SS2D_OK;
}

// ---- backward of the fused core ---------------------------------------------------------

namespace {

// Workspace of the backward, in this order: checkpoints, x with transposed planes (fp32),
// dy with transposed planes, and for bf16 inputs their fp32 copies (x, then dts).  The
// projection form adds: the x_proj error word, x_dbl, B and C copied out of x_dbl, the
// gradients of B, C and dts, the gradient of dt_low, and the per-CTA partial sums of the
// x_proj weight gradient; its dts copy holds dt_proj's output.
struct BwdPlan {
    size_t ckpt_bytes, xT_bytes, dyT_bytes, x32_bytes, dts32_bytes;
    size_t seg_bytes;  // segment states, (3, B, 4D, nseg, 16) fp32, for the larger of the two plans
    int ck_nseg, ck_seg_len;  // the checkpoint pass: the forward scan's plan
    int nseg, seg_len;        // the backward walk: its own plan, for its own CTAs per SM
    size_t hdr_bytes, xdbl_bytes, bc_bytes, ddts_bytes, dtlow_bytes, wxpart_bytes;
    size_t xcf_bytes, dycf_bytes, dxcf_bytes;  // channels-last: x, dy and dx in channels-first order
    size_t a16_bytes, bc16_bytes;  // N < 16: A_log (4D, 16) and B, C, dB, dC (B, 4, 16, L) padded to 16 states
    int nck;
    size_t direct_total() const { return ckpt_bytes + xT_bytes + dyT_bytes + x32_bytes + dts32_bytes + seg_bytes; }
    size_t proj_total() const
    {
        return hdr_bytes + xdbl_bytes + 4 * bc_bytes + ddts_bytes + dtlow_bytes + wxpart_bytes;
    }
    size_t pad_total() const { return 2 * a16_bytes + 4 * bc16_bytes; }
    size_t total() const { return direct_total() + proj_total() + xcf_bytes + dycf_bytes + dxcf_bytes + pad_total(); }
};

size_t round256(size_t n) { return (n + 255) & ~(size_t)255; }

BwdPlan bwd_plan(const ss2d_core_args &a)
{
    const size_t L = (size_t)a.H * a.W;
    BwdPlan p{};
    p.nck = (int)((L + ss2d::kBTC - 1) / ss2d::kBTC);
    p.ckpt_bytes = round256((size_t)a.B * 4 * a.D * p.nck * 16 * sizeof(float));
    p.xT_bytes = round256((size_t)a.B * a.D * L * sizeof(float));
    p.dyT_bytes = round256((size_t)a.B * a.D * L * sizeof(float));
    const bool bf16 = a.x_dtype == SS2D_BF16;
    p.x32_bytes = bf16 ? round256((size_t)a.B * a.D * L * sizeof(float)) : 0;
    p.dts32_bytes = bf16 ? round256((size_t)a.B * 4 * a.D * L * sizeof(float)) : 0;
    // long sequences with few channels: the checkpoint pass and the backward walk run in
    // segments, each planned for its own kernel's wave (whole sequences where the rows are not
    // whole 16-byte pieces: the segmented first passes take 16-byte rows).  The direct form's
    // checkpoint pass reads bf16 x and dts as they are; the projection form's backward hands it
    // fp32 ones.
    const int ck_bf16 = bf16 && !a.x_proj_weight ? 1 : 0;
    ss2d::plan_segments(a.B, 4, a.D, (int)L, 16, ss2d::kFused, ck_bf16, ck_bf16, 1, &p.ck_nseg, &p.ck_seg_len);
    if (L % 4 != 0 || (ck_bf16 && L % 8 != 0)) {
        p.ck_nseg = 1;
        p.ck_seg_len = (int)L;
    }
    ss2d::plan_bwd_segments(a.B, a.D, (int)L, &p.nseg, &p.seg_len);
    const int nseg_max = p.ck_nseg > p.nseg ? p.ck_nseg : p.nseg;
    p.seg_bytes = round256(ss2d::segment_workspace_bytes(a.B, 4 * a.D, nseg_max, 16));
    if (a.x_proj_weight) {
        const size_t Cp = (size_t)a.R + 2 * a.N;
        p.hdr_bytes = round256(ss2d::xproj_header_bytes());
        p.xdbl_bytes = round256((size_t)a.B * 4 * Cp * L * sizeof(float));
        p.bc_bytes = round256((size_t)a.B * 4 * a.N * L * sizeof(float));
        p.ddts_bytes = round256((size_t)a.B * 4 * a.D * L * sizeof(float));
        p.dtlow_bytes = round256((size_t)a.B * 4 * a.R * L * sizeof(float));
        p.wxpart_bytes = round256(ss2d::xproj_bwd_partial_bytes(a.N, a.R, a.D, a.W));
    }
    if (core_layout(&a) == SS2D_CHANNELS_LAST) {
        p.xcf_bytes = round256((size_t)a.B * a.D * L * esize(a.x_dtype));
        p.dycf_bytes = round256((size_t)a.B * a.D * L * sizeof(float));
        p.dxcf_bytes = round256((size_t)a.B * a.D * L * sizeof(float));
    }
    if (!a.x_proj_weight && a.N < 16) {
        p.a16_bytes = round256((size_t)4 * a.D * 16 * sizeof(float));
        p.bc16_bytes = round256((size_t)a.B * 4 * 16 * L * sizeof(float));
    }
    return p;
}

// Checks of the backward's forward arguments (y is not used): the forward checks and the
// supported forms and shapes.
int check_core_bwd_args(const ss2d_core_args *args)
{
    if (!args)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core_backward: args must be non-null");
    int st = check_core(args, false);
    if (st != SS2D_OK)
        return st;
    const ss2d_core_args &a = *args;
    const int L = a.H * a.W;
    const long long plane_tiles = (long long)((a.H + 31) / 32) * ((a.W + 31) / 32);
    if (plane_tiles > 65535)  // x and dy are read with their planes transposed, one launch each
        return fail(SS2D_ERR_UNSUPPORTED,
                    "ss2d_forward_core_backward: x and dy are transposed plane by plane in one launch of at most "
                    "65535 tiles of 32x32: ceil(H/32) * ceil(W/32) is %lld", plane_tiles);
    if (a.x_proj_weight) {
        if (a.N != 16 || !a.delta_softplus || !ss2d::proj_bwd_supported(a.N, a.R, a.D, a.W))
            return fail(SS2D_ERR_UNSUPPORTED,
                        "ss2d_forward_core_backward: the projection form's backward supports N = 16, softplus on, "
                        "1 <= R <= 64, D %% 16 == 0 (got N=%d, softplus %d, R=%d, D=%d)",
                        a.N, a.delta_softplus, a.R, a.D);
        if (a.B > 16383)  // dt_proj's adjoint kernels put (image, direction) in the grid's y, at most 65535
            return fail(SS2D_ERR_UNSUPPORTED,
                        "ss2d_forward_core_backward: the projection form's backward takes at most 16383 images "
                        "(got B=%d)", a.B);
        return SS2D_OK;
    }
    if (core_layout(&a) == SS2D_CHANNELS_LAST && !channels_last_transpose_fits(&a))
        return fail(SS2D_ERR_UNSUPPORTED,
                    "ss2d_forward_core_backward: channels-last x, dy and dx are transposed per image in 32x32 "
                    "tiles, at most 65535 of them: ceil(H*W/32) * ceil(D/32) is %lld",
                    channels_last_transpose_tiles(&a));
    // N < 16 runs as N = 16 with inert padded states (B = C = 0)
    if (a.N > 16 || !ss2d::scan_bwd_supported(16, a.x_dtype == SS2D_BF16, a.dts_dtype == SS2D_BF16,
                                              a.delta_softplus != 0, L))
        return fail(SS2D_ERR_UNSUPPORTED,
                    "ss2d_forward_core_backward: supported are N <= 16, x and dts both bf16 or both fp32, "
                    "softplus on (got N=%d, x %d, dts %d, H*W=%d, softplus %d)",
                    a.N, a.x_dtype, a.dts_dtype, L, a.delta_softplus);
    return SS2D_OK;
}

// The grads struct of the call, with the members an older caller's struct lacks set to NULL.
int read_core_grads(const ss2d_core_grads *g, ss2d_core_grads *out)
{
    const size_t v102 = offsetof(ss2d_core_grads, dx_proj_weight);
    if (!g)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core_backward: grads must be non-null");
    if (g->struct_size != sizeof(ss2d_core_grads) && g->struct_size != v102)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core_backward: grads struct_size %zu is neither %zu nor %zu",
                    g->struct_size, sizeof(ss2d_core_grads), v102);
    *out = ss2d_core_grads{};
    memcpy(out, g, g->struct_size);
    return SS2D_OK;
}

// All checks of the backward call: the arguments, and the gradients (no gradient may overlap
// an input or another gradient).
int check_core_bwd(const ss2d_core_args *args, const ss2d_core_grads &g)
{
    int st0 = check_core_bwd_args(args);
    if (st0 != SS2D_OK)
        return st0;
    const ss2d_core_args &a = *args;
    const bool proj = a.x_proj_weight != nullptr;
    if (!g.dy || !g.dx || !g.dA_logs)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core_backward: dy, dx and dA_logs must be non-null");
    if (proj && (!g.dx_proj_weight || !g.ddt_projs_weight))
        return fail(SS2D_ERR_INVALID_ARG,
                    "ss2d_forward_core_backward: the projection form needs dx_proj_weight and ddt_projs_weight");
    if (!proj && (!g.ddts || !g.dBs || !g.dCs))
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core_backward: the dts/Bs/Cs form needs ddts, dBs and dCs");
    if (!proj && (g.dx_proj_weight || g.ddt_projs_weight))
        return fail(SS2D_ERR_INVALID_ARG,
                    "ss2d_forward_core_backward: weight gradients are only defined for the projection form");
    const int L = a.H * a.W;
    const size_t B = a.B, D = a.D, N = a.N, R = a.R, Ls = L, Cp = R + 2 * N;
    const Span out_spans[] = {{g.dx, B * D * Ls * 4},
                              {g.ddts, g.ddts ? B * 4 * D * Ls * 4 : 0},
                              {g.dA_logs, 4 * D * N * 4},
                              {g.dBs, g.dBs ? B * 4 * N * Ls * 4 : 0},
                              {g.dCs, g.dCs ? B * 4 * N * Ls * 4 : 0},
                              {g.dDs, g.dDs ? 4 * D * 4 : 0},
                              {g.ddt_bias, g.ddt_bias ? 4 * D * 4 : 0},
                              {g.dx_proj_weight, g.dx_proj_weight ? 4 * Cp * D * 4 : 0},
                              {g.ddt_projs_weight, g.ddt_projs_weight ? 4 * D * R * 4 : 0}};
    if (!aligned16(g.dy))
        return fail(SS2D_ERR_MISALIGNED, "ss2d_forward_core_backward: every tensor must be 16-byte aligned");
    for (const Span &o : out_spans)
        if (o.p && !aligned16(o.p))
            return fail(SS2D_ERR_MISALIGNED, "ss2d_forward_core_backward: every tensor must be 16-byte aligned");
    const Span in_spans[] = {{a.x, B * D * Ls * esize(a.x_dtype)},
                             {a.dts, a.dts ? B * 4 * D * Ls * esize(a.dts_dtype) : 0},
                             {a.Bs, a.Bs ? B * 4 * N * Ls * 4 : 0},
                             {a.Cs, a.Cs ? B * 4 * N * Ls * 4 : 0},
                             {a.x_proj_weight, proj ? 4 * Cp * D * 2 : 0},
                             {a.dt_projs_weight, proj ? 4 * D * R * 4 : 0},
                             {a.A_logs, 4 * D * N * 4},
                             {a.Ds, a.Ds ? 4 * D * 4 : 0},
                             {a.dt_bias, a.dt_bias ? 4 * D * 4 : 0},
                             {g.dy, B * D * Ls * 4},
                             {core_ckpt(&a), core_ckpt(&a) ? ckpt_bytes(&a) : 0}};
    constexpr size_t n_out = sizeof(out_spans) / sizeof(out_spans[0]);
    for (size_t i = 0; i < n_out; ++i) {
        for (const Span &in : in_spans)
            if (overlaps(out_spans[i], in))
                return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core_backward: a gradient overlaps an input");
        for (size_t k = i + 1; k < n_out; ++k)
            if (overlaps(out_spans[i], out_spans[k]))
                return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core_backward: two gradients overlap");
    }
    return SS2D_OK;
}

// The backward of the dts/Bs/Cs form (checks done): zero the accumulated gradients, widen
// bf16 inputs, transpose x and dy, run the checkpoint pass and the backward scan.
int core_bwd_run(const ss2d_core_args &a, const ss2d_core_grads &g, char *w, const BwdPlan &p, cudaStream_t s)
{
    const size_t B = a.B, D = a.D, N = a.N;
    const int L = a.H * a.W;
    float *ckpt = reinterpret_cast<float *>(w);
    float *xT = reinterpret_cast<float *>(w + p.ckpt_bytes);
    float *dyT = reinterpret_cast<float *>(w + p.ckpt_bytes + p.xT_bytes);
    const bool bf16 = a.x_dtype == SS2D_BF16;
    const void *x32 = a.x, *dts32 = a.dts;

    // accumulated gradients start at zero; ddts is written in full
    cudaError_t e = cudaSuccess;
    struct {
        float *p;
        size_t n;
    } zero[] = {{g.dx, B * D * L}, {g.dA_logs, 4 * D * N}, {g.dBs, B * 4 * N * L}, {g.dCs, B * 4 * N * L},
                {g.dDs, g.dDs ? 4 * D : 0}, {g.ddt_bias, g.ddt_bias ? 4 * D : 0}};
    for (auto &z : zero)
        if (z.p && z.n && e == cudaSuccess)
            e = ss2d::launch_fill_zero(z.p, z.n, s);
    if (e != cudaSuccess)
        return cuda_fail(e, "ss2d_forward_core_backward preparation launch");

    // The checkpoint pass: the forward scan, storing its state before every 16th step.  bf16
    // inputs are read as they are (the bf16 layout fits 12 CTAs per SM, the fp32 one 10), with
    // their plane-transposed copy parked in the space the widened x takes afterwards; the
    // values are the same, as the widening is exact.
    ss2d::ScanArgs sa{};
    sa.A_log = a.A_logs;
    sa.Bm = a.Bs;
    sa.Cm = a.Cs;
    sa.gs = (long long)a.N * L;
    sa.Dv = a.Ds;
    sa.bias = a.dt_bias;
    sa.B = a.B;
    sa.C = 4 * a.D;
    sa.G = 4;
    sa.L = L;
    sa.per_group = a.D;
    sa.W = a.W;
    sa.divH = {a.H, 1.0f / (float)a.H};
    sa.softplus = 1;
    float *xw = reinterpret_cast<float *>(w + p.ckpt_bytes + p.xT_bytes + p.dyT_bytes);
    float *dw = reinterpret_cast<float *>(w + p.ckpt_bytes + p.xT_bytes + p.dyT_bytes + p.x32_bytes);
    float *seg_ws = reinterpret_cast<float *>(w + p.ckpt_bytes + p.xT_bytes + p.dyT_bytes + p.x32_bytes +
                                              p.dts32_bytes);
    const size_t seg_n = (size_t)a.B * 4 * a.D * p.nseg * 16;
    float *given = core_ckpt(&a);
    if (given) {
        ckpt = given;  // kept by the forward call with these arguments
    } else {
        if (bf16) {
            sa.u = a.x;
            sa.delta = a.dts;
            sa.u_bf16 = 1;
            sa.delta_bf16 = 1;
            sa.delta_bytes = (size_t)a.B * 4 * a.D * L * 2;
            sa.uT = nullptr;
            if (ss2d::scan_reads_transposed_u(16, ss2d::kFused, 1, 1, 1, L)) {
                e = ss2d::launch_transpose_planes(a.x, true, xw, a.B * a.D, a.H, a.W, s);
                sa.uT = xw;
            }
        } else {
            // fp32 inputs: the scan reads x and its plane-transposed copy, made here for the walk too
            e = ss2d::launch_transpose_planes(a.x, false, xT, a.B * a.D, a.H, a.W, s);
            sa.u = a.x;
            sa.uT = xT;
            sa.delta = a.dts;
            sa.delta_bytes = (size_t)a.B * 4 * a.D * L * sizeof(float);
        }
        if (e == cudaSuccess && p.ck_nseg > 1) {
            sa.nseg = p.ck_nseg;
            sa.seg_len = p.ck_seg_len;
            e = ss2d::launch_scan_checkpoints_segmented(sa, ckpt, seg_ws, s);
        } else if (e == cudaSuccess) {
            e = ss2d::launch_scan_checkpoints(sa, ckpt, s);
        }
        if (e != cudaSuccess)
            return cuda_fail(e, "ss2d_forward_core_backward checkpoint launch");
    }

    // the backward scan runs on fp32 x and dts: bf16 inputs are widened into the workspace
    // (over the checkpoint pass's transposed copy, which it has finished reading; that copy is
    // first widened into the fp32 transposed copy the walk reads)
    const bool xT_from_bf16 = bf16 && !given && sa.uT != nullptr;
    if (xT_from_bf16)
        e = ss2d::launch_bf16_to_f32(xw, xT, B * D * L, s);
    if (bf16 && e == cudaSuccess) {
        e = ss2d::launch_bf16_to_f32(a.x, xw, B * D * L, s);
        if (e == cudaSuccess)
            e = ss2d::launch_bf16_to_f32(a.dts, dw, B * 4 * D * L, s);
        x32 = xw;
        dts32 = dw;
    }
    if (e == cudaSuccess && (bf16 || given) && !xT_from_bf16)
        e = ss2d::launch_transpose_planes(x32, false, xT, a.B * a.D, a.H, a.W, s);
    if (e == cudaSuccess)
        e = ss2d::launch_transpose_planes(g.dy, false, dyT, a.B * a.D, a.H, a.W, s);
    if (e != cudaSuccess)
        return cuda_fail(e, "ss2d_forward_core_backward preparation launch");

    ss2d::BwdArgs ba{};
    ba.x = x32;
    ba.xT = xT;
    ba.dts = dts32;
    ba.A_log = a.A_logs;
    ba.Bm = a.Bs;
    ba.Cm = a.Cs;
    ba.Dv = a.Ds;
    ba.bias = a.dt_bias;
    ba.ckpt = ckpt;
    ba.dy = g.dy;
    ba.dyT = dyT;
    ba.dx = g.dx;
    ba.ddts = g.ddts;
    ba.dA_log = g.dA_logs;
    ba.dBm = g.dBs;
    ba.dCm = g.dCs;
    ba.dDv = g.dDs;
    ba.dbias = g.ddt_bias;
    ba.B = a.B;
    ba.D = a.D;
    ba.W = a.W;
    ba.L = L;
    ba.C = 4 * a.D;
    ba.nck = p.nck;
    ba.divH = {a.H, 1.0f / (float)a.H};
    ba.nseg = p.nseg;
    ba.seg_len = p.seg_len;
    if (p.nseg > 1) {
        // the checkpoint pass's segment states are dead: the backward's carry reuses the space
        ba.e_out = seg_ws;
        ba.p_out = seg_ws + seg_n;
        ba.g_in = seg_ws + 2 * seg_n;
    }
    e = ss2d::launch_scan_bwd(ba, s);
    return e == cudaSuccess ? SS2D_OK : cuda_fail(e, "ss2d_forward_core_backward launch");
}

// The dts/Bs/Cs backward for N < 16: the kernels run 16 states, so A_log, B and C are padded
// with states whose B and C are zero (their states stay zero and add nothing to any gradient),
// and the first N states of dA_log, dB and dC are copied back.
int core_bwd_padded(const ss2d_core_args &a, const ss2d_core_grads &g, char *w, const BwdPlan &p, cudaStream_t s)
{
    const size_t B = a.B, D = a.D, N = a.N, L = (size_t)a.H * a.W;
    char *q = w + p.direct_total() + p.proj_total() + p.xcf_bytes + p.dycf_bytes + p.dxcf_bytes;
    float *A16 = reinterpret_cast<float *>(q);
    float *dA16 = reinterpret_cast<float *>(q + p.a16_bytes);
    q += 2 * p.a16_bytes;
    float *B16 = reinterpret_cast<float *>(q);
    float *C16 = reinterpret_cast<float *>(q + p.bc16_bytes);
    float *dB16 = reinterpret_cast<float *>(q + 2 * p.bc16_bytes);
    float *dC16 = reinterpret_cast<float *>(q + 3 * p.bc16_bytes);
    const size_t rowsA = 4 * D, rowsBC = B * 4;
    cudaError_t e = ss2d::launch_fill_zero(A16, rowsA * 16, s);
    if (e == cudaSuccess)
        e = ss2d::launch_fill_zero(B16, rowsBC * 16 * L, s);
    if (e == cudaSuccess)
        e = ss2d::launch_fill_zero(C16, rowsBC * 16 * L, s);
    const cudaMemcpyKind dd = cudaMemcpyDeviceToDevice;
    if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(A16, 16 * sizeof(float), a.A_logs, N * sizeof(float), N * sizeof(float), rowsA, dd, s);
    if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(B16, 16 * L * sizeof(float), a.Bs, N * L * sizeof(float), N * L * sizeof(float),
                              rowsBC, dd, s);
    if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(C16, 16 * L * sizeof(float), a.Cs, N * L * sizeof(float), N * L * sizeof(float),
                              rowsBC, dd, s);
    if (e != cudaSuccess)
        return cuda_fail(e, "ss2d_forward_core_backward state padding launch");
    ss2d_core_args d = a;
    d.N = 16;
    d.A_logs = A16;
    d.Bs = B16;
    d.Cs = C16;
    ss2d_core_grads gd = g;
    gd.dA_logs = dA16;
    gd.dBs = dB16;
    gd.dCs = dC16;
    int st = core_bwd_run(d, gd, w, p, s);
    if (st != SS2D_OK)
        return st;
    e = cudaMemcpy2DAsync(g.dA_logs, N * sizeof(float), dA16, 16 * sizeof(float), N * sizeof(float), rowsA, dd, s);
    if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(g.dBs, N * L * sizeof(float), dB16, 16 * L * sizeof(float), N * L * sizeof(float),
                              rowsBC, dd, s);
    if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(g.dCs, N * L * sizeof(float), dC16, 16 * L * sizeof(float), N * L * sizeof(float),
                              rowsBC, dd, s);
    return e == cudaSuccess ? SS2D_OK : cuda_fail(e, "ss2d_forward_core_backward state unpadding launch");
}

// The backward of the projection form: recompute x_dbl (x_proj on the tensor cores) and
// dts = dt_proj(x_dbl), run the dts/Bs/Cs backward on them in fp32, then the projections'
// adjoints.
int core_bwd_proj(const ss2d_core_args &a, const ss2d_core_grads &g, char *w, const BwdPlan &p, cudaStream_t s)
{
    const size_t B = a.B, D = a.D, N = a.N, R = a.R, Cp = R + 2 * N;
    const int L = a.H * a.W;
    float *x32 = reinterpret_cast<float *>(w + p.ckpt_bytes + p.xT_bytes + p.dyT_bytes);
    float *dts32 = reinterpret_cast<float *>(w + p.ckpt_bytes + p.xT_bytes + p.dyT_bytes + p.x32_bytes);
    char *q = w + p.direct_total();
    int *err = reinterpret_cast<int *>(q);
    q += p.hdr_bytes;
    float *xdbl = reinterpret_cast<float *>(q);
    q += p.xdbl_bytes;
    float *Bs32 = reinterpret_cast<float *>(q);
    q += p.bc_bytes;
    float *Cs32 = reinterpret_cast<float *>(q);
    q += p.bc_bytes;
    float *dB = reinterpret_cast<float *>(q);
    q += p.bc_bytes;
    float *dC = reinterpret_cast<float *>(q);
    q += p.bc_bytes;
    float *ddts = reinterpret_cast<float *>(q);
    q += p.ddts_bytes;
    float *d_dtlow = reinterpret_cast<float *>(q);
    q += p.dtlow_bytes;
    float *wxpart = reinterpret_cast<float *>(q);

    // dx_proj_weight is written in full at the end; ddt_projs_weight accumulates
    cudaError_t e = ss2d::launch_fill_zero(g.ddt_projs_weight, 4 * D * R, s);
    if (e == cudaSuccess)
        e = ss2d::launch_clear_error_word(err, s);
    if (e == cudaSuccess)
        e = ss2d::launch_xproj_gemm(a.x, a.x_proj_weight, xdbl, err, a.B, a.D, a.H, a.W, a.N, a.R, s);
    if (e == cudaSuccess)
        e = ss2d::launch_dtproj_expand(xdbl, a.dt_projs_weight, dts32, a.B, a.D, L, a.R, a.N, s);
    // B and C rows of x_dbl, as dense (B, 4, N, L) arrays
    const size_t row = (size_t)N * L * sizeof(float), pitch = Cp * L * sizeof(float);
    if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(Bs32, row, xdbl + R * L, pitch, row, B * 4, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(Cs32, row, xdbl + (R + N) * L, pitch, row, B * 4, cudaMemcpyDeviceToDevice, s);
    // The checkpoint pass on bf16 x as it is (with a bf16 plane-transposed copy, parked where
    // the walk's fp32 copy goes afterwards) and the expanded fp32 dts: that layout fits 11 CTAs
    // per SM where the all-fp32 one fits 10, so the projection workload's 3072 CTAs take two
    // waves instead of three.  Whole sequences with 16-byte bf16 rows; else the dts/Bs/Cs
    // backward makes its own checkpoints from the widened x.
    float *ckpt = reinterpret_cast<float *>(w);
    const bool own_ckpt = p.ck_nseg == 1 && ((size_t)L * 2) % 16 == 0;
    if (e == cudaSuccess && own_ckpt) {
        void *xT16 = w + p.ckpt_bytes;
        e = ss2d::launch_transpose_planes(a.x, true, xT16, a.B * a.D, a.H, a.W, s);
        ss2d::ScanArgs sa{};
        sa.u = a.x;
        sa.uT = xT16;
        sa.delta = dts32;
        sa.A_log = a.A_logs;
        sa.Bm = Bs32;
        sa.Cm = Cs32;
        sa.gs = (long long)N * L;
        sa.Dv = a.Ds;
        sa.bias = a.dt_bias;
        sa.B = a.B;
        sa.C = 4 * a.D;
        sa.G = 4;
        sa.L = L;
        sa.per_group = a.D;
        sa.W = a.W;
        sa.divH = {a.H, 1.0f / (float)a.H};
        sa.u_bf16 = 1;
        sa.delta_bf16 = 0;
        sa.softplus = 1;
        sa.delta_bytes = B * 4 * D * L * sizeof(float);
        if (e == cudaSuccess)
            e = ss2d::launch_scan_checkpoints(sa, ckpt, s);
    }
    if (e == cudaSuccess)
        e = ss2d::launch_bf16_to_f32(a.x, x32, B * D * L, s);
    if (e != cudaSuccess)
        return cuda_fail(e, "ss2d_forward_core_backward projection launch");

    ss2d_core_args d = a;
    if (own_ckpt)
        d.ckpt = ckpt;  // the dts/Bs/Cs backward takes these checkpoints as given
    d.x = x32;
    d.x_dtype = SS2D_F32;
    d.dts = dts32;
    d.dts_dtype = SS2D_F32;
    d.Bs = Bs32;
    d.Cs = Cs32;
    d.x_proj_weight = nullptr;
    d.dt_projs_weight = nullptr;
    ss2d_core_grads gd = g;
    gd.ddts = ddts;
    gd.dBs = dB;
    gd.dCs = dC;
    int st = core_bwd_run(d, gd, w, p, s);
    if (st != SS2D_OK)
        return st;

    ss2d::ProjGradRows rows{d_dtlow, dB, dC, a.R, a.N};
    e = ss2d::launch_proj_bwd(rows, ddts, xdbl, a.dt_projs_weight, a.x_proj_weight, a.x, g.dx,
                              g.ddt_projs_weight, g.dx_proj_weight, wxpart, err, a.B, a.D, a.H, a.W, s);
    // the intermediates' gradients, when asked for
    struct {
        float *dst;
        const float *src;
        size_t n;
    } outs[] = {{g.ddts, ddts, B * 4 * D * L}, {g.dBs, dB, B * 4 * N * L}, {g.dCs, dC, B * 4 * N * L}};
    for (auto &o : outs)
        if (o.dst && e == cudaSuccess)
            e = cudaMemcpyAsync(o.dst, o.src, o.n * sizeof(float), cudaMemcpyDeviceToDevice, s);
    return e == cudaSuccess ? SS2D_OK : cuda_fail(e, "ss2d_forward_core_backward projection gradient launch");
}

}  // namespace

extern "C" size_t ss2d_forward_core_backward_workspace(const ss2d_core_args *args)
{
    g_err[0] = 0;
    if (check_core_bwd_args(args) != SS2D_OK)
        return (size_t)-1;
    return bwd_plan(*args).total();
}

extern "C" int ss2d_forward_core_backward(const ss2d_core_args *args, const ss2d_core_grads *grads, void *workspace,
                                          size_t workspace_bytes, void *stream)
{
    g_err[0] = 0;
    ss2d_core_grads g;
    int st = read_core_grads(grads, &g);
    if (st != SS2D_OK)
        return st;
    st = check_core_bwd(args, g);
    if (st != SS2D_OK)
        return st;
    // a full-size copy: members an older caller's struct lacks take their defaults (zero)
    ss2d_core_args a{};
    memcpy(&a, args, args->struct_size);
    a.struct_size = sizeof(ss2d_core_args);
    const BwdPlan p = bwd_plan(a);
    const size_t need = p.total();
    if (!workspace || workspace_bytes < need)
        return fail(SS2D_ERR_WORKSPACE, "ss2d_forward_core_backward: workspace of %zu bytes needed, %zu given", need,
                    workspace_bytes);
    if (!aligned16(workspace))
        return fail(SS2D_ERR_MISALIGNED, "ss2d_forward_core_backward: workspace must be 16-byte aligned");
    const size_t B = a.B, D = a.D, N = a.N, R = a.R, Cp = R + 2 * N;
    const int L = a.H * a.W;
    const bool proj = a.x_proj_weight != nullptr;
    const Span ws{workspace, need};
    const Span touched[] = {{g.dx, B * D * L * 4},
                            {g.ddts, g.ddts ? B * 4 * D * L * 4 : 0},
                            {g.dA_logs, 4 * D * N * 4},
                            {g.dBs, g.dBs ? B * 4 * N * L * 4 : 0},
                            {g.dCs, g.dCs ? B * 4 * N * L * 4 : 0},
                            {g.dDs, g.dDs ? 4 * D * 4 : 0},
                            {g.ddt_bias, g.ddt_bias ? 4 * D * 4 : 0},
                            {g.dx_proj_weight, g.dx_proj_weight ? 4 * Cp * D * 4 : 0},
                            {g.ddt_projs_weight, g.ddt_projs_weight ? 4 * D * R * 4 : 0},
                            {g.dy, B * D * L * 4},
                            {a.x, B * D * L * esize(a.x_dtype)},
                            {a.dts, a.dts ? B * 4 * D * L * esize(a.dts_dtype) : 0},
                            {a.Bs, a.Bs ? B * 4 * N * L * 4 : 0},
                            {a.Cs, a.Cs ? B * 4 * N * L * 4 : 0},
                            {a.x_proj_weight, proj ? 4 * Cp * D * 2 : 0},
                            {a.dt_projs_weight, proj ? 4 * D * R * 4 : 0},
                            {core_ckpt(&a), core_ckpt(&a) ? ckpt_bytes(&a) : 0}};
    for (const Span &t : touched)
        if (overlaps(ws, t))
            return fail(SS2D_ERR_INVALID_ARG, "ss2d_forward_core_backward: workspace overlaps a tensor");
    cudaStream_t s = (cudaStream_t)stream;
    char *w = static_cast<char *>(workspace);
    if (core_layout(&a) != SS2D_CHANNELS_LAST) {
        if (proj)
            return core_bwd_proj(a, g, w, p, s);
        return a.N < 16 ? core_bwd_padded(a, g, w, p, s) : core_bwd_run(a, g, w, p, s);
    }

    // Channels-last x, dy and dx, (B, H, W, D): the backward runs on channels-first copies,
    // each image's (L, D) matrix transposed into the workspace and dx transposed back.
    char *c = w + p.direct_total() + p.proj_total();
    void *x_cf = c;
    float *dy_cf = reinterpret_cast<float *>(c + p.xcf_bytes);
    float *dx_cf = reinterpret_cast<float *>(c + p.xcf_bytes + p.dycf_bytes);
    cudaError_t e = ss2d::launch_transpose_planes(a.x, a.x_dtype == SS2D_BF16, x_cf, a.B, L, a.D, s);
    if (e == cudaSuccess)
        e = ss2d::launch_transpose_planes(g.dy, false, dy_cf, a.B, L, a.D, s);
    if (e != cudaSuccess)
        return cuda_fail(e, "ss2d_forward_core_backward channels-last preparation launch");
    ss2d_core_args acf = a;
    acf.struct_size = sizeof(ss2d_core_args);
    acf.layout = SS2D_CHANNELS_FIRST;
    acf.x = x_cf;
    ss2d_core_grads gcf = g;
    gcf.dy = dy_cf;
    gcf.dx = dx_cf;
    st = proj ? core_bwd_proj(acf, gcf, w, p, s) : core_bwd_run(acf, gcf, w, p, s);
    if (st != SS2D_OK)
        return st;
    e = ss2d::launch_transpose_planes(dx_cf, false, g.dx, a.B, a.D, L, s);
    return e == cudaSuccess ? SS2D_OK : cuda_fail(e, "ss2d_forward_core_backward channels-last dx launch");
}

extern "C" int ss2d_device_status(const ss2d_core_args *args, const void *workspace, int backward, void *stream)
{
    g_err[0] = 0;
    if (backward != 0 && backward != 1)
        return fail(SS2D_ERR_INVALID_ARG, "ss2d_device_status: backward must be 0 or 1, got %d", backward);
    const int st = backward ? check_core_bwd_args(args) : check_core(args, false);
    if (st != SS2D_OK)
        return st;
    if (!args->x_proj_weight)
        return SS2D_OK;  // the dts/Bs/Cs form runs no tensor-core kernel and waits on nothing
    ss2d_core_args a{};
    memcpy(&a, args, args->struct_size);
    a.struct_size = sizeof(ss2d_core_args);
    // the word sits at the start of the projection path's workspace; in the backward's
    // workspace that part follows the direct form's
    const char *word = static_cast<const char *>(workspace);
    if (backward) {
        if (!workspace)
            return fail(SS2D_ERR_WORKSPACE, "ss2d_device_status: the backward's workspace is required");
        word += bwd_plan(a).direct_total();
    } else if (!workspace) {
        void *scratch = nullptr;
        const cudaError_t e = ss2d::static_scratch_address(&scratch);
        if (e != cudaSuccess)
            return cuda_fail(e, "ss2d_device_status static scratch lookup");
        word = static_cast<const char *>(scratch);
    }
    if (!aligned16(word))
        return fail(SS2D_ERR_MISALIGNED, "ss2d_device_status: workspace must be 16-byte aligned");
    int flag = 0;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(&flag, word, sizeof(flag), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(s);
    if (e != cudaSuccess)
        return cuda_fail(e, "ss2d_device_status read");
    if (flag != 0)
        return fail(SS2D_ERR_DEVICE,
                    "ss2d_device_status: a tensor-core kernel's bounded wait ran out; that call's outputs are not "
                    "valid");
    return SS2D_OK;
}
