// static_scratch.cu -- ss2d_forward_core_static: the projection form of the
// fused core for callers that cannot allocate device memory.
//
// The projection form needs scratch for x_dbl (4*(R+2N) fp32 values per pixel
// and image).  Here that scratch is a fixed array in the library's own device
// memory instead of a caller-provided workspace: the batch is processed in
// slices of as many images as fit in the array, one after another on the
// caller's stream, with the same kernels ss2d_forward_core launches.
//
// The array lives in static device memory, so every GPU that loads the
// library holds kStaticScratchBytes until the process exits.  In host code
// the array's name is only a host-side stand-in, so its device address is
// looked up once per device with cudaGetSymbolAddress and cached; a device
// reset (cudaDeviceReset) drops the array's memory with the context, so the
// cached address is not valid after one and the library must not be called on
// that device again in the same process.
#include <mutex>
#include <stddef.h>
#include <stdio.h>

#include "api_internal.h"
#include "kernels.h"
#include "ss2d.h"
#include "xproj.h"

namespace {

constexpr size_t kStaticScratchBytes = SS2D_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 128;

static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

std::mutex g_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

int static_fail(int status, const char *msg) { return ss2d::set_last_error(status, msg); }

}  // namespace

// Device address of g_scratch on the current device (looked up on first use).
cudaError_t ss2d::static_scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess)
            return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

// Images in the next slice of ss2d_forward_core_static when `left` images of the batch
// remain.  The projection form's workspace is not linear in the batch (the segmented
// scan picks its segment count from the batch, and its segment states grow with it),
// so the slice is sized by asking ss2d_forward_core_workspace for the exact image count:
// the largest count, at most `left`, whose workspace fits the static array.  0 if not
// even one image fits.
static int next_slice_images(const ss2d_core_args *args, int left)
{
    ss2d_core_args q = *args;
    // every image needs at least its x_dbl block, so no slice holds more than this
    const size_t xdbl_img = (size_t)4 * (q.R + 2 * q.N) * q.H * q.W * sizeof(float);
    const size_t hdr = ss2d::xproj_header_bytes();
    const size_t room = kStaticScratchBytes > hdr ? kStaticScratchBytes - hdr : 0;
    int n = (room / xdbl_img) < (size_t)left ? (int)(room / xdbl_img) : left;
    for (; n > 0; --n) {
        q.B = n;
        const size_t w = ss2d_forward_core_workspace(&q);
        if (w != (size_t)-1 && w <= kStaticScratchBytes)
            break;
    }
    return n;
}

int ss2d::static_slice_plan(const ss2d_core_args *args, int *nb, int max_slices)
{
    int slices = 0;
    for (int left = args->B; left > 0;) {
        const int n = next_slice_images(args, left);
        if (n == 0)
            return -1;
        if (nb && slices < max_slices)
            nb[slices] = n;
        ++slices;
        left -= n;
    }
    return slices;
}

extern "C" int ss2d_forward_core_static(const ss2d_core_args *args, void *stream)
{
    ss2d::set_last_error(SS2D_OK, "");
    // Same argument checks as ss2d_forward_core.
    const int st = ss2d::validate_core_args(args);
    if (st != SS2D_OK)
        return st;
    if (!args->x_proj_weight)
        return static_fail(SS2D_ERR_UNSUPPORTED,
                           "ss2d_forward_core_static: only the projection form (x_proj_weight, dt_projs_weight) uses "
                           "scratch; call ss2d_forward_core for the dts/Bs/Cs form");
    const ss2d_core_args &a = *args;
    if (a.struct_size >= offsetof(ss2d_core_args, y_dtype) + sizeof(int) && a.y_dtype != SS2D_F32)
        return static_fail(SS2D_ERR_UNSUPPORTED, "ss2d_forward_core_static: y must be fp32");
    // The whole plan is checked before anything is enqueued.
    if (ss2d::static_slice_plan(args, nullptr, 0) < 0) {
        ss2d_core_args q = a;
        q.B = 1;
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "ss2d_forward_core_static: one image needs %zu bytes of scratch, more than the %zu-byte static "
                 "scratch",
                 ss2d_forward_core_workspace(&q), kStaticScratchBytes);
        return static_fail(SS2D_ERR_UNSUPPORTED, msg);
    }
    void *scratch = nullptr;
    cudaError_t e = ss2d::static_scratch_address(&scratch);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof(msg), "ss2d_forward_core_static: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        return static_fail(SS2D_ERR_CUDA, msg);
    }
    const size_t L = (size_t)a.H * a.W;
    const size_t x_img = (size_t)a.D * L * 2;  // bf16 x (the projection form takes bf16 x)
    const size_t y_img = (size_t)a.D * L * 4;
    cudaStream_t s = (cudaStream_t)stream;
    for (int b0 = 0; b0 < a.B;) {
        const int nb = next_slice_images(args, a.B - b0);
        ss2d_core_args q = a;
        q.B = nb;
        const size_t need = nb > 0 ? ss2d_forward_core_workspace(&q) : (size_t)-1;
        if (need == (size_t)-1 || need > kStaticScratchBytes)  // never enqueue a slice that overruns the array
            return static_fail(SS2D_ERR_UNSUPPORTED, "ss2d_forward_core_static: a slice does not fit the scratch");
        const void *xs = static_cast<const char *>(a.x) + (size_t)b0 * x_img;
        float *ys = reinterpret_cast<float *>(reinterpret_cast<char *>(a.y) + (size_t)b0 * y_img);
        e = ss2d::launch_core_with_projections(xs, a.x_proj_weight, a.dt_projs_weight, a.A_logs, a.Ds, a.dt_bias,
                                                   a.delta_softplus != 0, ys, scratch, nb, a.D, a.H, a.W, a.N, a.R,
                                                   ss2d::core_channels_last(args), b0 == 0, s);
        if (e != cudaSuccess) {
            char msg[256];
            snprintf(msg, sizeof(msg), "ss2d_forward_core_static launch: %s", cudaGetErrorString(e));
            return static_fail(SS2D_ERR_CUDA, msg);
        }
        b0 += nb;
    }
    return SS2D_OK;
}
