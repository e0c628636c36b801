// perm.cu -- CrossScan and CrossMerge as standalone kernels.
//
// Both work on 32x32 pixel tiles of one (b, d) plane staged in shared memory,
// so that every global read and write is contiguous along the innermost
// index of its own tensor: rows of x for the row-major orders, and runs of
// consecutive scan steps (down a column of x) for the column-major orders.
#include "common.cuh"
#include "kernels.h"

namespace ss2d {

namespace {

constexpr int kTile = 32;
constexpr int kRows = 8;  // threads per tile column; each covers kTile/kRows rows

// CrossScan, SS2D article section 3.1: xs[b,k,d,l] = x[b,d,pi_k(l)].
template <typename T>
__global__ void __launch_bounds__(kTile *kRows) cross_scan_kernel(const T *__restrict__ x, T *__restrict__ xs,
                                                                   int D, int H, int W, int tiles_w)
{
    __shared__ T tile[kTile][kTile + 1];
    const int plane = blockIdx.x;  // b*D + d
    const int b = plane / D;
    const int d = plane % D;
    const int h0 = (blockIdx.y / tiles_w) * kTile;
    const int w0 = (blockIdx.y % tiles_w) * kTile;
    const int L = H * W;
    const T *src = x + (size_t)plane * L;
    const size_t dir_stride = (size_t)D * L;
    T *dst0 = xs + ((size_t)b * 4 * D + d) * L;
    T *dst1 = dst0 + dir_stride;
    T *dst2 = dst1 + dir_stride;
    T *dst3 = dst2 + dir_stride;
    const int tx = threadIdx.x % kTile;
    const int ty = threadIdx.x / kTile;

#pragma unroll
    for (int r = 0; r < kTile; r += kRows) {
        const int h = h0 + ty + r, w = w0 + tx;
        if (h < H && w < W) {
            const T v = src[(size_t)h * W + w];
            tile[ty + r][tx] = v;
            const int p = h * W + w;
            dst0[p] = v;              // row-major
            dst2[L - 1 - p] = v;      // reverse row-major
        }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kTile; r += kRows) {
        const int h = h0 + tx, w = w0 + ty + r;  // consecutive threads walk down a column
        if (h < H && w < W) {
            const T v = tile[tx][ty + r];
            const int l = w * H + h;
            dst1[l] = v;              // column-major
            dst3[L - 1 - l] = v;      // reverse column-major
        }
    }
}

// CrossMerge, SS2D article section 3.3:
// y[b,d,p] = ((ys0[p] + ys2[L-1-p]) + ys1[w*H+h]) + ys3[L-1-(w*H+h)].
__global__ void __launch_bounds__(kTile *kRows) cross_merge_kernel(const float *__restrict__ ys, float *__restrict__ y,
                                                                    int D, int H, int W, int tiles_w)
{
    __shared__ float t1[kTile][kTile + 1];
    __shared__ float t3[kTile][kTile + 1];
    const int plane = blockIdx.x;
    const int b = plane / D;
    const int d = plane % D;
    const int h0 = (blockIdx.y / tiles_w) * kTile;
    const int w0 = (blockIdx.y % tiles_w) * kTile;
    const int L = H * W;
    const size_t dir_stride = (size_t)D * L;
    const float *ys0 = ys + ((size_t)b * 4 * D + d) * L;
    const float *ys1 = ys0 + dir_stride;
    const float *ys2 = ys1 + dir_stride;
    const float *ys3 = ys2 + dir_stride;
    const int tx = threadIdx.x % kTile;
    const int ty = threadIdx.x / kTile;

#pragma unroll
    for (int r = 0; r < kTile; r += kRows) {
        const int h = h0 + tx, w = w0 + ty + r;
        if (h < H && w < W) {
            const int l = w * H + h;
            t1[ty + r][tx] = ys1[l];
            t3[ty + r][tx] = ys3[L - 1 - l];
        }
    }
    __syncthreads();
    float *dst = y + (size_t)plane * L;
#pragma unroll
    for (int r = 0; r < kTile; r += kRows) {
        const int h = h0 + ty + r, w = w0 + tx;
        if (h < H && w < W) {
            const int p = h * W + w;
            float v = ys0[p] + ys2[L - 1 - p];
            v = v + t1[tx][ty + r];
            v = v + t3[tx][ty + r];
            dst[p] = v;
        }
    }
}

// Transpose of every (H, W) plane: xT[plane, w*H + h] = x[plane, h*W + w], i.e. the
// planes in the visiting order of the column-major scan (direction 1 of CrossScan).
template <typename T>
__global__ void __launch_bounds__(kTile *kRows) transpose_planes_kernel(const T *__restrict__ x, T *__restrict__ xT,
                                                                         int H, int W, int tiles_w)
{
    __shared__ T tile[kTile][kTile + 1];
    const size_t plane = blockIdx.x;
    const int h0 = (blockIdx.y / tiles_w) * kTile;
    const int w0 = (blockIdx.y % tiles_w) * kTile;
    const size_t L = (size_t)H * W;
    const T *src = x + plane * L;
    T *dst = xT + plane * L;
    const int tx = threadIdx.x % kTile;
    const int ty = threadIdx.x / kTile;
#pragma unroll
    for (int r = 0; r < kTile; r += kRows) {
        const int h = h0 + ty + r, w = w0 + tx;
        if (h < H && w < W)
            tile[ty + r][tx] = src[(size_t)h * W + w];
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kTile; r += kRows) {
        const int h = h0 + tx, w = w0 + ty + r;
        if (h < H && w < W)
            dst[(size_t)w * H + h] = tile[tx][ty + r];
    }
}

// The same transpose for 2-byte elements with H and W even, on 64x64 tiles moved as
// 4-byte pairs: a thread reads the pairs (w, w+1) of rows h and h+1, regroups them into
// the pairs (h, h+1) of columns w and w+1, and the tile is written back one column pair
// per thread, so every global access is a 4-byte word in a 128-byte warp-wide run.
constexpr int kT2 = 64;
__global__ void __launch_bounds__(256) transpose_planes_pairs_kernel(const uint32_t *__restrict__ x,
                                                                      uint32_t *__restrict__ xT, int H, int W,
                                                                      int tiles_w, float *__restrict__ y_zero)
{
    __shared__ uint32_t t[kT2][kT2 / 2 + 1];  // t[w][h/2] = (x[h][w], x[h+1][w])
    const size_t plane = blockIdx.x;
    const int h0 = (blockIdx.y / tiles_w) * kT2;
    const int w0 = (blockIdx.y % tiles_w) * kT2;
    const size_t half_l = (size_t)H * W / 2;  // words per plane
    const uint32_t *src = x + plane * half_l;
    uint32_t *dst = xT + plane * half_l;
    const int lane = threadIdx.x % 32;
    const int warp = threadIdx.x / 32;
    const int w = w0 + 2 * lane;  // this thread's column pair (w, w+1)
#pragma unroll
    for (int r = 0; r < kT2 / 2; r += 8) {
        const int hp = warp + r;  // row pair (h, h+1) = (h0 + 2hp, h0 + 2hp + 1)
        const int h = h0 + 2 * hp;
        if (h < H && w < W) {
            const uint32_t a = src[((size_t)h * W + w) / 2];        // (x[h][w],   x[h][w+1])
            const uint32_t b = src[((size_t)(h + 1) * W + w) / 2];  // (x[h+1][w], x[h+1][w+1])
            t[2 * lane][hp] = __byte_perm(a, b, 0x5410);            // (x[h][w],   x[h+1][w])
            t[2 * lane + 1][hp] = __byte_perm(a, b, 0x7632);        // (x[h][w+1], x[h+1][w+1])
        }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kT2; r += 8) {
        const int wl = warp + r;
        const int ww = w0 + wl, hh = h0 + 2 * lane;
        if (ww < W && hh < H)
            dst[((size_t)ww * H + hh) / 2] = t[wl][lane];
    }
    if (y_zero) {
        // the same (h, w) tile of the (H, W) plane of y set to zero, ready for the merge's adds:
        // 16-byte stores when the rows start on 16-byte boundaries (W % 4 == 0; w0 is a multiple
        // of 64), else one float per thread
        float *yp = y_zero + plane * 2 * half_l;
        if ((W & 3) == 0) {
            for (int idx = threadIdx.x; idx < kT2 * (kT2 / 4); idx += 256) {
                const int h = h0 + idx / (kT2 / 4), w = w0 + 4 * (idx % (kT2 / 4));
                if (h < H && w < W)
                    *reinterpret_cast<float4 *>(yp + (size_t)h * W + w) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        } else {
            for (int idx = threadIdx.x; idx < kT2 * kT2; idx += 256) {
                const int h = h0 + idx / kT2, w = w0 + idx % kT2;
                if (h < H && w < W)
                    yp[(size_t)h * W + w] = 0.0f;
            }
        }
    }
}

// The same transpose for 2-byte elements with H and W multiples of 8, without shared memory:
// a thread moves one 8x8 block, eight 16-byte row pieces in, regrouped in registers into
// 32-bit pairs of consecutive rows (word p of column c holds rows 2p and 2p+1), eight 16-byte
// column pieces out (faster than the 64x64 pair kernel on 56x56 planes).  With y_zero, the
// block's 8x8 square of the fp32 plane of y is zeroed too.
constexpr int kB8Threads = 256;
__global__ void __launch_bounds__(kB8Threads) transpose_planes_b8_kernel(const uint4 *__restrict__ x,
                                                                         uint4 *__restrict__ xT, int H, int W,
                                                                         long long nblocks, float *__restrict__ y_zero)
{
    const long long t = (long long)blockIdx.x * kB8Threads + threadIdx.x;
    if (t >= nblocks)
        return;
    const int WB = W / 8, HB = H / 8;
    const int wb = (int)(t % WB);
    const long long r = t / WB;
    const int hb = (int)(r % HB);
    const size_t plane = (size_t)(r / HB);
    const size_t L = (size_t)H * W;
    const int h0 = 8 * hb, w0 = 8 * wb;
    const uint4 *src = x + (plane * L + (size_t)h0 * W + w0) / 8;
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        v[i] = __ldg(src + (size_t)i * (W / 8));
    uint32_t o[8][4];  // o[c][p] = (x[h0+2p][w0+c], x[h0+2p+1][w0+c])
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint4 a = v[2 * p], b = v[2 * p + 1];
        o[0][p] = __byte_perm(a.x, b.x, 0x5410);
        o[1][p] = __byte_perm(a.x, b.x, 0x7632);
        o[2][p] = __byte_perm(a.y, b.y, 0x5410);
        o[3][p] = __byte_perm(a.y, b.y, 0x7632);
        o[4][p] = __byte_perm(a.z, b.z, 0x5410);
        o[5][p] = __byte_perm(a.z, b.z, 0x7632);
        o[6][p] = __byte_perm(a.w, b.w, 0x5410);
        o[7][p] = __byte_perm(a.w, b.w, 0x7632);
    }
    uint4 *dst = xT + (plane * L + (size_t)w0 * H + h0) / 8;
#pragma unroll
    for (int c = 0; c < 8; ++c)
        dst[(size_t)c * (H / 8)] = make_uint4(o[c][0], o[c][1], o[c][2], o[c][3]);
    if (y_zero) {
        float4 *yp = reinterpret_cast<float4 *>(y_zero + plane * L + (size_t)h0 * W + w0);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            yp[(size_t)i * (W / 4)] = make_float4(0.f, 0.f, 0.f, 0.f);
            yp[(size_t)i * (W / 4) + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
}

// bf16 -> fp32, eight elements per 16-byte load, written as two 16-byte stores (both buffers
// are 16-byte aligned).  A thread issues the loads of four such pieces, a grid stride apart,
// before it stores any, so that four loads per thread are in flight; then the tail of fewer
// than eight elements one by one.
__device__ __forceinline__ void widen8(float4 *d, uint4 v)
{
    d[0] = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u), __uint_as_float(v.y << 16),
                       __uint_as_float(v.y & 0xFFFF0000u));
    d[1] = make_float4(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xFFFF0000u), __uint_as_float(v.w << 16),
                       __uint_as_float(v.w & 0xFFFF0000u));
}

__global__ void bf16_to_f32_kernel(const __nv_bfloat16 *__restrict__ src, float *__restrict__ dst, size_t n)
{
    constexpr int kU = 4;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    const size_t n8 = n / 8;
    const uint4 *s8 = reinterpret_cast<const uint4 *>(src);
    float4 *d4 = reinterpret_cast<float4 *>(dst);
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; i + (kU - 1) * stride < n8; i += kU * stride) {
        uint4 v[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u)
            v[u] = __ldg(s8 + i + u * stride);
#pragma unroll
        for (int u = 0; u < kU; ++u)
            widen8(d4 + 2 * (i + u * stride), v[u]);
    }
    for (; i < n8; i += stride)
        widen8(d4 + 2 * i, __ldg(s8 + i));
    for (size_t j = n8 * 8 + (size_t)blockIdx.x * blockDim.x + threadIdx.x; j < n; j += stride)
        dst[j] = __bfloat162float(src[j]);
}

__global__ void f32_to_bf16_kernel(const float *__restrict__ src, __nv_bfloat16 *__restrict__ dst, size_t n)
{
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        dst[i] = __float2bfloat16_rn(src[i]);
}

__global__ void fill_zero_kernel(float *__restrict__ p, size_t n)
{
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    const size_t n4 = n / 4;
    float4 *p4 = reinterpret_cast<float4 *>(p);
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride)
        p4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (size_t i = n4 * 4 + (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        p[i] = 0.f;
}

// The page-order CrossMerge of four per-direction outputs (SS2D article, section 3.3: y0 +
// inv_y0 + wh_y + invwh_y, added left to right): y = ((y + y2) + y1) + y3 with y holding
// direction 0's output on entry.  All four are laid out alike, so the sum is element-wise.
__global__ void page_order_sum_kernel(float *__restrict__ y, const float *__restrict__ y1,
                                      const float *__restrict__ y2, const float *__restrict__ y3, size_t n)
{
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    const size_t n4 = n / 4;
    float4 *o4 = reinterpret_cast<float4 *>(y);
    const float4 *a4 = reinterpret_cast<const float4 *>(y1), *b4 = reinterpret_cast<const float4 *>(y2),
                 *c4 = reinterpret_cast<const float4 *>(y3);
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
        const float4 v0 = o4[i], v1 = __ldg(a4 + i), v2 = __ldg(b4 + i), v3 = __ldg(c4 + i);
        o4[i] = make_float4(__fadd_rn(__fadd_rn(__fadd_rn(v0.x, v2.x), v1.x), v3.x),
                            __fadd_rn(__fadd_rn(__fadd_rn(v0.y, v2.y), v1.y), v3.y),
                            __fadd_rn(__fadd_rn(__fadd_rn(v0.z, v2.z), v1.z), v3.z),
                            __fadd_rn(__fadd_rn(__fadd_rn(v0.w, v2.w), v1.w), v3.w));
    }
    for (size_t i = n4 * 4 + (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        y[i] = __fadd_rn(__fadd_rn(__fadd_rn(y[i], y2[i]), y1[i]), y3[i]);
}

}  // namespace

cudaError_t launch_cross_scan(const void *x, bool bf16, void *xs, int B, int D, int H, int W, cudaStream_t s)
{
    const int tiles_w = (W + kTile - 1) / kTile;
    const int tiles_h = (H + kTile - 1) / kTile;
    dim3 grid(B * D, tiles_w * tiles_h);
    if (bf16)
        cross_scan_kernel<__nv_bfloat16><<<grid, kTile * kRows, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(xs), D, H, W, tiles_w);
    else
        cross_scan_kernel<float><<<grid, kTile * kRows, 0, s>>>(static_cast<const float *>(x),
                                                               static_cast<float *>(xs), D, H, W, tiles_w);
    return cudaGetLastError();
}

cudaError_t launch_cross_merge(const float *ys, float *y, int B, int D, int H, int W, cudaStream_t s)
{
    const int tiles_w = (W + kTile - 1) / kTile;
    const int tiles_h = (H + kTile - 1) / kTile;
    dim3 grid(B * D, tiles_w * tiles_h);
    cross_merge_kernel<<<grid, kTile * kRows, 0, s>>>(ys, y, D, H, W, tiles_w);
    return cudaGetLastError();
}

cudaError_t launch_transpose_planes(const void *x, bool bf16, void *xT, int planes, int H, int W, cudaStream_t s)
{
    const int tiles_w = (W + kTile - 1) / kTile;
    const int tiles_h = (H + kTile - 1) / kTile;
    if (planes <= 0 || (long long)tiles_w * tiles_h > 65535)
        return cudaErrorInvalidConfiguration;
    if (bf16 && H % 8 == 0 && W % 8 == 0) {
        const long long nb = (long long)planes * (H / 8) * (W / 8);
        transpose_planes_b8_kernel<<<(unsigned)((nb + kB8Threads - 1) / kB8Threads), kB8Threads, 0, s>>>(
            static_cast<const uint4 *>(x), static_cast<uint4 *>(xT), H, W, nb, nullptr);
        return cudaGetLastError();
    }
    if (bf16 && H % 2 == 0 && W % 2 == 0) {
        const int tw = (W + kT2 - 1) / kT2, th = (H + kT2 - 1) / kT2;
        transpose_planes_pairs_kernel<<<dim3(planes, tw * th), 256, 0, s>>>(
            static_cast<const uint32_t *>(x), static_cast<uint32_t *>(xT), H, W, tw, nullptr);
        return cudaGetLastError();
    }
    dim3 grid(planes, tiles_w * tiles_h);
    if (bf16)
        transpose_planes_kernel<__nv_bfloat16><<<grid, kTile * kRows, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(xT), H, W, tiles_w);
    else
        transpose_planes_kernel<float><<<grid, kTile * kRows, 0, s>>>(static_cast<const float *>(x),
                                                                     static_cast<float *>(xT), H, W, tiles_w);
    return cudaGetLastError();
}

bool transpose_planes_can_zero(bool bf16, int H, int W) { return bf16 && H % 2 == 0 && W % 2 == 0; }

cudaError_t launch_transpose_planes_zero(const void *x, void *xT, float *y_zero, int planes, int H, int W,
                                         cudaStream_t s)
{
    const int tw = (W + kT2 - 1) / kT2, th = (H + kT2 - 1) / kT2;
    if (planes <= 0 || !transpose_planes_can_zero(true, H, W) || (long long)tw * th > 65535)
        return cudaErrorInvalidValue;
    // the pair kernel: with the zero fill it measured as fast as the 8x8 kernel
    transpose_planes_pairs_kernel<<<dim3(planes, tw * th), 256, 0, s>>>(
        static_cast<const uint32_t *>(x), static_cast<uint32_t *>(xT), H, W, tw, y_zero);
    return cudaGetLastError();
}

cudaError_t launch_bf16_to_f32(const void *src, float *dst, size_t n, cudaStream_t s)
{
    size_t want = (n / 8 + 255) / 256;
    int blocks = (int)(want < (size_t)148 * 16 ? want : (size_t)148 * 16);
    if (blocks < 1)
        blocks = 1;
    bf16_to_f32_kernel<<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(src), dst, n);
    return cudaGetLastError();
}

cudaError_t launch_f32_to_bf16(const float *src, void *dst, size_t n, cudaStream_t s)
{
    size_t want = (n + 255) / 256;
    int blocks = (int)(want < (size_t)148 * 16 ? want : (size_t)148 * 16);
    if (blocks < 1)
        blocks = 1;
    f32_to_bf16_kernel<<<blocks, 256, 0, s>>>(src, static_cast<__nv_bfloat16 *>(dst), n);
    return cudaGetLastError();
}

cudaError_t launch_page_order_sum(float *y, const float *y1, const float *y2, const float *y3, size_t n, cudaStream_t s)
{
    // all four 16-byte aligned (workspace parts at 256-byte offsets, y checked by the caller)
    size_t want = (n / 4 + 255) / 256;
    int blocks = (int)(want < (size_t)148 * 16 ? want : (size_t)148 * 16);
    if (blocks < 1)
        blocks = 1;
    page_order_sum_kernel<<<blocks, 256, 0, s>>>(y, y1, y2, y3, n);
    return cudaGetLastError();
}

cudaError_t launch_fill_zero(float *p, size_t n, cudaStream_t s)
{
    // p is 16-byte aligned (checked by the caller).
    size_t want = (n / 4 + 255) / 256;
    int blocks = (int)(want < (size_t)148 * 16 ? want : (size_t)148 * 16);
    if (blocks < 1)
        blocks = 1;
    fill_zero_kernel<<<blocks, 256, 0, s>>>(p, n);
    return cudaGetLastError();
}

}  // namespace ss2d
