// Runs the permutation kernels of perm.cu (CrossScan, CrossMerge, the plane transposes and
// the bf16-pair transpose that also zeroes y) on the host: one std::thread per thread of
// each CTA, __syncthreads on a per-CTA barrier, each CTA's tiles in its own shared memory;
// built with AddressSanitizer and UBSan by tests/test_permutation_emulation.py.  The grids
// are the launchers'.
// Arguments: which B D H W dir
//   which 0 / 1: CrossScan of dir/x (B, D, H, W) fp32 / bf16 into dir/out (B, 4, D, H*W)
//   which 2:     CrossMerge of dir/x (B, 4, D, H*W) fp32 into dir/out (B, D, H, W)
//   which 3 / 4: every (H, W) plane of dir/x (B*D planes) transposed, fp32 / bf16 (32x32 tiles)
//   which 5:     the same for bf16 with H and W even (64x64 tiles of pairs); dir/y (B, D, H, W)
//                fp32 is read, zeroed by the kernel and written back
//   which 6:     the same for bf16 with H and W multiples of 8 (8x8 blocks in registers), y too
#include <string>
#include <vector>
#include "kernel_emu.h"
using namespace ss2d;
std::vector<unsigned char> rd(const std::string &f, size_t n)
{
    std::vector<unsigned char> v(n);
    FILE *fp = fopen(f.c_str(), "rb");
    if (!fp || fread(v.data(), 1, n, fp) != n) { fprintf(stderr, "read %s\n", f.c_str()); exit(2); }
    fclose(fp);
    return v;
}
void wr(const std::string &f, const void *p, size_t n)
{
    FILE *fo = fopen(f.c_str(), "wb");
    fwrite(p, 1, n, fo);
    fclose(fo);
}
int main(int argc, char **argv)
{
    if (argc < 7) return 1;
    const int which = atoi(argv[1]), B = atoi(argv[2]), D = atoi(argv[3]), H = atoi(argv[4]), W = atoi(argv[5]);
    const std::string dir = argv[6];
    const size_t L = (size_t)H * W, planes = (size_t)B * D;
    const int esz = (which == 1 || which == 4 || which == 5 || which == 6) ? 2 : 4;
    const size_t in_elems = which == 2 ? 4 * planes * L : planes * L;
    const size_t out_elems = which <= 1 ? 4 * planes * L : planes * L;
    auto x = rd(dir + "/x", in_elems * esz);
    std::vector<unsigned char> out(out_elems * esz, 0xEE);
    const int tw = (W + kTile - 1) / kTile, th = (H + kTile - 1) / kTile;
    const size_t tile_bytes = (size_t)kTile * (kTile + 1) * esz;
    switch (which) {
    case 0:
        emu_grid(planes, tw * th, kTile * kRows, tile_bytes, [&] {
            cross_scan_kernel<float>((const float *)x.data(), (float *)out.data(), D, H, W, tw); });
        break;
    case 1:
        emu_grid(planes, tw * th, kTile * kRows, tile_bytes, [&] {
            cross_scan_kernel<__nv_bfloat16>((const __nv_bfloat16 *)x.data(), (__nv_bfloat16 *)out.data(), D, H, W,
                                             tw); });
        break;
    case 2:
        emu_grid(planes, tw * th, kTile * kRows, 2 * tile_bytes, [&] {
            cross_merge_kernel((const float *)x.data(), (float *)out.data(), D, H, W, tw); });
        break;
    case 3:
        emu_grid(planes, tw * th, kTile * kRows, tile_bytes, [&] {
            transpose_planes_kernel<float>((const float *)x.data(), (float *)out.data(), H, W, tw); });
        break;
    case 4:
        emu_grid(planes, tw * th, kTile * kRows, tile_bytes, [&] {
            transpose_planes_kernel<__nv_bfloat16>((const __nv_bfloat16 *)x.data(), (__nv_bfloat16 *)out.data(), H,
                                                   W, tw); });
        break;
    case 5: {
        if (H % 2 || W % 2) return 1;
        auto y = rd(dir + "/y", planes * L * 4);
        const int tw2 = (W + kT2 - 1) / kT2, th2 = (H + kT2 - 1) / kT2;
        emu_grid(planes, tw2 * th2, 256, (size_t)kT2 * (kT2 / 2 + 1) * 4, [&] {
            transpose_planes_pairs_kernel((const uint32_t *)x.data(), (uint32_t *)out.data(), H, W, tw2,
                                          (float *)y.data()); });
        wr(dir + "/y", y.data(), y.size());
        break;
    }
    case 6: {
        if (H % 8 || W % 8) return 1;
        auto y = rd(dir + "/y", planes * L * 4);
        const long long nb = (long long)planes * (H / 8) * (W / 8);
        emu_grid((unsigned)((nb + kB8Threads - 1) / kB8Threads), 1, kB8Threads, 0, [&] {
            transpose_planes_b8_kernel((const uint4 *)x.data(), (uint4 *)out.data(), H, W, nb, (float *)y.data()); });
        wr(dir + "/y", y.data(), y.size());
        break;
    }
    default: return 1;
    }
    wr(dir + "/out", out.data(), out.size());
    return 0;
}
