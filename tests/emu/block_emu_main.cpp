// Runs the SS2D block's CUDA-core kernels of block.cu (the depthwise convolution with SiLU and
// the gated LayerNorm) on the host: one std::thread per thread of each CTA, __syncthreads on a
// per-CTA barrier, each CTA's shared memory in its own buffer; built with AddressSanitizer and
// UBSan by tests/test_block_kernel_emulation.py.  The grids and shared-memory sizes are the
// launchers'.
// Arguments: which B H W D dir [k]
//   which 0: dwconv_silu_kernel<k> on dir/xz ((B*H*W, 2D) bf16) with dir/w ((D, k, k) fp32) and
//            dir/bias ((D) fp32) into dir/out ((B, D, H, W) bf16)
//   which 1 / 2: norm_gate_kernel<true / false> on dir/y ((B, D, H*W) fp32) and the z half of
//            dir/xz, with dir/gamma, dir/beta ((D) fp32) and eps 1e-5, into dir/out ((B*H*W, D) bf16)
//   which 3: as 0, channels-last out (dir/out (B, H, W, D) bf16)
//   which 4: norm_gate_cl_kernel on channels-last dir/y ((B*H*W, D) fp32), otherwise as 1
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
template <int KS>
void run_conv(const ConvArgs &c)
{
    const unsigned blocks = (unsigned)((long long)c.B * c.tiles_h * c.tiles_w * c.tiles_c);
    if (c.cl_out)
        emu_grid(blocks, 1, kCvThreads, cv_smem_bytes(KS), [&] { dwconv_silu_kernel<KS, true>(c); });
    else
        emu_grid(blocks, 1, kCvThreads, cv_smem_bytes(KS), [&] { dwconv_silu_kernel<KS, false>(c); });
}
template <int NPL>
void run_norm_cl(const NormArgs &n)
{
    const long long pixels = (long long)n.B * n.L;
    emu_grid((unsigned)((pixels + kNgThreads / 32 - 1) / (kNgThreads / 32)), 1, kNgThreads, 0,
             [&] { norm_gate_cl_kernel<NPL>(n); });
}
int main(int argc, char **argv)
{
    if (argc < 7) return 1;
    const int which = atoi(argv[1]), B = atoi(argv[2]), H = atoi(argv[3]), W = atoi(argv[4]), D = atoi(argv[5]);
    const std::string dir = argv[6];
    const int k = argc > 7 ? atoi(argv[7]) : 3;
    const size_t L = (size_t)H * W, M = (size_t)B * L;
    auto xz = rd(dir + "/xz", M * 2 * D * 2);
    if (which == 0 || which == 3) {
        auto w = rd(dir + "/w", (size_t)D * k * k * 4);
        auto bias = rd(dir + "/bias", (size_t)D * 4);
        std::vector<unsigned char> out(M * D * 2, 0xEE);
        ConvArgs c{};
        c.xz = (const __nv_bfloat16 *)xz.data();
        c.w = (const float *)w.data();
        c.bias = (const float *)bias.data();
        c.xc = (__nv_bfloat16 *)out.data();
        c.B = B;
        c.D = D;
        c.H = H;
        c.W = W;
        c.ldx = 2 * D;
        c.tiles_h = (H + kCvTH - 1) / kCvTH;
        c.tiles_w = (W + kCvTW - 1) / kCvTW;
        c.tiles_c = (D + kCvTC - 1) / kCvTC;
        c.cl_out = which == 3;
        switch (k) {
        case 1: run_conv<1>(c); break;
        case 3: run_conv<3>(c); break;
        case 5: run_conv<5>(c); break;
        case 7: run_conv<7>(c); break;
        default: return 1;
        }
        wr(dir + "/out", out.data(), out.size());
        return 0;
    }
    auto y = rd(dir + "/y", M * D * 4);
    auto gamma = rd(dir + "/gamma", (size_t)D * 4);
    auto beta = rd(dir + "/beta", (size_t)D * 4);
    std::vector<unsigned char> out(M * D * 2, 0xEE);
    NormArgs n{};
    n.y = (const float *)y.data();
    n.z = (const __nv_bfloat16 *)xz.data() + D;
    n.gamma = (const float *)gamma.data();
    n.beta = (const float *)beta.data();
    n.g = (__nv_bfloat16 *)out.data();
    n.eps = 1e-5f;
    n.B = B;
    n.D = D;
    n.L = (int)L;
    n.ldz = 2 * D;
    n.tiles_l = (int)((L + kNgP - 1) / kNgP);
    const unsigned blocks = (unsigned)((long long)B * n.tiles_l);
    if (which == 4) {
        const int npl = (D / 2 + 31) / 32;
        if (npl <= 1) run_norm_cl<1>(n);
        else if (npl <= 2) run_norm_cl<2>(n);
        else if (npl <= 3) run_norm_cl<3>(n);
        else if (npl <= 4) run_norm_cl<4>(n);
        else if (npl <= 6) run_norm_cl<6>(n);
        else if (npl <= 8) run_norm_cl<8>(n);
        else if (npl <= kNgClMaxPairs) run_norm_cl<kNgClMaxPairs>(n);
        else return 1;
    } else if (which == 1)
        emu_grid(blocks, 1, kNgThreads, ng_smem_bytes(D, true), [&] { norm_gate_kernel<true>(n); });
    else
        emu_grid(blocks, 1, kNgThreads, ng_smem_bytes(D, false), [&] { norm_gate_kernel<false>(n); });
    wr(dir + "/out", out.data(), out.size());
    return 0;
}
