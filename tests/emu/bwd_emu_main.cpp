// Runs the backward kernels' source on the host (one std::thread per lane) over raw input
// files and writes the gradients; built with AddressSanitizer and UBSan by
// tests/test_backward_kernel_emulation.py.  Arguments: B D H W bf16(0/1) dir [nseg seg_len].
#include <thread>
#include <vector>
#include <string>
#include "kernel_emu.h"
using namespace ss2d;
template <class T> std::vector<T> rd(const std::string &f, size_t n)
{
    std::vector<T> v(n);
    FILE *fp = fopen(f.c_str(), "rb");
    if (!fp || fread(v.data(), sizeof(T), n, fp) != n) { fprintf(stderr, "read %s\n", f.c_str()); exit(2); }
    fclose(fp);
    return v;
}
template <class T> void wr(const std::string &f, const std::vector<T> &v)
{
    FILE *fp = fopen(f.c_str(), "wb"); fwrite(v.data(), sizeof(T), v.size(), fp); fclose(fp);
}
template <int DT>
void run(int B, int D, int H, int W, const std::string &dir, int nseg, int seg_len)
{
    using S = BwdShape<DT>;
    const int L = H * W, C = 4 * D, N = 16, nck = (L + 15) / 16, esz = (DT & 1) ? 2 : 4;
    auto x = rd<unsigned char>(dir + "/x", (size_t)B * D * L * esz);
    auto xT = rd<unsigned char>(dir + "/xT", (size_t)B * D * L * esz);
    auto dts = rd<unsigned char>(dir + "/dts", (size_t)B * C * L * esz);
    auto A = rd<float>(dir + "/A", (size_t)C * N);
    auto Bm = rd<float>(dir + "/Bm", (size_t)B * 4 * N * L), Cm = rd<float>(dir + "/Cm", (size_t)B * 4 * N * L);
    auto Dv = rd<float>(dir + "/Dv", C), bias = rd<float>(dir + "/bias", C);
    auto ckpt = rd<float>(dir + "/ckpt", (size_t)B * C * nck * N);
    auto dy = rd<float>(dir + "/dy", (size_t)B * D * L), dyT = rd<float>(dir + "/dyT", (size_t)B * D * L);
    std::vector<float> dx((size_t)B * D * L), ddts((size_t)B * C * L), dA((size_t)C * N), dB(Bm.size()), dC(Bm.size()), dD(C), db(C);
    BwdArgs a{};
    a.x = x.data(); a.xT = xT.data(); a.dts = dts.data(); a.A_log = A.data(); a.Bm = Bm.data(); a.Cm = Cm.data();
    a.Dv = Dv.data(); a.bias = bias.data(); a.ckpt = ckpt.data(); a.dy = dy.data(); a.dyT = dyT.data();
    a.dx = dx.data(); a.ddts = ddts.data(); a.dA_log = dA.data(); a.dBm = dB.data(); a.dCm = dC.data(); a.dDv = dD.data(); a.dbias = db.data();
    a.B = B; a.D = D; a.W = W; a.L = L; a.C = C; a.nck = nck; a.divH = {H, 1.0f / (float)H}; a.tiles = (D + S::CW - 1) / S::CW;
    const BwdLayout lay = S::layout();
    a.nseg = nseg; a.seg_len = seg_len;
    const int items = a.tiles * 4 * B * nseg;
    std::vector<float> eo((size_t)B * C * nseg * N, 0.f), po(eo.size(), 0.f), gi(eo.size(), 0.f);
    auto launch = [&](bool carry) {
    for (int blk = 0; blk < items; ++blk) {
        WarpCtx ctx;
        std::vector<unsigned char> smem(lay.smem_bytes);
        ctx.smem = smem.data();
        ctx.smem_bytes = lay.smem_bytes;
        std::vector<std::thread> th;
        for (int lane = 0; lane < 32; ++lane)
            th.emplace_back([&, lane] {
                threadIdx = {(unsigned)lane, 0, 0};
                blockIdx = {(unsigned)blk, 0, 0};
                g_warp = &ctx;
                g_lane = lane;
                if (carry) adjoint_carry_kernel<S>(a, lay); else scan_bwd_kernel<S>(a, lay);
            });
        for (auto &t : th) t.join();
    }
    };
    if (nseg > 1) {
        a.e_out = eo.data(); a.p_out = po.data(); a.g_in = gi.data();
        launch(true);
        // carry-in, from the last segment down, in the launcher's grid
        const long long total = (long long)B * C * N;
        emu_grid((unsigned)((total + 255) / 256), 1, 256, 0,
                 [&] { adjoint_carry_in_kernel(eo.data(), po.data(), gi.data(), total, nseg, N); });
    }
    launch(false);
    wr(dir + "/out_dx", dx); wr(dir + "/out_ddts", ddts); wr(dir + "/out_dA", dA); wr(dir + "/out_dB", dB);
    wr(dir + "/out_dC", dC); wr(dir + "/out_dD", dD); wr(dir + "/out_db", db);
    printf("emulated %d CTAs, smem %d\n", items, lay.smem_bytes);
}
int main(int argc, char **argv)
{
    if (argc < 7) return 1;
    const int B = atoi(argv[1]), D = atoi(argv[2]), H = atoi(argv[3]), W = atoi(argv[4]), bf = atoi(argv[5]);
    const int nseg = argc > 7 ? atoi(argv[7]) : 1, seg_len = argc > 8 ? atoi(argv[8]) : H * W;
    if (bf) run<7>(B, D, H, W, argv[6], nseg, seg_len); else run<4>(B, D, H, W, argv[6], nseg, seg_len);
    return 0;
}
