// Runs the forward scan kernel's source (scan2_kernel, the fused N = 16 core) on the host, one
// std::thread per lane, over raw input files and writes y; built with AddressSanitizer and
// UBSan by tests/test_forward_kernel_emulation.py.
// Arguments: B D H W bf16(0/1; 2 = bf16 u, fp32 dts) channels_last(0/1) dir nseg seg_len
//            [keep_checkpoints(0/1/2) [R [page(0/1)]]]
// With R > 0 the kernel runs its projection mode: dt_low, B and C rows come from dir/xdbl,
// (B, 4, R+2N, L) fp32 in scan order, dt_proj's weights from dir/Wdt (4, D, R), and x is bf16.
// Channels-first x is read with its transposed-planes copy xT (column-major orders as rows);
// channels-last x is (B, H, W, D) and y is written in the same layout.  With nseg > 1 the
// first pass, the carry of the segment states (segment_carry_kernel) and the second pass run.  With
// keep_checkpoints the pass that produces y also stores the backward's checkpoints (SEGP 3),
// written to dir/ckpt as (B, 4D, ceil(L/16), 16) fp32.
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
template <int MODE, int DT, int SEGP, int CL>
void launch(const ScanArgs &a, int items)
{
    using S = Scan2Shape<MODE, DT, SEGP, CL>;
    const Scan2Layout lay = S::layout();
    for (int blk = 0; blk < items; ++blk) {
        WarpCtx ctx;
        std::vector<unsigned char> smem(lay.smem_bytes + 16);
        ctx.smem = smem.data() + (16 - ((uintptr_t)smem.data() & 15)) % 16;
        ctx.smem_bytes = lay.smem_bytes;
        memset(ctx.smem, 0xCD, lay.smem_bytes);
        std::vector<std::thread> th;
        for (int lane = 0; lane < 32; ++lane)
            th.emplace_back([&, lane] {
                threadIdx = {(unsigned)lane, 0, 0};
                blockIdx = {(unsigned)blk, 0, 0};
                g_warp = &ctx;
                g_lane = lane;
                scan2_kernel<S>(a, lay);
            });
        for (auto &t : th) t.join();
    }
}
// The pass that produces y: with checkpoints (keep 1; the direct form only, as in the library)
// or without; keep 2 is the backward's checkpoint pass, which stores the checkpoints alone.
template <int MODE, int DT, int CL>
void pass(const ScanArgs &a, int items, int keep)
{
    if constexpr (MODE == kFused) {
        if (keep == 1) {
            launch<MODE, DT, 3, CL>(a, items);
            return;
        }
        if (keep == 2) {
            launch<MODE, DT, 2, CL>(a, items);
            return;
        }
    }
    launch<MODE, DT, 0, CL>(a, items);
}
template <int MODE, int DT, int CL>
void run(int B, int D, int H, int W, const std::string &dir, int nseg, int seg_len, int keep, int R, bool page)
{
    const int L = H * W, C = 4 * D, N = 16, Cp = R + 2 * N;
    const int esz_u = (DT & 2) ? 2 : 4, esz_d = (DT & 1) ? 2 : 4;
    constexpr bool PROJ = MODE == kFusedProj;
    auto x = rd<unsigned char>(dir + "/x", (size_t)B * D * L * esz_u);
    std::vector<unsigned char> xT;
    if (!CL) xT = rd<unsigned char>(dir + "/xT", (size_t)B * D * L * esz_u);
    std::vector<unsigned char> dts;
    std::vector<float> Bm, Cm, xdbl, Wdt;
    if (PROJ) {
        xdbl = rd<float>(dir + "/xdbl", (size_t)B * 4 * Cp * L);
        Wdt = rd<float>(dir + "/Wdt", (size_t)C * R);
    } else {
        dts = rd<unsigned char>(dir + "/dts", (size_t)B * C * L * esz_d);
        Bm = rd<float>(dir + "/Bm", (size_t)B * 4 * N * L);
        Cm = rd<float>(dir + "/Cm", (size_t)B * 4 * N * L);
    }
    auto A = rd<float>(dir + "/A", (size_t)C * N);
    auto Dv = rd<float>(dir + "/Dv", C), bias = rd<float>(dir + "/bias", C);
    std::vector<float> y((size_t)B * D * L, 0.0f);
    std::vector<float> ck(keep ? (size_t)B * C * ((L + 15) / 16) * N : 0, -12345.0f);
    ScanArgs a{};
    a.u = x.data();
    a.uT = CL ? nullptr : xT.data();
    a.A_log = A.data(); a.Dv = Dv.data(); a.bias = bias.data(); a.y = y.data();
    if (PROJ) {  // as the projection path sets them up: rows of x_dbl
        a.delta = nullptr;
        a.dtl = xdbl.data();
        a.Bm = xdbl.data() + (size_t)R * L;
        a.Cm = xdbl.data() + (size_t)(R + N) * L;
        a.Wdt = Wdt.data();
        a.R = R;
        a.gs = (long long)Cp * L;
    } else {
        a.delta = dts.data();
        a.Bm = Bm.data();
        a.Cm = Cm.data();
        a.gs = (long long)N * L;
    }
    a.B = B; a.C = C; a.G = 4; a.L = L; a.per_group = D; a.W = W; a.divH = {H, 1.0f / (float)H};
    a.u_bf16 = (DT & 2) ? 1 : 0; a.delta_bf16 = (DT & 1) ? 1 : 0; a.softplus = 1; a.ch_last = CL;
    a.delta_bytes = dts.size();  // 0 in the projection mode, as the library passes it
    a.tiles = (D + 15) / 16;
    a.nseg = nseg; a.seg_len = seg_len;
    const int items = a.tiles * 4 * B * nseg;
    // page-order outputs: channel-first, the four directions in scan order (B, 4D, L); channels-
    // last, direction 0 into y and 1..3 into copies of y
    std::vector<float> ys, yb1, yb2, yb3;
    if (page) {
        if (CL) {
            yb1.assign(y.size(), -12345.0f);
            yb2 = yb1;
            yb3 = yb1;
            y.assign(y.size(), -12345.0f);
            a.ydir[0] = y.data(); a.ydir[1] = yb1.data(); a.ydir[2] = yb2.data(); a.ydir[3] = yb3.data();
        } else {
            ys.assign((size_t)B * C * L, -12345.0f);
            a.ydir[0] = ys.data();
        }
    }
    if (nseg > 1) {
        const size_t n = (size_t)B * C * nseg * N;
        std::vector<float> hend(n, 0.f), pend(n, 0.f), hin(n, 0.f);
        ScanArgs p1 = a;
        p1.hend = hend.data();
        p1.pend = pend.data();
        launch<MODE, DT, 1, CL>(p1, items);
        // carry of the segment states, in the launcher's grid
        const long long total = (long long)B * C * N;
        emu_grid((unsigned)((total + 255) / 256), 1, 256, 0,
                 [&] { segment_carry_kernel(hend.data(), pend.data(), hin.data(), total, nseg, N); });
        ScanArgs p2 = a;
        p2.h0 = hin.data();
        p2.ckpt = keep ? ck.data() : nullptr;
        pass<MODE, DT, CL>(p2, items, keep);
    } else {
        ScanArgs p = a;
        p.ckpt = keep ? ck.data() : nullptr;
        pass<MODE, DT, CL>(p, items, keep);
    }
    FILE *fo = fopen((dir + "/y").c_str(), "wb");
    fwrite(y.data(), 4, y.size(), fo);
    fclose(fo);
    if (keep) {
        fo = fopen((dir + "/ckpt").c_str(), "wb");
        fwrite(ck.data(), 4, ck.size(), fo);
        fclose(fo);
    }
    const std::vector<float> *extra[4] = {&ys, &yb1, &yb2, &yb3};
    const char *names[4] = {"/ys", "/yb1", "/yb2", "/yb3"};
    for (int k = 0; k < 4; ++k)
        if (!extra[k]->empty()) {
            fo = fopen((dir + names[k]).c_str(), "wb");
            fwrite(extra[k]->data(), 4, extra[k]->size(), fo);
            fclose(fo);
        }
}
int main(int argc, char **argv)
{
    if (argc < 10) return 1;
    const int B = atoi(argv[1]), D = atoi(argv[2]), H = atoi(argv[3]), W = atoi(argv[4]);
    const int bf = atoi(argv[5]), cl = atoi(argv[6]), nseg = atoi(argv[8]), seg_len = atoi(argv[9]);
    const std::string dir = argv[7];
    const int keep = argc > 10 ? atoi(argv[10]) : 0;
    const int R = argc > 11 ? atoi(argv[11]) : 0;
    const bool page = argc > 12 && atoi(argv[12]) != 0;
    if (R > 0) {  // projection mode: bf16 x, no checkpoints
        if (!bf || keep || page || R > kMaxR) return 1;
        if (cl) run<kFusedProj, 6, 1>(B, D, H, W, dir, nseg, seg_len, false, R, false);
        else run<kFusedProj, 6, 0>(B, D, H, W, dir, nseg, seg_len, false, R, false);
    }
    else if (bf == 2) {  // bf16 u with fp32 delta: the projection form backward's checkpoint pass
        if (cl || keep != 2 || nseg > 1 || page) return 1;
        run<kFused, 6, 0>(B, D, H, W, dir, nseg, seg_len, keep, 0, false);
    }
    else if (bf && cl) run<kFused, 7, 1>(B, D, H, W, dir, nseg, seg_len, keep, 0, page);
    else if (bf) run<kFused, 7, 0>(B, D, H, W, dir, nseg, seg_len, keep, 0, page);
    else if (cl) run<kFused, 4, 1>(B, D, H, W, dir, nseg, seg_len, keep, 0, page);
    else run<kFused, 4, 0>(B, D, H, W, dir, nseg, seg_len, keep, 0, page);
    return 0;
}
