// Runs the general selective-scan kernel's source (scan_kernel of scan.cuh: any N in
// {1, 2, 4, 8, 16}, element types read at run time) on the host, one std::thread per lane,
// over raw input files, and writes y (and h_last); built with AddressSanitizer and UBSan by
// tests/test_scan_kernel_emulation.py.  The warp shapes are the library's for each N.
// Arguments: mode B C H W N G u_bf16 d_bf16 softplus has_D has_bias has_h0 want_hlast R dir
//   mode 0, standalone: u, delta (B, C, L) with L = H*W, Bm, Cm (B, G, N, L), y (B, C, L).
//   mode 1, fused: C is D; x (B, D, H, W), dts (B, 4, D, L), Bm, Cm (B, 4, N, L); y (B, D, H, W)
//           accumulates the four directions.
//   mode 2, projections: as mode 1 with bf16 x, no dts, xdbl (B, 4, R+2N, L) fp32 and
//           Wdt (4, D, R).
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
template <class S>
void launch(ScanArgs a)
{
    S::layout(a);
    a.tiles = (a.per_group + S::CW - 1) / S::CW;
    const int items = a.tiles * a.G * a.B * a.nseg;
    for (int blk = 0; blk < items; ++blk) {
        WarpCtx ctx;
        std::vector<unsigned char> smem(a.smem_bytes + 16);
        ctx.smem = smem.data() + (16 - ((uintptr_t)smem.data() & 15)) % 16;
        ctx.smem_bytes = a.smem_bytes;
        memset(ctx.smem, 0xCD, a.smem_bytes);
        std::vector<std::thread> th;
        for (int lane = 0; lane < 32; ++lane)
            th.emplace_back([&, lane] {
                threadIdx = {(unsigned)lane, 0, 0};
                blockIdx = {(unsigned)blk, 0, 0};
                g_warp = &ctx;
                g_lane = lane;
                scan_kernel<S>(a);
            });
        for (auto &t : th) t.join();
    }
}
// The shapes the library's dispatch picks: <N, lanes per channel, channels per lane, CTAs per SM>.
template <int MODE>
void dispatch(const ScanArgs &a, int N)
{
    constexpr int RT = kDtRuntime;
    switch (N) {
    case 16:
        if constexpr (MODE == kStandalone) launch<ScanShape<16, 2, 1, 12, MODE, RT>>(a);
        else launch<ScanShape<16, 4, 1, 12, MODE, RT>>(a);
        break;
    case 8: launch<ScanShape<8, 2, 1, 12, MODE, RT>>(a); break;
    case 4: launch<ScanShape<4, 1, 1, 8, MODE, RT>>(a); break;
    case 2: launch<ScanShape<2, 1, 1, 8, MODE, RT>>(a); break;
    case 1: launch<ScanShape<1, 1, 1, 8, MODE, RT>>(a); break;
    default: exit(3);
    }
}
int main(int argc, char **argv)
{
    if (argc < 17) return 1;
    int i = 1;
    const int mode = atoi(argv[i++]), B = atoi(argv[i++]), C = atoi(argv[i++]), H = atoi(argv[i++]),
              W = atoi(argv[i++]), N = atoi(argv[i++]), G = atoi(argv[i++]), ub = atoi(argv[i++]),
              db = atoi(argv[i++]), sp = atoi(argv[i++]), hasD = atoi(argv[i++]), hasb = atoi(argv[i++]),
              hash0 = atoi(argv[i++]), wantlast = atoi(argv[i++]), R = atoi(argv[i++]);
    const std::string dir = argv[i++];
    const int L = H * W, esz_u = ub ? 2 : 4, esz_d = db ? 2 : 4;
    const int Ctot = mode == 0 ? C : 4 * C;  // channels of the scan
    const int Gtot = mode == 0 ? G : 4;
    const int Cp = R + 2 * N;
    auto u = rd<unsigned char>(dir + "/u", (size_t)B * C * L * esz_u);  // (B, C, L) or x (B, D, H, W)
    std::vector<unsigned char> delta;
    std::vector<float> Bm, Cm, xdbl, Wdt;
    if (mode == 2) {
        xdbl = rd<float>(dir + "/xdbl", (size_t)B * 4 * Cp * L);
        Wdt = rd<float>(dir + "/Wdt", (size_t)Ctot * R);
    } else {
        delta = rd<unsigned char>(dir + "/delta", (size_t)B * Ctot * L * esz_d);
        Bm = rd<float>(dir + "/Bm", (size_t)B * Gtot * N * L);
        Cm = rd<float>(dir + "/Cm", (size_t)B * Gtot * N * L);
    }
    auto A = rd<float>(dir + "/A", (size_t)Ctot * N);
    std::vector<float> Dv, bias, h0;
    if (hasD) Dv = rd<float>(dir + "/Dv", Ctot);
    if (hasb) bias = rd<float>(dir + "/bias", Ctot);
    if (hash0) h0 = rd<float>(dir + "/h0", (size_t)B * Ctot * N);
    std::vector<float> y((size_t)B * C * L, 0.0f), hlast(wantlast ? (size_t)B * Ctot * N : 0, -12345.0f);
    ScanArgs a{};
    a.u = u.data();
    a.A_log = A.data();
    a.Dv = hasD ? Dv.data() : nullptr;
    a.bias = hasb ? bias.data() : nullptr;
    a.y = y.data();
    a.B = B; a.C = Ctot; a.G = Gtot; a.L = L; a.per_group = Ctot / Gtot;
    a.W = W; a.divH = {H, 1.0f / (float)H};
    a.u_bf16 = ub; a.delta_bf16 = db; a.softplus = sp;
    a.nseg = 1; a.seg_len = L;
    a.h0 = hash0 ? h0.data() : nullptr;
    a.hlast = wantlast ? hlast.data() : nullptr;
    if (mode == 2) {  // as the projection path sets them up: rows of x_dbl
        a.dtl = xdbl.data();
        a.Bm = xdbl.data() + (size_t)R * L;
        a.Cm = xdbl.data() + (size_t)(R + N) * L;
        a.Wdt = Wdt.data();
        a.R = R;
        a.gs = (long long)Cp * L;
        a.delta_bf16 = 0;
        if (!ub || R > kMaxR) return 1;
    } else {
        a.delta = delta.data();
        a.delta_bytes = delta.size();
        a.Bm = Bm.data();
        a.Cm = Cm.data();
        a.gs = (long long)N * L;
    }
    if (mode == 0) dispatch<kStandalone>(a, N);
    else if (mode == 1) dispatch<kFused>(a, N);
    else dispatch<kFusedProj>(a, N);
    FILE *fo = fopen((dir + "/y").c_str(), "wb");
    fwrite(y.data(), 4, y.size(), fo);
    fclose(fo);
    if (wantlast) {
        fo = fopen((dir + "/hlast").c_str(), "wb");
        fwrite(hlast.data(), 4, hlast.size(), fo);
        fclose(fo);
    }
    return 0;
}
