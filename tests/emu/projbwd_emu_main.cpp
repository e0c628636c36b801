// Runs dt_proj's kernels of the projection form's backward (dtproj_expand_kernel,
// dtproj_dgrad_kernel, dtproj_wgrad_kernel of proj_bwd.cu) on the host: one std::thread per
// thread of each CTA, warp shuffles on a per-warp barrier, __syncthreads on a per-CTA barrier;
// built with AddressSanitizer and UBSan by tests/test_projection_backward_emulation.py.
// Arguments: B D H W N R batch_per_block dir [adj_ctas]
// adj_ctas > 0 runs the two adjoints as dtproj_adj_kernel on (adj_ctas, 4) CTAs instead.
// Reads dir/xdbl (B, 4, R+2N, L), dir/Wdt (4, D, R) and dir/ddts (B, 4, D, L), all fp32, and
// writes dir/dts (B, 4, D, L), dir/dtlow (B, 4, R, L) and dir/dWdt (4, D, R).
#include <algorithm>
#include <cstring>
#include <string>
#include <vector>
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
void wr(const std::string &f, const std::vector<float> &v)
{
    FILE *fo = fopen(f.c_str(), "wb");
    fwrite(v.data(), 4, v.size(), fo);
    fclose(fo);
}
int main(int argc, char **argv)
{
    if (argc < 9) return 1;
    const int B = atoi(argv[1]), D = atoi(argv[2]), H = atoi(argv[3]), W = atoi(argv[4]), N = atoi(argv[5]),
              R = atoi(argv[6]), bpb = atoi(argv[7]);
    const std::string dir = argv[8];
    const int adj_ctas = argc > 9 ? atoi(argv[9]) : 0;
    const int L = H * W, Cp = R + 2 * N;
    if (R < 1 || R > kMaxRLarge || bpb < 1) return 1;
    auto xdbl = rd<float>(dir + "/xdbl", (size_t)B * 4 * Cp * L);
    auto Wdt = rd<float>(dir + "/Wdt", (size_t)4 * D * R);
    auto ddts = rd<float>(dir + "/ddts", (size_t)B * 4 * D * L);
    std::vector<float> dts((size_t)B * 4 * D * L, -12345.0f), dtlow((size_t)B * 4 * R * L, -12345.0f),
        dWdt((size_t)4 * D * R, 0.0f);
    const unsigned lx = (L + kDtThreads - 1) / kDtThreads;
    if (dt_chunked(D, R)) {
        const size_t csm = sizeof(float) * kDtChunk * kMaxRLarge;
        emu_grid(lx, B * 4, kDtThreads, csm,
                 [&] { dtproj_expand_chunked_kernel(xdbl.data(), Wdt.data(), dts.data(), D, L, R, Cp); });
        emu_grid(lx, B * 4, kDtThreads, csm,
                 [&] { dtproj_dgrad_chunked_kernel(ddts.data(), Wdt.data(), dtlow.data(), D, L, R); });
    } else {
        const size_t dsm = dt_smem_bytes(D, R);
        emu_grid(lx, B * 4, kDtThreads, dsm, [&] { dtproj_expand_kernel(xdbl.data(), Wdt.data(), dts.data(), D, L, R, Cp); });
        if (L % 4 == 0) {
            // the four-step expansion must give the same bits
            std::vector<float> dts4((size_t)B * 4 * D * L, -12345.0f);
            const unsigned lx4 = (L / 4 + kDtThreads - 1) / kDtThreads;
            emu_grid(lx4, B * 4, kDtThreads, dsm,
                     [&] { dtproj_expand4_kernel(xdbl.data(), Wdt.data(), dts4.data(), D, L, R, Cp); });
            if (memcmp(dts4.data(), dts.data(), dts.size() * sizeof(float)) != 0) {
                fprintf(stderr, "dtproj_expand4_kernel differs from dtproj_expand_kernel\n");
                return 3;
            }
        }
        emu_grid(lx, B * 4, kDtThreads, dsm, [&] { dtproj_dgrad_kernel(ddts.data(), Wdt.data(), dtlow.data(), D, L, R); });
    }
    if (adj_ctas > 0) {
        if (R > 16 || D > kAdjMaxD || L % 4 != 0) return 1;
        std::fill(dtlow.begin(), dtlow.end(), -12345.0f);  // written again by the fused kernel alone
        if (R <= 8)
            emu_grid(adj_ctas, 4, kAdjThreads, adj_smem_bytes(D, 8), [&] {
                dtproj_adj_kernel<8>(ddts.data(), xdbl.data(), Wdt.data(), dtlow.data(), dWdt.data(), B, D, L, R, Cp);
            });
        else
            emu_grid(adj_ctas, 4, kAdjThreads, adj_smem_bytes(D, 16), [&] {
                dtproj_adj_kernel<16>(ddts.data(), xdbl.data(), Wdt.data(), dtlow.data(), dWdt.data(), B, D, L, R, Cp);
            });
        wr(dir + "/dts", dts);
        wr(dir + "/dtlow", dtlow);
        wr(dir + "/dWdt", dWdt);
        return 0;
    }
    const int tile = R <= 16 ? 4 : (R <= 32 ? 2 : 1);
    const int nt = (D + tile - 1) / tile;
    const unsigned gy = (B + bpb - 1) / bpb;
    const int rm = R <= 8 ? 8 : (R <= 16 ? 16 : (R <= 32 ? 32 : 64));
    const size_t wsm = sizeof(float) * tile * rm * (kWgThreads / 32);
    if (R <= 8)
        emu_grid(4 * nt, gy, kWgThreads, wsm,
                 [&] { dtproj_wgrad_kernel<8, 4>(ddts.data(), xdbl.data(), dWdt.data(), B, D, L, R, Cp, bpb); });
    else if (R <= 16)
        emu_grid(4 * nt, gy, kWgThreads, wsm,
                 [&] { dtproj_wgrad_kernel<16, 4>(ddts.data(), xdbl.data(), dWdt.data(), B, D, L, R, Cp, bpb); });
    else if (R <= 32)
        emu_grid(4 * nt, gy, kWgThreads, wsm,
                 [&] { dtproj_wgrad_kernel<32, 2>(ddts.data(), xdbl.data(), dWdt.data(), B, D, L, R, Cp, bpb); });
    else
        emu_grid(4 * nt, gy, kWgThreads, wsm,
                 [&] { dtproj_wgrad_kernel<64, 1>(ddts.data(), xdbl.data(), dWdt.data(), B, D, L, R, Cp, bpb); });
    wr(dir + "/dts", dts);
    wr(dir + "/dtlow", dtlow);
    wr(dir + "/dWdt", dWdt);
    return 0;
}
