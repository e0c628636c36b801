// scan_bwd.cuh -- reverse-mode gradient of the fused SS2D core scan (N = 16).
//
// The forward recurrence (the selective scan called in section 3.2 of the
// VMamba SS2D article, on the discrete SSM of the DAMamba article, section 2.1)
//     dt_l = softplus(z_l), z_l = dts_l + bias,  dA_l[n] = exp(dt_l A[n]),
//     h_l[n] = dA_l[n] h_{l-1}[n] + dt_l B_l[n] u_l,   y_l = C_l . h_l + D u_l
// is differentiated by carrying the adjoint g_l[n] = dLoss/dh_l[n] backwards:
//     g_l = C_l dy_l + dA_{l+1} g_{l+1}
//     du_l    = D dy_l + dt_l sum_n g_l B_l
//     ddts_l  = (u_l sum_n g_l B_l + sum_n A g_l dA_l h_{l-1}) * sigmoid(z_l)
//     dA[n]  += g_l dt_l dA_l h_{l-1},   dB_l += g_l dt_l u_l,   dC_l += dy_l h_l
//     dD += dy_l u_l,   dbias += ddts_l.
// In the fused core the gradient of direction k's output at step l is dy at the
// pixel pi_k(l) (CrossMerge's adjoint is CrossScan) and du is added into dx at
// that pixel (CrossScan's adjoint is CrossMerge).
//
// Work item = one warp (one CTA): 16 channels of one (batch, direction), lanes
// 2c and 2c+1 holding states q, q+2, ..., q+14 of channel c (q = lane & 1), as in
// the forward kernel.  The sequence is walked backwards in chunks of 16 steps:
//   stage    B/C, dts, u and dy rows of chunk j-1 and the checkpointed state
//            before chunk j-1 are copied into the two-deep ring with cp.async
//            (the checkpoint pass stores the state before every 16th step);
//   forward  from the checkpoint, the chunk is rescanned in four blocks of four
//            steps, keeping each block's entry state, dt, dt*u and sigmoid(z)
//            in shared memory;
//   reverse  blocks 3..0: the block's four decays per state are recomputed into
//            registers together with its four entry states, then the four
//            steps are run backwards updating the adjoint; dB/dC terms of the
//            16 channels are summed through a shared-memory transpose, du and
//            ddts of each channel through one shuffle;
//   write    ddts rows are stored; du is added into dx at the step's pixel and
//            the chunk's dB/dC rows into dBs/dCs (shared by the direction's
//            channels of other warps) with atomics.
// dA_log, dD and dbias are accumulated in registers and added at the end.
#pragma once

#include "common.cuh"
#include "scan.cuh"
#include "scan2.cuh"

namespace ss2d {

constexpr int kBTC = 16;  // steps per backward chunk; also the checkpoint interval

struct BwdArgs {
    const void *x;        // (B, D, H, W): u of scan orders 0 and 2
    const void *xT;       // (B, D, W, H): u of scan orders 1 and 3
    const void *dts;      // (B, 4D, L) in scan order
    const float *A_log;   // (4D, 16)
    const float *Bm;      // (B, 4, 16, L)
    const float *Cm;      // (B, 4, 16, L)
    const float *Dv;      // (4D) or null
    const float *bias;    // (4D) or null
    const float *ckpt;    // (B, 4D, nck, 16): state before step 16j, state q + 2n at q*8 + n
    const float *dy;      // (B, D, H, W)
    const float *dyT;     // (B, D, W, H)
    float *dx;            // (B, D, H, W), accumulated
    float *ddts;          // (B, 4D, L), written
    float *dA_log;        // (4D, 16), accumulated
    float *dBm, *dCm;     // (B, 4, 16, L), accumulated
    float *dDv, *dbias;   // (4D) or null, accumulated
    int B, D, W, L, C, tiles, nck;
    SmallDiv divH;
    // Segments (long sequences with few channels): segment s covers steps
    // [s*seg_len, min(L, (s+1)*seg_len)), seg_len a multiple of 32.  nseg = 1 walks whole
    // sequences.  g_in (B, 4D, nseg, 16): the adjoint term dA_b * g_b entering each segment
    // from the step after its last one (zero for the last segment), or null for zero.
    int nseg, seg_len;
    float *g_in;
    // adjoint_carry_kernel outputs, (B, 4D, nseg, 16): the term dA_a * g_a leaving each
    // segment at its first step a when nothing enters it, and the product of its decays.
    float *e_out, *p_out;
};

struct BwdLayout {
    int stage_bytes, off_bc, off_d, off_u, off_dy, off_ck;
    int off_dl, off_du, off_sg, off_hb, off_red, off_dbc, off_gdt, off_gdx, off_pix, smem_bytes;
};

template <int DT_>
struct BwdShape {
    static constexpr int N = 16, NS = 8, CW = 16, BTC = kBTC;
    static constexpr bool D_BF16 = (DT_ & 1) != 0;
    static constexpr bool U_BF16 = (DT_ & 2) != 0;
    static constexpr int ESZ_D = D_BF16 ? 2 : 4;
    static constexpr int ESZ_U = U_BF16 ? 2 : 4;
    static constexpr int BCP = BTC + 4;            // B/C row pitch (floats)
    static constexpr int DROW = BTC * ESZ_D + 16;  // dts row pitch (bytes)
    static constexpr int UROW = BTC * ESZ_U + 16;  // u row pitch (bytes)
    static constexpr int YROW = BTC * 4 + 16;      // dy row pitch (bytes)
    static constexpr int XP = BTC + 4;             // per-chunk cache row pitch (floats)
    static constexpr int RP = NS * 4 + 4;          // reduce buffer: 8 values x 4 steps per lane (dB, then dC), padded

    static BwdLayout layout()
    {
        BwdLayout l{};
        int off = 0;
        l.off_bc = off;
        off += 2 * N * BCP * 4;
        l.off_d = off;
        off += CW * DROW;
        l.off_u = off;
        off += CW * UROW;
        l.off_dy = off;
        off += CW * YROW;
        l.off_ck = off;
        off += 32 * NS * 4;
        l.stage_bytes = (off + 15) & ~15;
        off = 2 * l.stage_bytes;
        l.off_dl = off;
        off += CW * XP * 4;
        l.off_du = off;
        off += CW * XP * 4;
        l.off_sg = off;
        off += CW * XP * 4;
        l.off_hb = off;
        off += (BTC / 4) * 32 * NS * 4;
        l.off_red = off;
        off += 32 * RP * 4;
        l.off_dbc = off;
        off += 2 * N * XP * 4;
        // the per-chunk dts and dx gradients take the rows of delta and delta*u: block m's
        // gradients are written after every lane has read block m's delta and delta*u, and
        // the write-out reads them before the next chunk's rescan rewrites those rows
        l.off_gdt = l.off_dl;
        l.off_gdx = l.off_du;
        l.off_pix = off;
        off += 2 * BTC * 4;
        l.smem_bytes = (off + 15) & ~15;
        return l;
    }
};

template <class S>
__global__ void __launch_bounds__(32, 8) scan_bwd_kernel(const BwdArgs a, const BwdLayout lay)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    constexpr int N = S::N, NS = S::NS, CW = S::CW, BTC = S::BTC, BCP = S::BCP, XP = S::XP, RP = S::RP;
    constexpr int ESZ_D = S::ESZ_D, ESZ_U = S::ESZ_U, DROW = S::DROW, UROW = S::UROW, YROW = S::YROW;
    constexpr bool U_BF16 = S::U_BF16, D_BF16 = S::D_BF16;

    const int lane = threadIdx.x;
    float *dlr = reinterpret_cast<float *>(smem_raw + lay.off_dl);
    float *dur = reinterpret_cast<float *>(smem_raw + lay.off_du);
    float *sgr = reinterpret_cast<float *>(smem_raw + lay.off_sg);
    float *hbr = reinterpret_cast<float *>(smem_raw + lay.off_hb);
    float *redr = reinterpret_cast<float *>(smem_raw + lay.off_red);
    float *dbcr = reinterpret_cast<float *>(smem_raw + lay.off_dbc);
    float *gdtr = reinterpret_cast<float *>(smem_raw + lay.off_gdt);
    float *gdxr = reinterpret_cast<float *>(smem_raw + lay.off_gdx);
    int *pixr = reinterpret_cast<int *>(smem_raw + lay.off_pix);

    if (a.nseg < 1 || a.seg_len < 1)
        return;  // launchers always set at least one segment covering the sequence
    int it = blockIdx.x;
    const int seg = it % a.nseg;
    it /= a.nseg;
    const int tile = it % a.tiles;
    it /= a.tiles;
    const int g = it % 4;
    const int b = it / 4;
    const int D = a.D, L = a.L;
    const int d0 = tile * CW;
    const int ch_valid = min(CW, D - d0);
    const int c0 = g * D + d0;

    const int ch = lane >> 1;
    const int q = lane & 1;
    const int cch = c0 + min(ch, ch_valid - 1);
    float a2[NS], gn[NS], dAacc[NS], h[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) {
        a2[n] = -expf(__ldg(a.A_log + (size_t)cch * N + q + 2 * n)) * kLog2e;
        // the adjoint entering this segment from the next one (zero at the sequence end)
        gn[n] = a.g_in ? __ldg(a.g_in + (((size_t)b * a.C + cch) * a.nseg + seg) * N + q + 2 * n) : 0.0f;
        dAacc[n] = 0.0f;
    }
    const float bias_ch = a.bias ? __ldg(a.bias + cch) : 0.0f;
    const float dsk_ch = a.Dv ? __ldg(a.Dv + cch) : 0.0f;
    float dD_acc = 0.0f, db_acc = 0.0f;

    // u and dy of orders 0/2 are rows of x / dy, of orders 1/3 rows of the transposed
    // planes; orders 2/3 walk their rows backwards.
    const bool rev = g >= 2;
    const char *ubase = reinterpret_cast<const char *>((g & 1) ? a.xT : a.x);
    const float *ybase = (g & 1) ? a.dyT : a.dy;
    const size_t prow0 = ((size_t)b * D + d0) * L;   // element of (channel row d0, pixel 0) in x / dy
    const size_t drow0 = ((size_t)b * a.C + c0) * L;  // element of (channel row c0, step 0) in dts
    const size_t grow = ((size_t)b * 4 + g) * N * L;  // row 0 of this (b, g) in Bm / Cm
    const float *Bg = a.Bm + grow;
    const float *Cg = a.Cm + grow;
    const char *dbase = reinterpret_cast<const char *>(a.dts);
    const uint64_t pol_once = l2_policy_evict_first();
    const uint64_t pol_keep = l2_policy_evict_last();

    // fp32 rows start on 16-byte boundaries when L % 4 == 0; otherwise (VMamba-T stage 4,
    // 7 x 7) every row is staged with 4-byte copies, into the same shared-memory layout
    const bool rows16 = (L & 3) == 0;

    // ---- staging of chunk j (steps [16j, 16j+16)) into ring stage st ----------
    auto stage_chunk = [&](int j, int st) {
        unsigned char *rs = smem_raw + st * lay.stage_bytes;
        const int l0 = j * BTC;
        if (lane < BTC) {
            const int l = l0 + lane;
            pixr[st * BTC + lane] = (l < L) ? scan_pixel(g, l, L, a.W, a.divH) : 0;
        }
        if constexpr (ESZ_D == 4 && ESZ_U == 4) {
            if (!rows16) {
                // element = (row, step v) with v fastest; steps past the sequence (and, for the
                // reversed orders, pixels before 0) are zero-filled
                float *bcd = reinterpret_cast<float *>(rs + lay.off_bc);
                for (int p = lane; p < 2 * N * BTC; p += 32) {
                    const int row = p / BTC, v = p % BTC, l = l0 + v;
                    const float *src = row < N ? Bg + (size_t)row * L : Cg + (size_t)(row - N) * L;
                    cp_async4(bcd + row * BCP + v, l < L ? src + l : src, l < L ? 4 : 0);
                }
                const float *dts32 = reinterpret_cast<const float *>(dbase);
                for (int p = lane; p < CW * BTC; p += 32) {
                    const int chl = p / BTC, v = p % BTC, l = l0 + v;
                    const float *src = dts32 + drow0 + (size_t)min(chl, ch_valid - 1) * L;
                    const bool ok = chl < ch_valid && l < L;
                    cp_async4(rs + lay.off_d + chl * DROW + v * 4, ok ? src + l : src, ok ? 4 : 0);
                    const int e = (rev ? L - l0 - BTC : l0) + v;
                    const bool oke = chl < ch_valid && e >= 0 && e < L;
                    const float *us = reinterpret_cast<const float *>(ubase) + prow0 + (size_t)min(chl, ch_valid - 1) * L;
                    cp_async4(rs + lay.off_u + chl * UROW + v * 4, oke ? us + e : us, oke ? 4 : 0);
                    const float *ys = ybase + prow0 + (size_t)min(chl, ch_valid - 1) * L;
                    cp_async4(rs + lay.off_dy + chl * YROW + v * 4, oke ? ys + e : ys, oke ? 4 : 0);
                }
                const float *src = a.ckpt + (((size_t)b * a.C + cch) * a.nck + j) * N + q * NS;
                float *dst = reinterpret_cast<float *>(rs + lay.off_ck) + lane * NS;
                cp_async16(dst, src, 16);
                cp_async16(dst + 4, src + 4, 16);
                return;
            }
        }
        // B and C rows: 32 rows x 4 pieces of 16 bytes
        {
            const int v = (lane & 3) * 4;
            const int bytes = max(0, min(16, (L - l0 - v) * 4));
            float *dst = reinterpret_cast<float *>(rs + lay.off_bc);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int row = (lane >> 2) + 8 * k;
                const float *src = (row < N ? Bg + (size_t)row * L : Cg + (size_t)(row - N) * L) + v;
                cp_async16(dst + row * BCP + v, bytes > 0 ? src + l0 : src, bytes);
            }
        }
        // dts rows (scan order)
        {
            constexpr int PER_ROW = BTC * ESZ_D / 16;
            for (int p = lane; p < CW * PER_ROW; p += 32) {
                const int chl = p / PER_ROW, v = p % PER_ROW;
                const int l = l0 + v * (16 / ESZ_D);
                const char *src = dbase + (drow0 + (size_t)min(chl, ch_valid - 1) * L) * ESZ_D;
                const int bytes = chl < ch_valid ? max(0, min(16, (L - l) * ESZ_D)) : 0;
                cp_async16_hint(rs + lay.off_d + chl * DROW + v * 16, bytes > 0 ? src + (size_t)l * ESZ_D : src,
                                bytes, pol_once);
            }
        }
        // u rows and dy rows: steps in order, or pixels [L-l0-16, L-l0) for the reversed orders
        {
            constexpr int PER_ROW = BTC * ESZ_U / 16;
            for (int p = lane; p < CW * PER_ROW; p += 32) {
                const int chl = p / PER_ROW, v = p % PER_ROW;
                const int e = (rev ? L - l0 - BTC : l0) + v * (16 / ESZ_U);
                const char *src = ubase + (prow0 + (size_t)min(chl, ch_valid - 1) * L) * ESZ_U;
                const int bytes = (chl < ch_valid && e >= 0) ? max(0, min(16, (L - e) * ESZ_U)) : 0;
                cp_async16(rs + lay.off_u + chl * UROW + v * 16, bytes > 0 ? src + (size_t)e * ESZ_U : src, bytes);
            }
            constexpr int YPER_ROW = BTC * 4 / 16;
            for (int p = lane; p < CW * YPER_ROW; p += 32) {
                const int chl = p / YPER_ROW, v = p % YPER_ROW;
                const int e = (rev ? L - l0 - BTC : l0) + v * 4;
                const float *src = ybase + prow0 + (size_t)min(chl, ch_valid - 1) * L;
                const int bytes = (chl < ch_valid && e >= 0) ? max(0, min(16, (L - e) * 4)) : 0;
                cp_async16_hint(rs + lay.off_dy + chl * YROW + v * 16, bytes > 0 ? src + e : src, bytes, pol_once);
            }
        }
        // this lane's checkpoint (state before step l0; states q + 2n stored at q*8 + n)
        {
            const float *src = a.ckpt + (((size_t)b * a.C + cch) * a.nck + j) * N + q * NS;
            float *dst = reinterpret_cast<float *>(rs + lay.off_ck) + lane * NS;
            cp_async16(dst, src, 16);
            cp_async16(dst + 4, src + 4, 16);
        }
    };

    // this segment's chunks [jbeg, jend), walked from the last
    const int jbeg = seg * a.seg_len / BTC;  // seg_len is L (one segment) or a multiple of 32
    const int jend = min(a.nck, ((seg + 1) * a.seg_len + BTC - 1) / BTC);
    const int nck = jend - jbeg;
    stage_chunk(jend - 1, 0);
    cp_async_commit();

    for (int jj = 0; jj < nck; ++jj) {
        const int j = jend - 1 - jj;
        const int l0 = j * BTC;
        const int valid = min(BTC, L - l0);
        const int st = jj & 1;
        const unsigned char *rs = smem_raw + st * lay.stage_bytes;

        cp_async_wait<0>();
        __syncwarp();
        if (jj + 1 < nck)
            stage_chunk(j - 1, st ^ 1);
        cp_async_commit();

        const float *bcs = reinterpret_cast<const float *>(rs + lay.off_bc);
        const unsigned char *drs = rs + lay.off_d + ch * DROW;
        const unsigned char *urs = rs + lay.off_u + ch * UROW;
        const float *yrs = reinterpret_cast<const float *>(rs + lay.off_dy + ch * YROW);
        {
            const float4 *ck = reinterpret_cast<const float4 *>(rs + lay.off_ck) + lane * 2;
            const float4 c0v = ck[0], c1v = ck[1];
            h[0] = c0v.x; h[1] = c0v.y; h[2] = c0v.z; h[3] = c0v.w;
            h[4] = c1v.x; h[5] = c1v.y; h[6] = c1v.z; h[7] = c1v.w;
        }

        // u of step s of this lane's channel
        auto u_at2 = [&](int s, float &u0, float &u1) {  // steps s, s+1 (s even)
            if constexpr (U_BF16) {
                const uint32_t w = *reinterpret_cast<const uint32_t *>(urs + 2 * (rev ? BTC - 2 - s : s));
                u0 = rev ? bf16_hi(w) : bf16_lo(w);
                u1 = rev ? bf16_lo(w) : bf16_hi(w);
            } else {
                const float2 t = *reinterpret_cast<const float2 *>(urs + 4 * (rev ? BTC - 2 - s : s));
                u0 = rev ? t.y : t.x;
                u1 = rev ? t.x : t.y;
            }
        };

        // ---- forward over the chunk: block entry states, dt, dt*u, sigmoid(z) ---------
#pragma unroll 1
        for (int m = 0; m < BTC / 4; ++m) {
            const int i = 4 * m;
            // block entry states: states 0-3 of every lane, then states 4-7 (16-byte lane stride)
            float4 *hb = reinterpret_cast<float4 *>(hbr) + m * 32 + lane;
            hb[0] = make_float4(h[0], h[1], h[2], h[3]);
            hb[(BTC / 4) * 32] = make_float4(h[4], h[5], h[6], h[7]);
            const int s0 = i + 2 * q;
            float z0, z1, u0, u1;
            if constexpr (D_BF16) {
                const uint32_t w = *reinterpret_cast<const uint32_t *>(drs + 2 * s0);
                z0 = bf16_lo(w);
                z1 = bf16_hi(w);
            } else {
                const float2 t = *reinterpret_cast<const float2 *>(drs + 4 * s0);
                z0 = t.x;
                z1 = t.y;
            }
            u_at2(s0, u0, u1);
            float d0v, d1v, sg0, sg1;
            softplus_sigmoid_f32(z0 + bias_ch, d0v, sg0);
            softplus_sigmoid_f32(z1 + bias_ch, d1v, sg1);
            const float w0 = d0v * u0, w1 = d1v * u1;
            *reinterpret_cast<float2 *>(dlr + ch * XP + s0) = make_float2(d0v, d1v);
            *reinterpret_cast<float2 *>(dur + ch * XP + s0) = make_float2(w0, w1);
            *reinterpret_cast<float2 *>(sgr + ch * XP + s0) = make_float2(sg0, sg1);
            const float pz0 = __shfl_xor_sync(0xffffffffu, d0v, 1), pz1 = __shfl_xor_sync(0xffffffffu, d1v, 1);
            const float pw0 = __shfl_xor_sync(0xffffffffu, w0, 1), pw1 = __shfl_xor_sync(0xffffffffu, w1, 1);
            const float2 dl01 = q ? make_float2(pz0, pz1) : make_float2(d0v, d1v);
            const float2 dl23 = q ? make_float2(d0v, d1v) : make_float2(pz0, pz1);
            const float2 du01 = q ? make_float2(pw0, pw1) : make_float2(w0, w1);
            const float2 du23 = q ? make_float2(w0, w1) : make_float2(pw0, pw1);
#pragma unroll
            for (int n = 0; n < NS; ++n) {
                const float4 bb = *reinterpret_cast<const float4 *>(bcs + (q + 2 * n) * BCP + i);
                const float2 an = make_float2(a2[n], a2[n]);
                const float2 x01 = __fmul2_rn(dl01, an), x23 = __fmul2_rn(dl23, an);
                const float2 bu01 = __fmul2_rn(du01, make_float2(bb.x, bb.y));
                const float2 bu23 = __fmul2_rn(du23, make_float2(bb.z, bb.w));
                float hh = fmaf(ex2_approx(x01.x), h[n], bu01.x);
                hh = fmaf(ex2_approx(x01.y), hh, bu01.y);
                hh = fmaf(ex2_approx(x23.x), hh, bu23.x);
                h[n] = fmaf(ex2_approx(x23.y), hh, bu23.y);
            }
        }
        __syncwarp();

        // ---- reverse over the chunk, four steps at a time ------------------------------
#pragma unroll 1
        for (int m = BTC / 4 - 1; m >= 0; --m) {
            const int i = 4 * m;
            float h0[NS];
            {
                const float4 *hb = reinterpret_cast<const float4 *>(hbr) + m * 32 + lane;
                const float4 v0 = hb[0], v1 = hb[(BTC / 4) * 32];
                h0[0] = v0.x; h0[1] = v0.y; h0[2] = v0.z; h0[3] = v0.w;
                h0[4] = v1.x; h0[5] = v1.y; h0[6] = v1.z; h0[7] = v1.w;
            }
            const float4 dl4 = *reinterpret_cast<const float4 *>(dlr + ch * XP + i);
            const float4 du4 = *reinterpret_cast<const float4 *>(dur + ch * XP + i);
            const float4 sg4 = *reinterpret_cast<const float4 *>(sgr + ch * XP + i);
            float4 dy4, u4;
            {
                const float4 t = *reinterpret_cast<const float4 *>(yrs + (rev ? BTC - 4 - i : i));
                dy4 = rev ? make_float4(t.w, t.z, t.y, t.x) : t;
                float ua, ub, uc, ud;
                u_at2(i, ua, ub);
                u_at2(i + 2, uc, ud);
                u4 = make_float4(ua, ub, uc, ud);
            }
            float su0 = 0.f, su1 = 0.f, su2 = 0.f, su3 = 0.f;  // sum_n g B per step
            float sa0 = 0.f, sa1 = 0.f, sa2 = 0.f, sa3 = 0.f;  // sum_n a2 g dA h_prev per step
            float *redl = redr + lane * RP;
            float4 dCk[NS];  // this lane's dC terms, reduced after the dB terms
#pragma unroll
            for (int n = 0; n < NS; ++n) {
                const int sr = q + 2 * n;
                const float4 bb = *reinterpret_cast<const float4 *>(bcs + sr * BCP + i);
                const float4 cc = *reinterpret_cast<const float4 *>(bcs + (N + sr) * BCP + i);
                const float e0 = ex2_approx(dl4.x * a2[n]), e1 = ex2_approx(dl4.y * a2[n]);
                const float e2 = ex2_approx(dl4.z * a2[n]), e3 = ex2_approx(dl4.w * a2[n]);
                const float hp0 = h0[n];
                const float hp1 = fmaf(e0, hp0, du4.x * bb.x);
                const float hp2 = fmaf(e1, hp1, du4.y * bb.y);
                const float hp3 = fmaf(e2, hp2, du4.z * bb.z);
                const float hc3 = fmaf(e3, hp3, du4.w * bb.w);
                float gg, gt;
                float4 dBv, dCv;
                // step i+3
                gg = fmaf(cc.w, dy4.w, gn[n]);
                dCv.w = dy4.w * hc3;
                dBv.w = gg * du4.w;
                su3 = fmaf(gg, bb.w, su3);
                gt = gg * (e3 * hp3);
                dAacc[n] = fmaf(dl4.w, gt, dAacc[n]);
                sa3 = fmaf(a2[n], gt, sa3);
                gn[n] = e3 * gg;
                // step i+2
                gg = fmaf(cc.z, dy4.z, gn[n]);
                dCv.z = dy4.z * hp3;
                dBv.z = gg * du4.z;
                su2 = fmaf(gg, bb.z, su2);
                gt = gg * (e2 * hp2);
                dAacc[n] = fmaf(dl4.z, gt, dAacc[n]);
                sa2 = fmaf(a2[n], gt, sa2);
                gn[n] = e2 * gg;
                // step i+1
                gg = fmaf(cc.y, dy4.y, gn[n]);
                dCv.y = dy4.y * hp2;
                dBv.y = gg * du4.y;
                su1 = fmaf(gg, bb.y, su1);
                gt = gg * (e1 * hp1);
                dAacc[n] = fmaf(dl4.y, gt, dAacc[n]);
                sa1 = fmaf(a2[n], gt, sa1);
                gn[n] = e1 * gg;
                // step i
                gg = fmaf(cc.x, dy4.x, gn[n]);
                dCv.x = dy4.x * hp1;
                dBv.x = gg * du4.x;
                su0 = fmaf(gg, bb.x, su0);
                gt = gg * (e0 * hp0);
                dAacc[n] = fmaf(dl4.x, gt, dAacc[n]);
                sa0 = fmaf(a2[n], gt, sa0);
                gn[n] = e0 * gg;
                reinterpret_cast<float4 *>(redl)[n] = dBv;
                dCk[n] = dCv;
            }
            __syncwarp();
            // sum of the dB terms, then of the dC terms, over the warp's 16 channels through one
            // 8-value buffer per lane: lanes (q', k', h) add value k' of the lanes 2c + q' for the
            // channels c = 2j + h, and the two halves h combine by shuffle into state q' + 2k'
            auto reduce_half = [&](int rowbase) {
                const int qo = lane & 1, ko = (lane >> 1) & (NS - 1), hc = lane >> 4;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int j = 0; j < CW / 2; ++j) {
                    const float4 v = reinterpret_cast<const float4 *>(redr + (2 * (2 * j + hc) + qo) * RP)[ko];
                    acc.x += v.x;
                    acc.y += v.y;
                    acc.z += v.z;
                    acc.w += v.w;
                }
                acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 16);
                acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 16);
                acc.z += __shfl_xor_sync(0xffffffffu, acc.z, 16);
                acc.w += __shfl_xor_sync(0xffffffffu, acc.w, 16);
                if (hc == 0)
                    *reinterpret_cast<float4 *>(dbcr + (rowbase + qo + 2 * ko) * XP + i) = acc;
            };
            reduce_half(0);
            __syncwarp();
#pragma unroll
            for (int n = 0; n < NS; ++n)
                reinterpret_cast<float4 *>(redl)[n] = dCk[n];
            __syncwarp();
            reduce_half(N);
            // per channel: combine the two lanes' halves of the state sums
            su0 += __shfl_xor_sync(0xffffffffu, su0, 1);
            su1 += __shfl_xor_sync(0xffffffffu, su1, 1);
            su2 += __shfl_xor_sync(0xffffffffu, su2, 1);
            su3 += __shfl_xor_sync(0xffffffffu, su3, 1);
            sa0 += __shfl_xor_sync(0xffffffffu, sa0, 1);
            sa1 += __shfl_xor_sync(0xffffffffu, sa1, 1);
            sa2 += __shfl_xor_sync(0xffffffffu, sa2, 1);
            sa3 += __shfl_xor_sync(0xffffffffu, sa3, 1);
            // lane q keeps steps i+2q, i+2q+1
            const float suA = q ? su2 : su0, suB = q ? su3 : su1;
            const float saA = q ? sa2 : sa0, saB = q ? sa3 : sa1;
            const float dlA = q ? dl4.z : dl4.x, dlB = q ? dl4.w : dl4.y;
            const float uA = q ? u4.z : u4.x, uB = q ? u4.w : u4.y;
            const float yA = q ? dy4.z : dy4.x, yB = q ? dy4.w : dy4.y;
            const float sgA = q ? sg4.z : sg4.x, sgB = q ? sg4.w : sg4.y;
            const float gxA = fmaf(dsk_ch, yA, dlA * suA), gxB = fmaf(dsk_ch, yB, dlB * suB);
            const float gdA = fmaf(uA, suA, kLn2 * saA) * sgA, gdB = fmaf(uB, suB, kLn2 * saB) * sgB;
            *reinterpret_cast<float2 *>(gdxr + ch * XP + i + 2 * q) = make_float2(gxA, gxB);
            *reinterpret_cast<float2 *>(gdtr + ch * XP + i + 2 * q) = make_float2(gdA, gdB);
            dD_acc = fmaf(yA, uA, fmaf(yB, uB, dD_acc));
            db_acc += gdA + gdB;
            __syncwarp();
        }

        // ---- write-out of the chunk -------------------------------------------------------
        {
            const int s = lane & (BTC - 1);
            const int r0 = lane / BTC;  // 0 or 1
            if (s < valid) {
                const int pix = pixr[st * BTC + s];
#pragma unroll
                for (int k = 0; k < CW / 2; ++k) {
                    const int chl = 2 * k + r0;
                    if (chl < ch_valid) {
                        a.ddts[drow0 + (size_t)chl * L + l0 + s] = gdtr[chl * XP + s];
                        red_add_hint(a.dx + prow0 + (size_t)chl * L + pix, gdxr[chl * XP + s], pol_keep);
                    }
                }
#pragma unroll
                for (int k = 0; k < N; ++k) {
                    const int row = 2 * k + r0;  // rows 0..15 dB, 16..31 dC
                    float *dst = (row < N ? a.dBm + grow + (size_t)row * L : a.dCm + grow + (size_t)(row - N) * L);
                    red_add_hint(dst + l0 + s, dbcr[row * XP + s], pol_keep);
                }
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();

    // ---- parameter gradients accumulated over the sequence ---------------------------------
    // each lane summed dD / dbias over its own two steps of every block: combine the pair
    const float dD_tot = dD_acc + __shfl_xor_sync(0xffffffffu, dD_acc, 1);
    const float db_tot = db_acc + __shfl_xor_sync(0xffffffffu, db_acc, 1);
    if (ch < ch_valid) {
#pragma unroll
        for (int n = 0; n < NS; ++n)
            atomicAdd(a.dA_log + (size_t)cch * N + q + 2 * n, dAacc[n] * a2[n] * kLn2);  // dA[n] * A[n]
        if (q == 0 && a.dDv)
            atomicAdd(a.dDv + cch, dD_tot);
        if (q == 0 && a.dbias)
            atomicAdd(a.dbias + cch, db_tot);
    }
}

// First pass of a segmented backward.  For every segment but the first (s >= 1), the
// adjoint recursion g_l = C_l dy_l + dA_{l+1} g_{l+1} is run backwards over the segment's
// steps [a, b) from nothing entering at b.  The term leaving at the first step, dA_a g_a,
// goes to e_out and the product of the segment's decays, exp2(a2 * sum of delta), to p_out.
// A carry over the segments then gives what enters each segment (adjoint_carry_in_kernel).
// Same warp layout and staging as scan_bwd_kernel (C, dts and dy rows only).
template <class S>
__global__ void __launch_bounds__(32, 8) adjoint_carry_kernel(const BwdArgs a, const BwdLayout lay)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    constexpr int N = S::N, NS = S::NS, CW = S::CW, BTC = S::BTC, BCP = S::BCP;
    constexpr int ESZ_D = S::ESZ_D, DROW = S::DROW, YROW = S::YROW;
    static_assert(!S::D_BF16 && !S::U_BF16, "the segmented backward runs on fp32 inputs");

    const int lane = threadIdx.x;
    if (a.nseg < 2 || a.seg_len < 1)
        return;
    int it = blockIdx.x;
    const int seg = it % a.nseg;
    it /= a.nseg;
    if (seg == 0)
        return;  // nothing is carried out of the first segment
    const int tile = it % a.tiles;
    it /= a.tiles;
    const int g = it % 4;
    const int b = it / 4;
    const int D = a.D, L = a.L;
    const int d0 = tile * CW;
    const int ch_valid = min(CW, D - d0);
    const int c0 = g * D + d0;
    const int ch = lane >> 1;
    const int q = lane & 1;
    const int cch = c0 + min(ch, ch_valid - 1);
    float a2[NS], cg[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) {
        a2[n] = -expf(__ldg(a.A_log + (size_t)cch * N + q + 2 * n)) * kLog2e;
        cg[n] = 0.0f;  // dA_{l+1} g_{l+1}, nothing at the segment's end
    }
    const float bias_ch = a.bias ? __ldg(a.bias + cch) : 0.0f;
    const bool rev = g >= 2;
    const float *ybase = (g & 1) ? a.dyT : a.dy;
    const size_t prow0 = ((size_t)b * D + d0) * L;
    const size_t drow0 = ((size_t)b * a.C + c0) * L;
    const float *Cg = a.Cm + ((size_t)b * 4 + g) * N * L;
    const char *dbase = reinterpret_cast<const char *>(a.dts);
    const uint64_t pol_once = l2_policy_evict_first();

    auto stage_chunk = [&](int j, int st) {
        unsigned char *rs = smem_raw + st * lay.stage_bytes;
        const int l0 = j * BTC;
        {   // C rows: 16 rows x 4 pieces of 16 bytes, into the C half of the B/C area
            const int v = (lane & 3) * 4;
            const int bytes = max(0, min(16, (L - l0 - v) * 4));
            float *dst = reinterpret_cast<float *>(rs + lay.off_bc);
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int row = (lane >> 2) + 8 * k;
                const float *src = Cg + (size_t)row * L + v;
                cp_async16(dst + (N + row) * BCP + v, bytes > 0 ? src + l0 : src, bytes);
            }
        }
        {
            constexpr int PER_ROW = BTC * ESZ_D / 16;
            for (int p = lane; p < CW * PER_ROW; p += 32) {
                const int chl = p / PER_ROW, v = p % PER_ROW;
                const int l = l0 + v * (16 / ESZ_D);
                const char *src = dbase + (drow0 + (size_t)min(chl, ch_valid - 1) * L) * ESZ_D;
                const int bytes = chl < ch_valid ? max(0, min(16, (L - l) * ESZ_D)) : 0;
                cp_async16_hint(rs + lay.off_d + chl * DROW + v * 16, bytes > 0 ? src + (size_t)l * ESZ_D : src,
                                bytes, pol_once);
            }
            constexpr int YPER_ROW = BTC * 4 / 16;
            for (int p = lane; p < CW * YPER_ROW; p += 32) {
                const int chl = p / YPER_ROW, v = p % YPER_ROW;
                const int e = (rev ? L - l0 - BTC : l0) + v * 4;
                const float *src = ybase + prow0 + (size_t)min(chl, ch_valid - 1) * L;
                const int bytes = (chl < ch_valid && e >= 0) ? max(0, min(16, (L - e) * 4)) : 0;
                cp_async16_hint(rs + lay.off_dy + chl * YROW + v * 16, bytes > 0 ? src + e : src, bytes, pol_once);
            }
        }
    };

    const int jbeg = seg * a.seg_len / BTC;  // seg_len is L (one segment) or a multiple of 32
    const int jend = min(a.nck, ((seg + 1) * a.seg_len + BTC - 1) / BTC);
    const int nck = jend - jbeg;
    float sd = 0.0f;  // sum of delta over the segment (this lane's channel)
    stage_chunk(jend - 1, 0);
    cp_async_commit();
    for (int jj = 0; jj < nck; ++jj) {
        const int j = jend - 1 - jj;
        const int l0 = j * BTC;
        const int valid = min(BTC, L - l0);  // a multiple of 4 (L % 4 == 0)
        const int st = jj & 1;
        const unsigned char *rs = smem_raw + st * lay.stage_bytes;
        cp_async_wait<0>();
        __syncwarp();
        if (jj + 1 < nck)
            stage_chunk(j - 1, st ^ 1);
        cp_async_commit();
        const float *bcs = reinterpret_cast<const float *>(rs + lay.off_bc);
        const float *drs = reinterpret_cast<const float *>(rs + lay.off_d + ch * DROW);
        const float *yrs = reinterpret_cast<const float *>(rs + lay.off_dy + ch * YROW);
#pragma unroll 1
        for (int m = valid / 4 - 1; m >= 0; --m) {
            const int i = 4 * m;
            const int s0 = i + 2 * q;
            const float2 zt = *reinterpret_cast<const float2 *>(drs + s0);
            const float d0v = softplus_f32(zt.x + bias_ch), d1v = softplus_f32(zt.y + bias_ch);
            const float pz0 = __shfl_xor_sync(0xffffffffu, d0v, 1), pz1 = __shfl_xor_sync(0xffffffffu, d1v, 1);
            const float4 dl4 = q ? make_float4(pz0, pz1, d0v, d1v) : make_float4(d0v, d1v, pz0, pz1);
            sd += (dl4.x + dl4.y) + (dl4.z + dl4.w);
            const float4 t = *reinterpret_cast<const float4 *>(yrs + (rev ? BTC - 4 - i : i));
            const float4 dy4 = rev ? make_float4(t.w, t.z, t.y, t.x) : t;
#pragma unroll
            for (int n = 0; n < NS; ++n) {
                const float4 cc = *reinterpret_cast<const float4 *>(bcs + (N + q + 2 * n) * BCP + i);
                float gg = fmaf(cc.w, dy4.w, cg[n]);
                float c = ex2_approx(dl4.w * a2[n]) * gg;
                gg = fmaf(cc.z, dy4.z, c);
                c = ex2_approx(dl4.z * a2[n]) * gg;
                gg = fmaf(cc.y, dy4.y, c);
                c = ex2_approx(dl4.y * a2[n]) * gg;
                gg = fmaf(cc.x, dy4.x, c);
                cg[n] = ex2_approx(dl4.x * a2[n]) * gg;
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    if (ch < ch_valid) {
        const size_t o = (((size_t)b * a.C + cch) * a.nseg + seg) * N + q;
#pragma unroll
        for (int n = 0; n < NS; ++n) {
            a.e_out[o + 2 * n] = cg[n];
            a.p_out[o + 2 * n] = ex2_approx(a2[n] * sd);
        }
    }
}

}  // namespace ss2d
