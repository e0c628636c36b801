// scan.cuh -- the selective-scan kernel of libss2d.
//
// Work item = one warp (one CTA): CW = (32 / TN) * CH consecutive channels of
// one (batch b, group g), walked over the whole sequence in chunks of TC
// steps.  Lane (grp, q) serves channels grp + k*(32/TN), k < CH, and holds
// states q, q + TN, q + 2TN, ... (NS = N / TN of them) of each in registers,
// so the recurrence
//     h[n] <- exp(delta A[n]) h[n] + delta B_l[n] u_l,   y_l = sum_n C_l[n] h[n] + D u_l
// (the selective scan called in section 3.2 of the VMamba SS2D article) runs
// sequentially in l with exactly one exponential per (step, state, channel),
// and every B/C value a lane loads from shared memory serves CH channels.
//
// Warps never wait for each other; each synchronises only with __syncwarp.
// Per chunk:
//   stage    B/C rows and delta rows of chunk j+1 are copied into the warp's
//            two-deep shared-memory ring with cp.async (16-byte row copies
//            where rows are aligned, 4-byte words otherwise), and u of chunk
//            j+1 is loaded into registers (lane = step, so u read through a
//            scan order of x costs one address per lane);
//   prepass  delta = softplus(dt + bias), delta*u and u of chunk j per
//            (channel, step) into the warp's shared memory (lane = step);
//   scan     per 4 steps each lane updates its states (exp2 on the MUFU,
//            packed fp32x2 multiplies over step pairs); the TN partial C.h of
//            each channel are reduce-scattered with shuffles;
//   write    y = C.h + D u is stored (standalone) or added into the merged
//            output at the pixel the direction visited at that step (the
//            CrossMerge of section 3.3 of the SS2D article).
#pragma once

#include "common.cuh"

namespace ss2d {

enum ScanMode { kStandalone = 0, kFused = 1, kFusedProj = 2 };

constexpr int kTC = 32;     // steps per chunk
constexpr int kMaxR = 16;       // largest dt_rank the scan fuses (dt_proj inside the scan loop)
constexpr int kMaxRLarge = 64;  // largest dt_rank of the projection path (above kMaxR dts is materialised)

// Element-type / softplus variants compiled in: bit 0 delta is bf16, bit 1 u is
// bf16, bit 2 softplus on.  kDtRuntime reads the three flags from ScanArgs.
constexpr int kDtRuntime = -1;

struct ScanArgs {
    const void *u;        // standalone: (B, C, L); fused: x (B, D, H, W)
    const void *uT;       // fused, optional: x with every (H, W) plane transposed, (B, D, W, H)
    const void *delta;    // (B, C, L) (fused: dts (B, 4, D, L), C = 4D); unused with projections
    const float *A_log;   // (C, N)
    const float *Bm;      // B rows: row n of group (b, g) at Bm + (b*G + g)*gs + n*L
    const float *Cm;      // C rows, same indexing
    const float *dtl;     // projections: dt_low rows r at dtl + (b*G + g)*gs + r*L
    const float *Wdt;     // projections: (G, per_group, R) dt_proj weights
    const float *Dv;      // (C) or null
    const float *bias;    // (C) or null
    float *y;             // standalone: (B, C, L); fused: (B, D, H, W), accumulated
    long long gs;         // floats between consecutive (b, g) row groups of Bm / Cm / dtl
    int B, C, G, L;
    int per_group;        // C / G (fused: D)
    int tiles;            // ceil(per_group / CW): warp work items per group
    int W;                // fused: image width
    SmallDiv divH;        // fused: division by the image height
    int R;                // projections: dt_rank
    int u_bf16, delta_bf16;
    int softplus;
    int ch_last;          // fused: x and y channels-last, (B, H, W, D) (the N = 16 kernel only)
    size_t delta_bytes;   // size of the delta tensor (bound of the 4-byte copies of misaligned rows)
    // shared-memory layout (bytes), set by the launcher
    int d_rows;           // 1: delta rows are 16-byte aligned (packed 16-byte copies); 0: 4-byte words
    int stage_bytes, off_bc, off_d, off_t, off_dl, off_du, off_us, off_pix, off_wdt, off_par, smem_bytes;
    int drow_bytes;
    // Long sequences split into segments (the two passes of scan2_kernel): segment s covers
    // steps [s*seg_len, min(L, (s+1)*seg_len)).  nseg = 1 scans whole sequences.
    int nseg, seg_len;
    const float *h0;      // (B, C, nseg, N) initial states per segment, or null for zero
    float *hend;          // first pass: (B, C, nseg, N) states after each segment from a zero start
    float *pend;          // first pass: (B, C, nseg, N) product of the decays over each segment
    float *hlast;         // whole-sequence scans: (B, C, N) state after the last step, or null
    // Direction range of a launch (the N = 16 kernel): groups g0 .. g0 + gn - 1 (gn <= 0: all G),
    // and how its outputs enter y: 0 atomic add, 1 plain store, 2 plain load-add-store (a launch
    // per direction, in a fixed order, makes the merge deterministic).
    int g0, gn, merge;
    float *ckpt;          // checkpoint pass, or a fused N = 16 forward that keeps them for its backward:
                          // (B, C, ceil(L/16), 16) state before step 16j, the state q + 2n (q = 0, 1)
                          // stored at q*8 + n
    // Fused N = 16 scan, direct form: when ydir[0] is set, direction g stores its output (each
    // element once, no atomics) into ydir[g], laid out as y, instead of merging into y.
    float *ydir[4];
};

template <int N_, int TN_, int CH_, int MINB_, int MODE_, int DT_>
struct ScanShape {
    static constexpr int N = N_;
    static constexpr int TN = TN_;                // lanes per channel
    static constexpr int NS = N_ / TN_;           // states per lane and channel
    static constexpr int CH = CH_;                // channels per lane
    static constexpr int GW = 32 / TN_;           // lane groups per warp
    static constexpr int CW = GW * CH_;           // channels per warp
    static constexpr int MINB = MINB_;
    static constexpr int MODE = MODE_;
    static constexpr int DT = DT_;
    static constexpr int BCP = kTC + 4;           // B/C ring row pitch (floats)
    static constexpr int XP = kTC + 4;            // dl / du / us row pitch (floats)
    static_assert(TN_ == 1 || TN_ == 2 || TN_ == 4, "1, 2 or 4 lanes per channel");
    static_assert(N_ % TN_ == 0, "TN must divide N");
    static_assert(CH_ >= 1 && CH_ <= 4, "1..4 channels per lane");

    // delta ring row: TC elements plus 16 bytes (room for the extra word of a misaligned row)
    static constexpr __host__ __device__ int drow_bytes_for(int esz_d) { return esz_d == 2 ? 80 : 144; }

    // Shared-memory layout for the given element types (host side).
    static void layout(ScanArgs &a)
    {
        const int esz_d = a.delta_bf16 ? 2 : 4;
        a.d_rows = ((size_t)a.L * esz_d) % 16 == 0;
        a.drow_bytes = drow_bytes_for(esz_d);
        int off = 0;
        a.off_bc = off;
        off += 2 * N_ * BCP * 4;
        a.off_d = off;
        off += (MODE_ == kFusedProj) ? 0 : CW * a.drow_bytes;
        a.off_t = off;
        off += (MODE_ == kFusedProj) ? kMaxR * BCP * 4 : 0;
        a.stage_bytes = (off + 15) & ~15;
        off = 2 * a.stage_bytes;
        a.off_dl = off;
        off += CW * XP * 4;
        a.off_du = off;
        off += CW * XP * 4;
        a.off_us = off;
        off += CW * XP * 4;
        a.off_pix = off;
        off += 2 * kTC * 4;
        a.off_wdt = off;
        off += (MODE_ == kFusedProj) ? CW * kMaxR * 4 : 0;
        a.off_par = off;
        off += 2 * CW * 4;
        a.smem_bytes = (off + 15) & ~15;
    }
};

template <class S>
__global__ void __launch_bounds__(32, S::MINB) scan_kernel(const ScanArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    constexpr int N = S::N, NS = S::NS, TN = S::TN, CH = S::CH, GW = S::GW, CW = S::CW, MODE = S::MODE,
                  BCP = S::BCP, XP = S::XP, TC = kTC, DT = S::DT;

    const bool d_bf16 = (DT >= 0) ? (DT & 1) != 0 : a.delta_bf16 != 0;
    const bool u_bf16 = (DT >= 0) ? (DT & 2) != 0 : a.u_bf16 != 0;
    const bool softplus = (DT >= 0) ? (DT & 4) != 0 : a.softplus != 0;
    const int esz_d = d_bf16 ? 2 : 4;
    const int drowb = (DT >= 0) ? S::drow_bytes_for(esz_d) : a.drow_bytes;

    const int lane = threadIdx.x;
    float *dlr = reinterpret_cast<float *>(smem_raw + a.off_dl);
    float *dur = reinterpret_cast<float *>(smem_raw + a.off_du);
    float *usr = reinterpret_cast<float *>(smem_raw + a.off_us);
    int *pixr = reinterpret_cast<int *>(smem_raw + a.off_pix);
    float *wdt = reinterpret_cast<float *>(smem_raw + a.off_wdt);
    float *biasr = reinterpret_cast<float *>(smem_raw + a.off_par);
    float *dskr = biasr + CW;

    if (a.nseg < 1 || a.seg_len < 1)
        return;  // launchers always set at least one segment covering the sequence
    int it = blockIdx.x;
    const int seg = it % a.nseg;
    it /= a.nseg;
    const int tile = it % a.tiles;
    it /= a.tiles;
    const int g = it % a.G;
    const int b = it / a.G;
    const int d0 = tile * CW;
    const int ch_valid = min(CW, a.per_group - d0);
    const bool full_warp = ch_valid == CW;
    const int c0 = g * a.per_group + d0;
    const int L = a.L;
    const int R = (MODE == kFusedProj) ? a.R : 0;
    const int lbeg = seg * a.seg_len;
    const int lend = min(L, lbeg + a.seg_len);

    // Scan role of this lane: channels grp + k*GW, states q + TN*n.
    const int grp = lane / TN;
    const int q = lane % TN;
    float a2[CH][NS], h[CH][NS];
#pragma unroll
    for (int k = 0; k < CH; ++k) {
        const int c = c0 + min(grp + k * GW, ch_valid - 1);
#pragma unroll
        for (int n = 0; n < NS; ++n) {
            a2[k][n] = -expf(__ldg(a.A_log + (size_t)c * N + q + TN * n)) * kLog2e;
            h[k][n] = a.h0 ? __ldg(a.h0 + (((size_t)b * a.C + c) * a.nseg + seg) * N + q + TN * n) : 0.0f;
        }
    }
    for (int c = lane; c < CW; c += 32) {
        const bool ok = c < ch_valid;
        biasr[c] = (ok && a.bias) ? __ldg(a.bias + c0 + c) : 0.0f;
        dskr[c] = (ok && a.Dv) ? __ldg(a.Dv + c0 + c) : 0.0f;
    }
    if (MODE == kFusedProj) {
        for (int e = lane; e < CW * kMaxR; e += 32) {
            const int c = e / kMaxR, r = e % kMaxR;
            wdt[e] = (c < ch_valid && r < R) ? a.Wdt[((size_t)g * a.per_group + d0 + c) * R + r] : 0.0f;
        }
    }

    const size_t grow = (size_t)b * a.G + g;
    const float *Bg = a.Bm + grow * a.gs;
    const float *Cg = a.Cm + grow * a.gs;
    const float *Tg = (MODE == kFusedProj) ? a.dtl + grow * a.gs : nullptr;
    const bool rows16 = (L & 3) == 0;  // fp32 rows are 16-byte aligned at every multiple of 4 steps
    const char *dbase = reinterpret_cast<const char *>(a.delta);

    // Per-lane source rows of the 16-byte B/C copies: piece p = lane + 32k covers row
    // p / 8 (B rows first, then C rows) and 4 steps at (p % 8) * 4.
    constexpr int BC_PIECES = 2 * N * (TC / 4);
    const int v4 = (lane & 7) * 4;

    // ---- staging of one chunk into ring stage `st` ------------------------
    auto stage_chunk = [&](int l0, int st) {
        unsigned char *rs = smem_raw + st * a.stage_bytes;
        if (MODE != kStandalone) {
            const int l = l0 + lane;
            pixr[st * TC + lane] = (l < L) ? scan_pixel(g, l, L, a.W, a.divH) : 0;
        }
        // B and C rows
        float *bcd = reinterpret_cast<float *>(rs + a.off_bc);
        if (rows16) {
            const int bytes = max(0, min(16, (L - l0 - v4) * 4));
#pragma unroll
            for (int k = 0; k < (BC_PIECES + 31) / 32; ++k) {
                const int row = (lane >> 3) + 4 * k;
                if (BC_PIECES % 32 == 0 || row < 2 * N) {
                    const float *src = (row < N ? Bg + (size_t)row * L : Cg + (size_t)(row - N) * L) + v4;
                    cp_async16(bcd + row * BCP + v4, bytes > 0 ? src + l0 : src, bytes);
                }
            }
        } else {
            for (int p = lane; p < 2 * N * TC; p += 32) {
                const int r = p / TC, v = p % TC, l = l0 + v;
                const float *src = r < N ? Bg + (size_t)r * L : Cg + (size_t)(r - N) * L;
                cp_async4(bcd + r * BCP + v, l < L ? src + l : src, l < L ? 4 : 0);
            }
        }
        // delta rows
        if (MODE != kFusedProj) {
            unsigned char *ddst = rs + a.off_d;
            if (a.d_rows) {
                const int per_row = TC * esz_d / 16;
                for (int p = lane; p < CW * per_row; p += 32) {
                    const int chl = p / per_row, v = p % per_row;
                    const int l = l0 + v * 16 / esz_d;
                    const size_t row = (size_t)b * a.C + c0 + min(chl, ch_valid - 1);
                    const char *src = dbase + row * L * esz_d;
                    const int bytes = (chl < ch_valid) ? max(0, min(16, (L - l) * esz_d)) : 0;
                    cp_async16(ddst + chl * drowb + v * 16, bytes > 0 ? src + (size_t)l * esz_d : src, bytes);
                }
            } else {
                const int per_row = TC * esz_d / 4 + 1;
                for (int p = lane; p < CW * per_row; p += 32) {
                    const int chl = p / per_row, v = p % per_row;
                    const size_t row = (size_t)b * a.C + c0 + min(chl, ch_valid - 1);
                    const size_t start = ((row * L + l0) * esz_d) & ~(size_t)3;
                    const size_t off = start + (size_t)v * 4;
                    const size_t end = (row * L + (size_t)L) * esz_d;
                    const int ok = (chl < ch_valid && off < end) ? (int)min((size_t)4, a.delta_bytes - off) : 0;
                    cp_async4(ddst + chl * drowb + v * 4, dbase + (ok ? off : start), ok);
                }
            }
        }
        // dt_low rows (projections)
        if (MODE == kFusedProj) {
            float *td = reinterpret_cast<float *>(rs + a.off_t);
            for (int p = lane; p < R * (TC / 4); p += 32) {
                const int r = p / (TC / 4), v = p % (TC / 4), l = l0 + 4 * v;
                const float *src = Tg + (size_t)r * L;
                if (rows16) {
                    const int bytes = max(0, min(16, (L - l) * 4));
                    cp_async16(td + r * BCP + 4 * v, bytes > 0 ? src + l : src, bytes);
                } else {
                    for (int k = 0; k < 4; ++k)
                        cp_async4(td + r * BCP + 4 * v + k, l + k < L ? src + l + k : src, l + k < L ? 4 : 0);
                }
            }
        }
    };

    // u of chunk l0 for step `lane` and every channel of the warp, loaded into registers one
    // chunk ahead.  Lane = step, so the pixel offset is computed once per lane and chunk.
    float ureg[CW];
    auto load_u = [&](int l0, int st) {
        const int l = l0 + lane;
        const bool ok = l < L;
        size_t el;
        if (MODE == kStandalone)
            el = ((size_t)b * a.C + c0) * L + (ok ? l : 0);
        else
            el = ((size_t)b * a.per_group + d0) * L + (ok ? pixr[st * TC + lane] : 0);
        if (u_bf16) {
            const __nv_bfloat16 *p = reinterpret_cast<const __nv_bfloat16 *>(a.u) + el;
#pragma unroll
            for (int chl = 0; chl < CW; ++chl)
                ureg[chl] = (ok && chl < ch_valid) ? __bfloat162float(__ldg(p + (size_t)chl * L)) : 0.0f;
        } else {
            const float *p = reinterpret_cast<const float *>(a.u) + el;
#pragma unroll
            for (int chl = 0; chl < CW; ++chl)
                ureg[chl] = (ok && chl < ch_valid) ? __ldg(p + (size_t)chl * L) : 0.0f;
        }
    };

    const int nchunks = (lend - lbeg + TC - 1) / TC;
    stage_chunk(lbeg, 0);
    cp_async_commit();
    __syncwarp();
    load_u(lbeg, 0);

    for (int j = 0; j < nchunks; ++j) {
        const int l0 = lbeg + j * TC;
        const int valid = min(TC, lend - l0);
        const int st = j & 1;
        const unsigned char *rs = smem_raw + st * a.stage_bytes;

        cp_async_wait<0>();
        __syncwarp();
        if (j + 1 < nchunks)
            stage_chunk(l0 + TC, st ^ 1);
        cp_async_commit();

        // ---- prepass: delta, delta*u, u (lane = step, loop over channels) -----
        {
            const int i = lane;
            const bool full = full_warp && valid == TC;
            const float *tsrc = reinterpret_cast<const float *>(rs + a.off_t);
            const unsigned char *drow = rs + a.off_d + i * esz_d;
            int dshift = 0;
            int rowshift = 0;
            if (MODE != kFusedProj && !a.d_rows) {
                // byte misalignment of this chunk's start in channel row c0 + chl
                dshift = (int)(((((size_t)b * a.C + c0) * L + l0) * esz_d) & 3);
                rowshift = (int)(((size_t)L * esz_d) & 3);
            }
            if (MODE != kFusedProj && full && a.d_rows) {
                // every channel and step valid, delta rows aligned: no masks, no misalignment shifts
#pragma unroll
                for (int chl = 0; chl < CW; ++chl) {
                    const unsigned char *p = drow + chl * drowb;
                    float dv = d_bf16 ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p))
                                      : *reinterpret_cast<const float *>(p);
                    dv += biasr[chl];
                    if (softplus)
                        dv = softplus_f32(dv);
                    const float uv = ureg[chl];
                    dlr[chl * XP + i] = dv;
                    dur[chl * XP + i] = dv * uv;
                    usr[chl * XP + i] = uv;
                }
            } else {
#pragma unroll
                for (int chl = 0; chl < CW; ++chl) {
                    float dv;
                    if (MODE == kFusedProj) {
                        dv = 0.0f;
                        for (int r = 0; r < R; ++r)
                            dv = fmaf(wdt[chl * kMaxR + r], tsrc[r * BCP + i], dv);
                    } else {
                        const int cc = min(chl, ch_valid - 1);
                        const int sh = (dshift + cc * rowshift) & 3;
                        const unsigned char *p = drow + chl * drowb + sh;
                        dv = d_bf16 ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p))
                                    : *reinterpret_cast<const float *>(p);
                    }
                    dv += biasr[chl];
                    if (softplus)
                        dv = softplus_f32(dv);
                    float uv = ureg[chl];
                    if (!full && (chl >= ch_valid || i >= valid)) {
                        dv = 0.0f;
                        uv = 0.0f;
                    }
                    dlr[chl * XP + i] = dv;
                    dur[chl * XP + i] = dv * uv;
                    usr[chl * XP + i] = uv;
                }
            }
        }
        __syncwarp();
        if (j + 1 < nchunks)
            load_u(l0 + TC, st ^ 1);

        // ---- scan ----------------------------------------------------------
        {
            const float *bcs = reinterpret_cast<const float *>(rs + a.off_bc);
            const int nsteps = (valid + 3) & ~3;
            for (int i = 0; i < nsteps; i += 4) {
                float4 dl[CH], du[CH];
#pragma unroll
                for (int k = 0; k < CH; ++k) {
                    dl[k] = *reinterpret_cast<const float4 *>(dlr + (grp + k * GW) * XP + i);
                    du[k] = *reinterpret_cast<const float4 *>(dur + (grp + k * GW) * XP + i);
                }
                float2 y01[CH], y23[CH];
#pragma unroll
                for (int k = 0; k < CH; ++k) {
                    y01[k] = make_float2(0.0f, 0.0f);
                    y23[k] = make_float2(0.0f, 0.0f);
                }
#pragma unroll
                for (int n = 0; n < NS; ++n) {
                    const int sr = q + TN * n;
                    const float4 bb = *reinterpret_cast<const float4 *>(bcs + sr * BCP + i);
                    const float4 cv = *reinterpret_cast<const float4 *>(bcs + (N + sr) * BCP + i);
                    const float2 b01 = make_float2(bb.x, bb.y), b23 = make_float2(bb.z, bb.w);
                    const float2 c01 = make_float2(cv.x, cv.y), c23 = make_float2(cv.z, cv.w);
#pragma unroll
                    for (int k = 0; k < CH; ++k) {
                        const float2 an = make_float2(a2[k][n], a2[k][n]);
                        const float2 x01 = __fmul2_rn(make_float2(dl[k].x, dl[k].y), an);
                        const float2 x23 = __fmul2_rn(make_float2(dl[k].z, dl[k].w), an);
                        const float2 bu01 = __fmul2_rn(make_float2(du[k].x, du[k].y), b01);
                        const float2 bu23 = __fmul2_rn(make_float2(du[k].z, du[k].w), b23);
                        float2 h01, h23;
                        const float e0 = ex2_approx(x01.x), e1 = ex2_approx(x01.y);
                        const float e2 = ex2_approx(x23.x), e3 = ex2_approx(x23.y);
                        h01.x = fmaf(e0, h[k][n], bu01.x);
                        h01.y = fmaf(e1, h01.x, bu01.y);
                        h23.x = fmaf(e2, h01.y, bu23.x);
                        h23.y = fmaf(e3, h23.x, bu23.y);
                        h[k][n] = h23.y;
                        y01[k] = __ffma2_rn(c01, h01, y01[k]);
                        y23[k] = __ffma2_rn(c23, h23, y23[k]);
                    }
                }
#pragma unroll
                for (int k = 0; k < CH; ++k) {
                    float *ys_row = dlr + (grp + k * GW) * XP;  // y of a step overwrites its delta
                    const float yv0 = y01[k].x, yv1 = y01[k].y, yv2 = y23[k].x, yv3 = y23[k].y;
                    if (TN == 1) {
                        *reinterpret_cast<float4 *>(ys_row + i) = make_float4(yv0, yv1, yv2, yv3);
                    } else if (TN == 2) {
                        const bool hi = q & 1;
                        float k0 = hi ? yv2 : yv0, k1 = hi ? yv3 : yv1;
                        const float s0 = hi ? yv0 : yv2, s1 = hi ? yv1 : yv3;
                        k0 += __shfl_xor_sync(0xffffffffu, s0, 1);
                        k1 += __shfl_xor_sync(0xffffffffu, s1, 1);
                        *reinterpret_cast<float2 *>(ys_row + i + 2 * q) = make_float2(k0, k1);
                    } else {
                        const bool hi = q & 2;
                        float k0 = hi ? yv2 : yv0, k1 = hi ? yv3 : yv1;
                        const float s0 = hi ? yv0 : yv2, s1 = hi ? yv1 : yv3;
                        k0 += __shfl_xor_sync(0xffffffffu, s0, 2);
                        k1 += __shfl_xor_sync(0xffffffffu, s1, 2);
                        const bool lo = q & 1;
                        float kk = lo ? k1 : k0;
                        const float sd = lo ? k0 : k1;
                        kk += __shfl_xor_sync(0xffffffffu, sd, 1);
                        ys_row[i + q] = kk;
                    }
                }
            }
        }
        __syncwarp();

        // ---- write-out (lane = step, loop over channels) -------------------
        {
            const int i = lane;
            if (i < valid) {
                if (MODE == kStandalone) {
                    float *yp = a.y + ((size_t)b * a.C + c0) * L + l0 + i;
#pragma unroll
                    for (int chl = 0; chl < CW; ++chl) {
                        if (full_warp || chl < ch_valid)
                            *yp = fmaf(dskr[chl], usr[chl * XP + i], dlr[chl * XP + i]);
                        yp += L;
                    }
                } else {
                    float *yp = a.y + ((size_t)b * a.per_group + d0) * L + pixr[st * TC + i];
#pragma unroll
                    for (int chl = 0; chl < CW; ++chl) {
                        if (full_warp || chl < ch_valid)
                            atomicAdd(yp, fmaf(dskr[chl], usr[chl * XP + i], dlr[chl * XP + i]));
                        yp += L;
                    }
                }
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    if (a.hlast) {
        // state after the last step (padding steps past L ran with delta = 0 and left it unchanged)
#pragma unroll
        for (int k = 0; k < CH; ++k) {
            const int ch = grp + k * GW;
            if (ch < ch_valid) {
                const size_t o = ((size_t)b * a.C + c0 + ch) * N + q;
#pragma unroll
                for (int n = 0; n < NS; ++n)
                    a.hlast[o + TN * n] = h[k][n];
            }
        }
    }
}

}  // namespace ss2d
