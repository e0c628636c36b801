// scan2.cuh -- the N = 16 selective-scan kernel with delta computed inside the scan loop.
//
// Same recurrence and outputs as scan_kernel (the selective scan called in
// section 3.2 of the VMamba SS2D article, optionally with the CrossMerge of
// section 3.3 folded into its write-out), arranged for fewer instructions per
// element.  One warp (one CTA) owns 16 channels of one (batch, group); lanes 2c
// and 2c+1 serve channel c and hold its states q, q+2, ..., q+14 (q = lane & 1).
// Per chunk of 32 steps:
//   stage  B/C rows, delta rows (or dt_low rows) and u rows of chunk j+1 are
//          copied into the warp's two-deep shared-memory ring with cp.async;
//          u of the column-major scan orders comes from x with its planes
//          transposed (rows in the order of direction 1, read forwards or
//          backwards) when the caller provides that copy, else it is gathered
//          from x one step per lane into registers one chunk ahead;
//   scan   per 4 steps lane (c, q) computes delta = softplus(dt + bias) and
//          delta*u of steps i+2q and i+2q+1 and swaps them with its partner by
//          shuffle, so softplus runs exactly once per element; then both lanes
//          run the 4 steps over their 8 states (exp2 on the MUFU, fp32x2
//          multiplies over step pairs) and reduce-scatter C.h with one shuffle
//          level, each lane adding D*u of the two steps it keeps;
//   write  lane = step: y is stored (standalone) or added into the merged
//          output at the pixel the direction visited at that step.
// Steps past the end of the sequence and channels past the end of the group
// run on zero-filled B, C, u and dt (their results are never written), so the
// loop needs no masks.
//
// Long sequences with few channels are split into segments of a multiple of 32
// steps (ScanArgs::nseg, seg_len), scanned in two passes around a carry:
// SEGP_ = 1 builds the first pass, which keeps no output and records for every
// segment but the last the state reached from a zero start and the product of
// its decays, exp(A * sum of delta over the segment); the second pass
// (SEGP_ = 0 with ScanArgs::h0) scans every segment from its carried-in state.
// SEGP_ = 2 builds the checkpoint pass of the backward scan: no output, and the
// state before every 16th step stored in ScanArgs::ckpt.  SEGP_ = 3 stores the same
// checkpoints from a normal (output-producing) pass: a forward that keeps what its
// backward will need.
//
// CL_ = 1 builds the fused core for channels-last x and y, (B, H, W, D): the 16
// channels of a warp at one pixel are one contiguous run, so u of every scan
// order is staged as one run per step (lane = step), and the merge adds each
// step's 16 channels as one contiguous run as well.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "scan.cuh"

namespace ss2d {

// Shared-memory layout of one scan2_kernel CTA (byte offsets).
struct Scan2Layout {
    int stage_bytes, off_bc, off_d, off_u, off_t, off_ys, off_pix, smem_bytes;
};

// MODE: kStandalone, kFused or kFusedProj.  DT_: bit 0 delta is bf16, bit 1 u is
// bf16, bit 2 softplus on (compiled in; the projection form has no delta input).
template <int MODE_, int DT_, int SEGP_ = 0, int CL_ = 0>
struct Scan2Shape {
    static constexpr int N = 16;
    static constexpr int NS = 8;     // states per lane
    static constexpr int CW = 16;    // channels per warp
    static constexpr int MODE = MODE_;
    static constexpr int SEGP = SEGP_;
    static constexpr bool CL = CL_ != 0;
    static constexpr bool D_BF16 = (DT_ & 1) != 0;
    static constexpr bool U_BF16 = (DT_ & 2) != 0;
    static constexpr bool SOFTPLUS = (DT_ & 4) != 0;
    static constexpr int ESZ_D = D_BF16 ? 2 : 4;
    static constexpr int ESZ_U = U_BF16 ? 2 : 4;
    static constexpr int BCP = kTC + 4;             // B/C/dt_low row pitch (floats)
    static constexpr int DROW = kTC * ESZ_D + 16;   // delta row pitch (bytes; one spare word for misaligned rows)
    static constexpr int UROW = kTC * ESZ_U + 16;   // u row pitch (bytes)
    static constexpr int UCP = CW * ESZ_U + 16;     // channels-last u: pitch of one step's channel run (bytes)
    static constexpr int YP = kTC + 4;              // y row pitch (floats)

    static Scan2Layout layout()
    {
        Scan2Layout l{};
        int off = 0;
        l.off_bc = off;
        off += 2 * N * BCP * 4;
        l.off_d = off;
        off += (MODE_ == kFusedProj) ? 0 : CW * DROW;
        l.off_u = off;
        off += CL_ ? kTC * UCP : CW * UROW;
        l.off_t = off;
        off += (MODE_ == kFusedProj) ? kMaxR * BCP * 4 : 0;
        l.stage_bytes = (off + 15) & ~15;
        off = 2 * l.stage_bytes;
        l.off_ys = off;
        off += CW * YP * 4;
        l.off_pix = off;
        off += 2 * kTC * 4;
        l.smem_bytes = (off + 15) & ~15;
        return l;
    }
};

// How u of a chunk reaches the ring (uniform per CTA).
enum ScanURows { kURows = 0, kURowsReversed = 1, kUGather = 2 };

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Where direction g's output goes: merged into y, or (the direct form's page-order merge with
// channels-last y) stored into its own buffer ydir[g]; and how it enters there
// (ScanArgs::merge, or a plain store into the own buffer).  Read from the arguments where used.
template <int MODE>
__device__ __forceinline__ float *scan2_out(const ScanArgs &a, int g)
{
    if constexpr (MODE == kFused) {
        if (a.ydir[0])
            return g == 0 ? a.ydir[0] : g == 1 ? a.ydir[1] : g == 2 ? a.ydir[2] : a.ydir[3];
    }
    return a.y;
}

template <int MODE>
__device__ __forceinline__ int scan2_merge_mode(const ScanArgs &a)
{
    if constexpr (MODE == kFused) {
        if (a.ydir[0])
            return 1;
    }
    return a.merge;
}

// The direct form's page-order merge with channel-first y: every direction stores its output
// in scan order, (B, 4D, L) at ydir[0] like the standalone scan's y, for a CrossMerge pass.
template <int MODE, bool CL>
__device__ __forceinline__ bool scan2_scan_order_out(const ScanArgs &a)
{
    if constexpr (MODE == kFused && !CL)
        return a.ydir[0] != nullptr;
    return false;
}

template <class S>
__global__ void __launch_bounds__(32, 12) scan2_kernel(const ScanArgs a, const Scan2Layout lay)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    constexpr int N = S::N, NS = S::NS, CW = S::CW, MODE = S::MODE, BCP = S::BCP, YP = S::YP, TC = kTC;
    constexpr int ESZ_D = S::ESZ_D, ESZ_U = S::ESZ_U, DROW = S::DROW, UROW = S::UROW, UCP = S::UCP;
    constexpr bool CL = S::CL;
    constexpr bool U_BF16 = S::U_BF16, D_BF16 = S::D_BF16;
    constexpr bool SEGP = S::SEGP == 1;   // first pass of a segmented scan
    constexpr bool CKPT = S::SEGP >= 2;   // states before every 16th step into a.ckpt
    constexpr bool NOOUT = SEGP || S::SEGP == 2;  // no C, no readout, no write-out
    using UT = typename std::conditional<U_BF16, unsigned short, float>::type;

    const int lane = threadIdx.x;
    float *ysr = reinterpret_cast<float *>(smem_raw + lay.off_ys);
    int *pixr = reinterpret_cast<int *>(smem_raw + lay.off_pix);

    if (a.nseg < 1 || a.seg_len < 1)
        return;  // launchers always set at least one segment covering the sequence
    int it = blockIdx.x;
    const int seg = it % a.nseg;
    it /= a.nseg;
    const int tile = it % a.tiles;
    it /= a.tiles;
    const int gn = a.gn > 0 ? a.gn : a.G;
    const int g = a.g0 + it % gn;
    const int b = it / gn;
    const int d0 = tile * CW;
    const int ch_valid = min(CW, a.per_group - d0);
    const bool full_warp = ch_valid == CW;
    const int c0 = g * a.per_group + d0;
    const int L = a.L;
    const int R = (MODE == kFusedProj) ? a.R : 0;
    const int lbeg = seg * a.seg_len;
    const int lend = min(L, lbeg + a.seg_len);
    if (SEGP && lend == L)
        return;  // the first pass needs no summary of the last segment

    // u staging: 16-byte row copies when rows are 16-byte aligned and the scan walks them
    // in (reverse) storage order -- x for the row-major orders, its transposed planes (when
    // given) for the column-major ones -- and one-step-per-lane gathers from x otherwise.
    const bool col_rows = MODE != kStandalone && (g & 1) && a.uT;
    int umode = kUGather;
    if (CL) {
        umode = kURows;  // unused: channels-last u is staged per step below
    } else if ((((size_t)L * ESZ_U) & 15) == 0) {
        if (MODE == kStandalone || g == 0 || (g == 1 && col_rows))
            umode = kURows;
        else if (g == 2 || (g == 3 && col_rows))
            umode = kURowsReversed;
    }
    const bool drows = (((size_t)L * ESZ_D) & 15) == 0;
    // 16-byte merge write-out: in the row-major scan orders four consecutive steps visit four
    // consecutive, 16-byte-aligned pixels of y
    const bool vec_merge = MODE != kStandalone && !CL && (L & 3) == 0 && (g == 0 || g == 2);


    // This lane: channel ch (clamped to a valid one for parameters), states q + 2n.
    const int ch = lane >> 1;
    const int q = lane & 1;
    const int cch = c0 + min(ch, ch_valid - 1);
    float a2[NS], h[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) {
        a2[n] = -expf(__ldg(a.A_log + (size_t)cch * N + q + 2 * n)) * kLog2e;
        h[n] = a.h0 ? __ldg(a.h0 + (((size_t)b * a.C + cch) * a.nseg + seg) * N + q + 2 * n) : 0.0f;
    }
    const float bias_ch = a.bias ? __ldg(a.bias + cch) : 0.0f;
    const float dsk_ch = a.Dv ? __ldg(a.Dv + cch) : 0.0f;
    float wdt[MODE == kFusedProj ? kMaxR : 1];
    if constexpr (MODE == kFusedProj) {
#pragma unroll
        for (int r = 0; r < kMaxR; ++r)
            wdt[r] = r < R ? __ldg(a.Wdt + (size_t)cch * R + r) : 0.0f;
    }

    const size_t grow = (size_t)b * a.G + g;
    const float *Bg = a.Bm + grow * a.gs;
    const float *Cg = a.Cm + grow * a.gs;
    const float *Tg = (MODE == kFusedProj) ? a.dtl + grow * a.gs : nullptr;
    const bool rows16 = (L & 3) == 0;  // fp32 rows are 16-byte aligned at every multiple of 4 steps
    const int v4 = (lane & 7) * 4;
    const char *dbase = reinterpret_cast<const char *>(a.delta);
    const char *ubase = reinterpret_cast<const char *>(col_rows ? a.uT : a.u);  // row staging source
    // element index of (channel row d0 / c0, step or pixel 0) in u
    const size_t urow0 = (MODE == kStandalone) ? ((size_t)b * a.C + c0) * L : ((size_t)b * a.per_group + d0) * L;
    // element index of (channel row c0, step 0) in delta
    const size_t drow0 = ((size_t)b * a.C + c0) * L;
    // L2 priorities: delta is read exactly once, so its lines go first; the merged output
    // takes four read-modify-write passes spread over the whole kernel, so its lines stay.
    const uint64_t pol_once = l2_policy_evict_first();
    const uint64_t pol_keep = l2_policy_evict_last();

    // Rows [0, nrows) of fp32 tensors: row r < split from base0 + r*L, else base1 + (r - split)*L.
    auto stage_rows_f32 = [&](float *dst, int nrows, const float *base0, const float *base1, int split, int l0) {
        if (rows16) {
            const int bytes = max(0, min(16, (L - l0 - v4) * 4));
            for (int row = lane >> 3; row < nrows; row += 4) {
                const float *src = (row < split ? base0 + (size_t)row * L : base1 + (size_t)(row - split) * L) + v4;
                cp_async16(dst + row * BCP + v4, bytes > 0 ? src + l0 : src, bytes);
            }
        } else {
            for (int p = lane; p < nrows * TC; p += 32) {
                const int r = p / TC, v = p % TC, l = l0 + v;
                const float *src = r < split ? base0 + (size_t)r * L : base1 + (size_t)(r - split) * L;
                cp_async4(dst + r * BCP + v, l < L ? src + l : src, l < L ? 4 : 0);
            }
        }
    };

    auto stage_chunk = [&](int l0, int st) {
        unsigned char *rs = smem_raw + st * lay.stage_bytes;
        if (MODE != kStandalone) {
            const int l = l0 + lane;
            pixr[st * TC + lane] = (l < L) ? scan_pixel(g, l, L, a.W, a.divH) : 0;
        }
        if (rows16) {
            // B and C rows: lane covers 4 steps at v4 of rows (lane >> 3) + 4k of each
            const int bytes = max(0, min(16, (L - l0 - v4) * 4));
            float *dst = reinterpret_cast<float *>(rs + lay.off_bc) + (lane >> 3) * BCP + v4;
            const float *sb = Bg + (size_t)(lane >> 3) * L + v4 + (bytes > 0 ? l0 : 0);
            const float *sc = Cg + (size_t)(lane >> 3) * L + v4 + (bytes > 0 ? l0 : 0);
            const size_t rows4 = (size_t)4 * L;
#pragma unroll
            for (int k = 0; k < N / 4; ++k) {
                cp_async16(dst + 4 * k * BCP, sb, bytes);
                if (!NOOUT)
                    cp_async16(dst + (N + 4 * k) * BCP, sc, bytes);
                sb += rows4;
                sc += rows4;
            }
        } else {
            stage_rows_f32(reinterpret_cast<float *>(rs + lay.off_bc), NOOUT ? N : 2 * N, Bg, Cg, N, l0);
        }
        if (MODE == kFusedProj)
            stage_rows_f32(reinterpret_cast<float *>(rs + lay.off_t), R, Tg, Tg, R, l0);
        if (MODE != kFusedProj) {
            unsigned char *ddst = rs + lay.off_d;
            if (drows) {
                constexpr int PER_ROW = TC * ESZ_D / 16;
                for (int p = lane; p < CW * PER_ROW; p += 32) {
                    const int chl = p / PER_ROW, v = p % PER_ROW;
                    const int l = l0 + v * (16 / ESZ_D);
                    const char *src = dbase + (drow0 + (size_t)min(chl, ch_valid - 1) * L) * ESZ_D;
                    const int bytes = chl < ch_valid ? max(0, min(16, (L - l) * ESZ_D)) : 0;
                    cp_async16_hint(ddst + chl * DROW + v * 16, bytes > 0 ? src + (size_t)l * ESZ_D : src, bytes,
                                    pol_once);
                }
            } else {
                // rows not 16-byte aligned: the 4-byte words covering the chunk, from the word
                // holding its first element (read back with the byte offset of that element)
                constexpr int PER_ROW = TC * ESZ_D / 4 + 1;
                for (int p = lane; p < CW * PER_ROW; p += 32) {
                    const int chl = p / PER_ROW, v = p % PER_ROW;
                    const size_t row = drow0 + (size_t)min(chl, ch_valid - 1) * L;
                    const size_t start = ((row + l0) * ESZ_D) & ~(size_t)3;
                    const size_t off = start + (size_t)v * 4;
                    const size_t end = (row + L) * ESZ_D;
                    const int ok = (chl < ch_valid && off < end) ? (int)min((size_t)4, a.delta_bytes - off) : 0;
                    cp_async4(ddst + chl * DROW + v * 4, dbase + (ok ? off : start), ok);
                }
            }
        }
        if constexpr (CL) {
            // channels-last u: the run of this warp's channels at the pixel of step `lane`
            constexpr int PIECES = CW * ESZ_U / 16;
            const int l = l0 + lane;
            const int pix = pixr[st * TC + lane];
            const char *src = ubase + (((size_t)b * L + pix) * a.per_group + d0) * ESZ_U;
            unsigned char *udst = rs + lay.off_u + lane * UCP;
#pragma unroll
            for (int k = 0; k < PIECES; ++k) {
                const int bytes = l < L ? max(0, min(16, (a.per_group - d0 - k * (16 / ESZ_U)) * ESZ_U)) : 0;
                cp_async16(udst + 16 * k, bytes > 0 ? src + 16 * k : ubase, bytes);
            }
        } else if (umode == kURows) {
            constexpr int PER_ROW = TC * ESZ_U / 16;
            unsigned char *udst = rs + lay.off_u;
            for (int p = lane; p < CW * PER_ROW; p += 32) {
                const int chl = p / PER_ROW, v = p % PER_ROW;
                const int l = l0 + v * (16 / ESZ_U);
                const char *src = ubase + (urow0 + (size_t)min(chl, ch_valid - 1) * L) * ESZ_U;
                const int bytes = chl < ch_valid ? max(0, min(16, (L - l) * ESZ_U)) : 0;
                cp_async16(udst + chl * UROW + v * 16, bytes > 0 ? src + (size_t)l * ESZ_U : src, bytes);
            }
        } else if (umode == kURowsReversed) {
            // pixels [L - l0 - TC, L - l0) in storage order: step s sits at position TC - 1 - s.
            // Piece starts are multiples of 16 bytes, so a piece lies wholly below 0 or not at all.
            constexpr int PER_ROW = TC * ESZ_U / 16;
            unsigned char *udst = rs + lay.off_u;
            for (int p = lane; p < CW * PER_ROW; p += 32) {
                const int chl = p / PER_ROW, v = p % PER_ROW;
                const int px = L - l0 - TC + v * (16 / ESZ_U);
                const char *src = ubase + (urow0 + (size_t)min(chl, ch_valid - 1) * L) * ESZ_U;
                const int bytes = (chl < ch_valid && px >= 0) ? 16 : 0;
                cp_async16(udst + chl * UROW + v * 16, bytes > 0 ? src + (size_t)px * ESZ_U : src, bytes);
            }
        }
    };

    // Gathered u of one chunk (lane = step), raw storage values.
    UT ug[CW];
    auto gather_u = [&](int l0, int st) {
        const int l = l0 + lane;
        const bool ok = l < L;
        const size_t el = urow0 + (ok ? (MODE == kStandalone ? l : pixr[st * TC + lane]) : 0);
        const UT *p = reinterpret_cast<const UT *>(a.u) + el;
#pragma unroll
        for (int chl = 0; chl < CW; ++chl) {
            ug[chl] = (ok && chl < ch_valid) ? __ldg(p) : UT(0);
            p += L;
        }
    };
    auto put_u = [&](int st) {
        UT *ud = reinterpret_cast<UT *>(smem_raw + st * lay.stage_bytes + lay.off_u);
#pragma unroll
        for (int chl = 0; chl < CW; ++chl)
            ud[chl * (UROW / ESZ_U) + lane] = ug[chl];
    };

    const int nchunks = (lend - lbeg + TC - 1) / TC;
    stage_chunk(lbeg, 0);
    cp_async_commit();
    if (umode == kUGather) {
        __syncwarp();
        gather_u(lbeg, 0);
    }
    float2 sdl = make_float2(0.0f, 0.0f);  // first pass: sum of delta over the segment

    for (int j = 0; j < nchunks; ++j) {
        const int l0 = lbeg + j * TC;
        const int valid = min(TC, lend - l0);
        const int st = j & 1;
        const unsigned char *rs = smem_raw + st * lay.stage_bytes;

        if (umode == kUGather)
            put_u(st);
        cp_async_wait<0>();
        __syncwarp();
        if (j + 1 < nchunks) {
            stage_chunk(l0 + TC, st ^ 1);
            if (umode == kUGather) {
                __syncwarp();
                gather_u(l0 + TC, st ^ 1);
            }
        }
        cp_async_commit();

        // ---- scan: 4 steps per iteration -----------------------------------
        const float *bcs = reinterpret_cast<const float *>(rs + lay.off_bc);
        const unsigned char *drs = rs + lay.off_d + ch * DROW;
        const unsigned char *urs = rs + lay.off_u + ch * UROW;
        const float *trs = reinterpret_cast<const float *>(rs + lay.off_t);
        // byte offset of this chunk's first delta element within its word (misaligned rows)
        const int dsh = drows ? 0 : (int)(((drow0 + (size_t)min(ch, ch_valid - 1) * L + l0) * ESZ_D) & 3);
        float *ys_row = ysr + ch * YP;
        const int nsteps = (valid + 3) & ~3;
        for (int i = 0; i < nsteps; i += 4) {
            const int s0 = i + 2 * q;  // this lane's two steps: s0, s0 + 1
            if (CKPT && (i & 15) == 0 && l0 + i < L && ch < ch_valid) {
                // the 16 states of a checkpoint are stored lane-major: state q + 2n at q*8 + n
                float4 *o = reinterpret_cast<float4 *>(
                    a.ckpt + (((size_t)b * a.C + cch) * ((L + 15) / 16) + (l0 + i) / 16) * N + q * NS);
                o[0] = make_float4(h[0], h[1], h[2], h[3]);
                o[1] = make_float4(h[4], h[5], h[6], h[7]);
            }
            float z0, z1, u0, u1;
            if constexpr (MODE == kFusedProj) {
                z0 = 0.0f;
                z1 = 0.0f;
#pragma unroll
                for (int r = 0; r < kMaxR; ++r) {
                    if (r < R) {
                        const float2 t = *reinterpret_cast<const float2 *>(trs + r * BCP + s0);
                        z0 = fmaf(wdt[r], t.x, z0);
                        z1 = fmaf(wdt[r], t.y, z1);
                    }
                }
            } else if constexpr (D_BF16) {
                if (drows) {
                    const uint32_t w = *reinterpret_cast<const uint32_t *>(drs + 2 * s0);
                    z0 = bf16_lo(w);
                    z1 = bf16_hi(w);
                } else {
                    const unsigned char *p = drs + 2 * s0 + dsh;
                    z0 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p));
                    z1 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p + 2));
                }
            } else {
                const float2 t = *reinterpret_cast<const float2 *>(drs + 4 * s0);
                z0 = t.x;
                z1 = t.y;
            }
            if constexpr (CL) {
                const unsigned char *uc = rs + lay.off_u + s0 * UCP + ch * ESZ_U;
                if constexpr (U_BF16) {
                    u0 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(uc));
                    u1 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(uc + UCP));
                } else {
                    u0 = *reinterpret_cast<const float *>(uc);
                    u1 = *reinterpret_cast<const float *>(uc + UCP);
                }
            } else if constexpr (U_BF16) {
                if (umode == kURowsReversed) {
                    const uint32_t w = *reinterpret_cast<const uint32_t *>(urs + 2 * (TC - 2 - s0));
                    u0 = bf16_hi(w);
                    u1 = bf16_lo(w);
                } else {
                    const uint32_t w = *reinterpret_cast<const uint32_t *>(urs + 2 * s0);
                    u0 = bf16_lo(w);
                    u1 = bf16_hi(w);
                }
            } else {
                if (umode == kURowsReversed) {
                    const float2 t = *reinterpret_cast<const float2 *>(urs + 4 * (TC - 2 - s0));
                    u0 = t.y;
                    u1 = t.x;
                } else {
                    const float2 t = *reinterpret_cast<const float2 *>(urs + 4 * s0);
                    u0 = t.x;
                    u1 = t.y;
                }
            }
            z0 += bias_ch;
            z1 += bias_ch;
            if constexpr (S::SOFTPLUS) {
                z0 = softplus_f32(z0);
                z1 = softplus_f32(z1);
            }
            if (valid & 3) {
                // steps past the end of the sequence get delta = 0: decay 1 and no input, so the
                // state after the last step is what the loop leaves behind
                z0 = s0 < valid ? z0 : 0.0f;
                z1 = s0 + 1 < valid ? z1 : 0.0f;
            }
            const float w0 = z0 * u0, w1 = z1 * u1;
            const float pz0 = __shfl_xor_sync(0xffffffffu, z0, 1), pz1 = __shfl_xor_sync(0xffffffffu, z1, 1);
            const float pw0 = __shfl_xor_sync(0xffffffffu, w0, 1), pw1 = __shfl_xor_sync(0xffffffffu, w1, 1);
            // steps i, i+1 come from lane q = 0, steps i+2, i+3 from lane q = 1
            const float2 dl01 = q ? make_float2(pz0, pz1) : make_float2(z0, z1);
            const float2 dl23 = q ? make_float2(z0, z1) : make_float2(pz0, pz1);
            const float2 du01 = q ? make_float2(pw0, pw1) : make_float2(w0, w1);
            const float2 du23 = q ? make_float2(w0, w1) : make_float2(pw0, pw1);
            if (SEGP) {
                sdl = __fadd2_rn(sdl, dl01);
                sdl = __fadd2_rn(sdl, dl23);
            }
            float2 y01 = make_float2(0.0f, 0.0f), y23 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int n = 0; n < NS; ++n) {
                const int sr = q + 2 * n;
                const float4 bb = *reinterpret_cast<const float4 *>(bcs + sr * BCP + i);
                const float4 cv = NOOUT ? make_float4(0.f, 0.f, 0.f, 0.f)
                                        : *reinterpret_cast<const float4 *>(bcs + (N + sr) * BCP + i);
                const float2 an = make_float2(a2[n], a2[n]);
                const float2 x01 = __fmul2_rn(dl01, an);
                const float2 x23 = __fmul2_rn(dl23, an);
                const float2 bu01 = __fmul2_rn(du01, make_float2(bb.x, bb.y));
                const float2 bu23 = __fmul2_rn(du23, make_float2(bb.z, bb.w));
                float2 h01, h23;
                h01.x = fmaf(ex2_approx(x01.x), h[n], bu01.x);
                h01.y = fmaf(ex2_approx(x01.y), h01.x, bu01.y);
                h23.x = fmaf(ex2_approx(x23.x), h01.y, bu23.x);
                h23.y = fmaf(ex2_approx(x23.y), h23.x, bu23.y);
                h[n] = h23.y;
                if (!NOOUT) {
                    y01 = __ffma2_rn(make_float2(cv.x, cv.y), h01, y01);
                    y23 = __ffma2_rn(make_float2(cv.z, cv.w), h23, y23);
                }
            }
            if (NOOUT)
                continue;
            // reduce-scatter over the channel's two lanes: lane q keeps steps s0, s0 + 1
            const float k0 = q ? y23.x : y01.x, k1 = q ? y23.y : y01.y;
            const float t0 = q ? y01.x : y23.x, t1 = q ? y01.y : y23.y;
            const float r0 = fmaf(dsk_ch, u0, k0 + __shfl_xor_sync(0xffffffffu, t0, 1));
            const float r1 = fmaf(dsk_ch, u1, k1 + __shfl_xor_sync(0xffffffffu, t1, 1));
            *reinterpret_cast<float2 *>(ys_row + s0) = make_float2(r0, r1);
        }
        __syncwarp();

        // ---- write-out (lane = step, loop over channels) ---------------------
        // a merged output: atomic add, or (one direction per launch, or every direction into
        // its own buffer) plain store / add
        auto merge_add = [&](float *p, float v) {
            if (scan2_merge_mode<MODE>(a) == 0)
                red_add_hint(p, v, pol_keep);
            else
                *p = scan2_merge_mode<MODE>(a) == 1 ? v : *p + v;
        };
        auto merge_add4 = [&](float *p, float4 v) {
            if (scan2_merge_mode<MODE>(a) == 0) {
                red_add_v4_hint(p, v, pol_keep);
            } else {
                float4 *q4 = reinterpret_cast<float4 *>(p);
                if (scan2_merge_mode<MODE>(a) == 2) {
                    const float4 o = *q4;
                    v = make_float4(o.x + v.x, o.y + v.y, o.z + v.z, o.w + v.w);
                }
                *q4 = v;
            }
        };
        if constexpr (CL && !NOOUT) {
            // channels-last y: lane = (channel c, step parity r); each instruction adds the
            // channel runs of two steps
            const int c = lane & (CW - 1), r = lane / CW;
            if (c < ch_valid) {
                float *ybase = scan2_out<MODE>(a, g) + (size_t)b * L * a.per_group + d0 + c;
#pragma unroll
                for (int k = 0; k < TC / 2; ++k) {
                    const int s = 2 * k + r;
                    if (s < valid)
                        merge_add(ybase + (size_t)pixr[st * TC + s] * a.per_group, ysr[c * YP + s]);
                }
            }
        } else if (!NOOUT && vec_merge && !scan2_scan_order_out<MODE, CL>(a)) {
            // lane = (channel row (lane >> 3) + 4k, steps 4 (lane & 7) .. + 3): one 16-byte atomic
            // add per lane and row; direction 2 visits those steps' pixels in decreasing order
            const int sx = 4 * (lane & 7);
            if (sx < valid) {
#pragma unroll
                for (int k = 0; k < CW / 4; ++k) {
                    const int chl = (lane >> 3) + 4 * k;
                    if (full_warp || chl < ch_valid) {
                        const float4 yv = *reinterpret_cast<const float4 *>(ysr + chl * YP + sx);
                        float *yrow = a.y + ((size_t)b * a.per_group + d0 + chl) * L;
                        if (g == 0)
                            merge_add4(yrow + l0 + sx, yv);
                        else
                            merge_add4(yrow + (L - 4 - l0 - sx), make_float4(yv.w, yv.z, yv.y, yv.x));
                    }
                }
            }
        } else if (!NOOUT && lane < valid) {
            const float *yr = ysr + lane;
            if (MODE == kStandalone || scan2_scan_order_out<MODE, CL>(a)) {
                float *yp = (MODE == kStandalone ? a.y : a.ydir[0]) + ((size_t)b * a.C + c0) * L + l0 + lane;
#pragma unroll
                for (int chl = 0; chl < CW; ++chl) {
                    if (full_warp || chl < ch_valid)
                        *yp = yr[chl * YP];
                    yp += L;
                }
            } else {
                float *yp = a.y + ((size_t)b * a.per_group + d0) * L + pixr[st * TC + lane];
#pragma unroll
                for (int chl = 0; chl < CW; ++chl) {
                    if (full_warp || chl < ch_valid)
                        merge_add(yp, yr[chl * YP]);
                    yp += L;
                }
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    if (!NOOUT && a.hlast && ch < ch_valid) {
        // state after the last step of a whole-sequence scan
        const size_t o = ((size_t)b * a.C + cch) * N + q;
#pragma unroll
        for (int n = 0; n < NS; ++n)
            a.hlast[o + 2 * n] = h[n];
    }
    if (SEGP && ch < ch_valid) {
        // first pass: state at the end of the segment from a zero start, and the product of
        // its decays exp2(a2 * sum of delta)
        const float sd = sdl.x + sdl.y;
        const size_t o = (((size_t)b * a.C + cch) * a.nseg + seg) * N + q;
#pragma unroll
        for (int n = 0; n < NS; ++n) {
            a.hend[o + 2 * n] = h[n];
            a.pend[o + 2 * n] = ex2_approx(a2[n] * sd);
        }
    }
}

}  // namespace ss2d
