// scan.cuh -- the chunked selective-scan kernel of libss2d.
//
// One CTA owns CT consecutive channels of one (batch b, group g) and walks
// the whole sequence in chunks of TC steps.  Within a CTA each channel is
// served by TN = N / NS threads, each holding NS of the N fp32 states in
// registers, so the recurrence
//     h[n] <- exp(delta A[n]) h[n] + delta B_l[n] u_l,   y_l = sum_n C_l[n] h[n] + D u_l
// (the selective scan called in section 3.2 of the VMamba SS2D article) runs
// sequentially in l with no extra exponentials for splitting the sequence.
//
// Per chunk:
//   1. B and C rows of the chunk (shared by every channel of the group) are
//      copied into shared memory with cp.async, one chunk ahead.
//   2. delta and u of the chunk were loaded into registers one chunk ahead;
//      the prepass turns them into delta = softplus(dt + bias), delta*u and u
//      in shared memory (one exponential and one logarithm per element).
//   3. The scan: per 4 steps, each thread reads delta/delta*u for its channel
//      and B/C for its states as float4, updates its states, and stores its
//      partial y for the 4 steps.
//   4. Write-out: the TN partials of each (channel, step) are added in a fixed
//      order, D*u is added, and the value is stored (standalone) or added into
//      the merged output at the pixel this direction visited at that step
//      (fused CrossMerge, section 3.3 of the SS2D article).
#pragma once

#include "common.cuh"

namespace ss2d {

enum ScanMode { kStandalone = 0, kFused = 1 };

struct ScanArgs {
    const void *u;        // standalone: (B, C, L); fused: x (B, D, H, W)
    const void *delta;    // (B, C, L)   (fused: dts (B, 4, D, L) with C = 4D)
    const float *A_log;   // (C, N)
    const float *Bm;      // (B, G, N, L)
    const float *Cm;      // (B, G, N, L)
    const float *Dv;      // (C) or null
    const float *bias;    // (C) or null
    float *y;             // standalone: (B, C, L); fused: (B, D, H, W), accumulated
    int B, C, G, L;
    int per_group;        // C / G   (fused: D)
    int tiles;            // ceil(per_group / CT)
    int W;                // fused: image width
    SmallDiv divH;        // fused: division by the image height
    int u_bf16, delta_bf16;
    int softplus;
};

template <int N_, int NS_, int CT_, int TC_>
struct ScanShape {
    static constexpr int N = N_;
    static constexpr int NS = NS_;           // states per thread
    static constexpr int TN = N_ / NS_;      // threads per channel
    static constexpr int CT = CT_;           // channels per CTA
    static constexpr int TC = TC_;           // steps per chunk
    static constexpr int TCP = TC_ + 4;      // padded row pitch (floats)
    static constexpr int THREADS = CT_ * TN;
    static constexpr int EPT = (CT_ * TC_ + THREADS - 1) / THREADS;  // prepass elements per thread
    static constexpr int BC_STAGE = 2 * N_ * TCP;
    static constexpr int OFF_BC = 0;
    static constexpr int OFF_DLT = OFF_BC + 2 * BC_STAGE;
    static constexpr int OFF_DLU = OFF_DLT + CT_ * TCP;
    static constexpr int OFF_U = OFF_DLU + CT_ * TCP;
    static constexpr int OFF_YP = OFF_U + CT_ * TCP;
    static constexpr int OFF_PAR = OFF_YP + CT_ * TN * TCP;
    static constexpr int SMEM_FLOATS = OFF_PAR + 2 * CT_;
    static constexpr size_t SMEM_BYTES = sizeof(float) * SMEM_FLOATS;
    static_assert(N_ % NS_ == 0, "NS must divide N");
    static_assert(TC_ % 4 == 0 && (TC_ & (TC_ - 1)) == 0, "TC must be a power of two >= 4");
};

template <class S, int MODE>
__global__ void __launch_bounds__(S::THREADS) scan_kernel(const ScanArgs a)
{
    extern __shared__ __align__(16) float smem[];
    constexpr int N = S::N, NS = S::NS, TN = S::TN, CT = S::CT, TC = S::TC, TCP = S::TCP;
    constexpr int THREADS = S::THREADS, EPT = S::EPT;

    const int tid = threadIdx.x;
    int blk = blockIdx.x;
    const int tile = blk % a.tiles;
    blk /= a.tiles;
    const int g = blk % a.G;
    const int b = blk / a.G;
    const int d0 = tile * CT;
    const int ch_valid = min(CT, a.per_group - d0);
    const int c0 = g * a.per_group + d0;
    const int L = a.L;

    float *bc = smem + S::OFF_BC;
    float *dlt = smem + S::OFF_DLT;
    float *dlu = smem + S::OFF_DLU;
    float *us = smem + S::OFF_U;
    float *yp = smem + S::OFF_YP;
    float *Dpar = smem + S::OFF_PAR;
    float *Bpar = Dpar + CT;

    if (tid < CT) {
        const bool ok = tid < ch_valid;
        Dpar[tid] = (ok && a.Dv) ? a.Dv[c0 + tid] : 0.0f;
        Bpar[tid] = (ok && a.bias) ? a.bias[c0 + tid] : 0.0f;
    }

    // Scan role of this thread: channel ch, states q, q+TN, q+2TN, ...
    const int ch = tid / TN;
    const int q = tid % TN;
    float a2[NS], h[NS];
    {
        const int c = c0 + min(ch, ch_valid - 1);
#pragma unroll
        for (int j = 0; j < NS; ++j) {
            a2[j] = -expf(__ldg(a.A_log + (size_t)c * N + q + TN * j)) * kLog2e;
            h[j] = 0.0f;
        }
    }

    const size_t bg = ((size_t)b * a.G + g) * N;
    const float *Brows = a.Bm + bg * L;
    const float *Crows = a.Cm + bg * L;

    // ---- loaders -----------------------------------------------------------
    auto issue_bc = [&](int l0, int stage) {
        float *dst = bc + stage * S::BC_STAGE;
        if ((L & 3) == 0) {
            constexpr int PER_ROW = TC / 4;
            constexpr int PIECES = 2 * N * PER_ROW;
            for (int p = tid; p < PIECES; p += THREADS) {
                const int row = p / PER_ROW;  // 0..2N-1: B rows then C rows
                const int v = p % PER_ROW;
                const int l = l0 + 4 * v;
                const float *rowp = (row < N ? Brows + (size_t)row * L : Crows + (size_t)(row - N) * L);
                const int bytes = max(0, min(16, (L - l) * 4));
                cp_async16(dst + row * TCP + 4 * v, bytes > 0 ? rowp + l : rowp, bytes);
            }
        } else {
            constexpr int PIECES = 2 * N * TC;
            for (int p = tid; p < PIECES; p += THREADS) {
                const int row = p / TC;
                const int v = p % TC;
                const int l = l0 + v;
                const float *rowp = (row < N ? Brows + (size_t)row * L : Crows + (size_t)(row - N) * L);
                const int bytes = l < L ? 4 : 0;
                cp_async4(dst + row * TCP + v, bytes > 0 ? rowp + l : rowp, bytes);
            }
        }
    };

    float rd[EPT], ru[EPT];
    auto load_regs = [&](int l0) {
#pragma unroll
        for (int m = 0; m < EPT; ++m) {
            const int e = tid + m * THREADS;
            const int chl = e / TC;
            const int l = l0 + e % TC;
            float dv = 0.0f, uv = 0.0f;
            if (e < CT * TC && chl < ch_valid && l < L) {
                const size_t row = (size_t)b * a.C + c0 + chl;
                const size_t di = row * L + l;
                dv = a.delta_bf16 ? ldg_f32(reinterpret_cast<const __nv_bfloat16 *>(a.delta) + di)
                                  : ldg_f32(reinterpret_cast<const float *>(a.delta) + di);
                size_t ui;
                if (MODE == kStandalone) {
                    ui = di;
                } else {
                    ui = ((size_t)b * a.per_group + d0 + chl) * L + scan_pixel(g, l, L, a.W, a.divH);
                }
                uv = a.u_bf16 ? ldg_f32(reinterpret_cast<const __nv_bfloat16 *>(a.u) + ui)
                              : ldg_f32(reinterpret_cast<const float *>(a.u) + ui);
            }
            rd[m] = dv;
            ru[m] = uv;
        }
    };

    const int nchunks = (L + TC - 1) / TC;
    issue_bc(0, 0);
    cp_async_commit();
    load_regs(0);
    __syncthreads();  // Dpar / Bpar visible

    for (int j = 0; j < nchunks; ++j) {
        const int l0 = j * TC;
        const int valid = min(TC, L - l0);

        // ---- prepass: delta, delta*u, u into shared memory -----------------
#pragma unroll
        for (int m = 0; m < EPT; ++m) {
            const int e = tid + m * THREADS;
            if (e < CT * TC) {
                const int chl = e / TC;
                const int i = e % TC;
                float dv = rd[m] + Bpar[chl];
                if (a.softplus)
                    dv = softplus_f32(dv);
                float uv = ru[m];
                if (chl >= ch_valid || i >= valid) {
                    dv = 0.0f;
                    uv = 0.0f;
                }
                dlt[chl * TCP + i] = dv;
                dlu[chl * TCP + i] = dv * uv;
                us[chl * TCP + i] = uv;
            }
        }
        if (j + 1 < nchunks)
            issue_bc(l0 + TC, (j + 1) & 1);
        cp_async_commit();
        if (j + 1 < nchunks)
            load_regs(l0 + TC);
        cp_async_wait<1>();
        __syncthreads();

        // ---- scan ----------------------------------------------------------
        {
            const float *bcs = bc + (j & 1) * S::BC_STAGE;
            const float *dl_row = dlt + ch * TCP;
            const float *du_row = dlu + ch * TCP;
            float *yp_row = yp + (ch * TN + q) * TCP;
            const int nsteps = (valid + 3) & ~3;
            for (int i = 0; i < nsteps; i += 4) {
                const float4 dl = *reinterpret_cast<const float4 *>(dl_row + i);
                const float4 du = *reinterpret_cast<const float4 *>(du_row + i);
                float y0 = 0.0f, y1 = 0.0f, y2 = 0.0f, y3 = 0.0f;
#pragma unroll
                for (int jj = 0; jj < NS; ++jj) {
                    const int n = q + TN * jj;
                    const float4 bb = *reinterpret_cast<const float4 *>(bcs + n * TCP + i);
                    const float4 cc = *reinterpret_cast<const float4 *>(bcs + (N + n) * TCP + i);
                    float dA;
                    dA = ex2_approx(dl.x * a2[jj]);
                    h[jj] = fmaf(dA, h[jj], du.x * bb.x);
                    y0 = fmaf(cc.x, h[jj], y0);
                    dA = ex2_approx(dl.y * a2[jj]);
                    h[jj] = fmaf(dA, h[jj], du.y * bb.y);
                    y1 = fmaf(cc.y, h[jj], y1);
                    dA = ex2_approx(dl.z * a2[jj]);
                    h[jj] = fmaf(dA, h[jj], du.z * bb.z);
                    y2 = fmaf(cc.z, h[jj], y2);
                    dA = ex2_approx(dl.w * a2[jj]);
                    h[jj] = fmaf(dA, h[jj], du.w * bb.w);
                    y3 = fmaf(cc.w, h[jj], y3);
                }
                *reinterpret_cast<float4 *>(yp_row + i) = make_float4(y0, y1, y2, y3);
            }
        }
        __syncthreads();

        // ---- write-out -----------------------------------------------------
#pragma unroll
        for (int m = 0; m < EPT; ++m) {
            const int e = tid + m * THREADS;
            if (e < CT * TC) {
                const int chl = e / TC;
                const int i = e % TC;
                if (chl < ch_valid && i < valid) {
                    float v = yp[(chl * TN) * TCP + i];
#pragma unroll
                    for (int qq = 1; qq < TN; ++qq)
                        v += yp[(chl * TN + qq) * TCP + i];
                    v = fmaf(Dpar[chl], us[chl * TCP + i], v);
                    const int l = l0 + i;
                    if (MODE == kStandalone) {
                        a.y[((size_t)b * a.C + c0 + chl) * L + l] = v;
                    } else {
                        const int p = scan_pixel(g, l, L, a.W, a.divH);
                        atomicAdd(a.y + ((size_t)b * a.per_group + d0 + chl) * L + p, v);
                    }
                }
            }
        }
        __syncthreads();
    }
}

}  // namespace ss2d
