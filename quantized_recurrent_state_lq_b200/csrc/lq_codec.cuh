// lq_codec.cuh -- the window-boundary quantizer on one head's FP32 state held
// in registers across the NT compute threads of a CTA (NT = 256 for the
// stand-alone codec kernels, 128 for the window flush).
//
// Steps (LeapQuant project page: Compensator Tokens paragraph, then the
// smoothing paragraph; STEPQuant article for key-row / value-column scales;
// DAMP abstract for the BF16 rows):
//   1. r compensators by deflated power iteration on the residual R:
//      w = 1/sqrt(dv); K times { w = R^T (R w), normalised };  c = R w;
//      R <- R - c w^T.  (R^T R w normalised is the oracle's z = Rw/|Rw|,
//      w = R^T z/|R^T z| without the intermediate scaling, which only changes
//      rounding.  The FP64 path accumulates norms in double; the FP32 path
//      takes them in FP32 when safely in range.)
//   2. BF16 rows: bf16_rne(R_i) for the head's listed key rows.
//   3. m_i = sqrt(mean_c R_ic^2) (double accumulation), 1 if zero or if
//      smoothing is off, the head's fixed scale with smoothing 2 (fitted
//      offline, STEPQuant article);  x = R / m.
//   4. s_c = max_i |x_ic| / qmax over INT8 rows (fixed with smoothing 2);
//      C = clamp(rne(x / s), +-qmax),
//      qmax = 2^(b-1) - 1 for b-bit codes (127, 31, 7: the LeapQuant page's
//      8-, 6- and 4-bit states).
//
// Tile layout: a thread owns RPT consecutive key rows and 16 value columns, in
// four groups of four adjacent columns spaced CG*4 apart:
//   cols(cg, q, u) = 4*cg + 4*CG*q + u,  q, u in [0, 4),
// with CG = dv/16 column groups and thread t in column group t % CG, row group
// t / CG.  The CG threads sharing rows are adjacent lanes, so every 16-byte
// shared-memory access of a column group touches consecutive words (no bank
// conflicts).
#pragma once

#include "lq_common.cuh"

namespace lq {

template <int DK, int DV, int NT = kThreads>
struct Tile {
    static constexpr int CG = DV / 16;
    static constexpr int RG = NT / CG;
    static constexpr int RPT = DK / RG;
    static constexpr int RGW = 32 / CG;  // row groups per warp
    static constexpr int NW = NT / 32;   // warps
    static_assert(RPT >= 1 && RG * RPT == DK, "tile shape");
    static_assert(CG <= 32 && (32 % CG) == 0, "column groups per warp");
    __device__ static int col(int cg, int q) { return 4 * cg + 4 * CG * q; }
};

template <int DK, int DV, int NT = kThreads>
struct CodecSmem {
    float red[2][NT / 32][DV];   // cross-warp partial column sums (double-buffered)
    float wv[NT / 32][DV];       // per-warp copy of the current power-iteration vector
    float sc[DV];
    float ysc[DV];               // RN(1 / sc)
    double dred[NT / 32];
};

// Where the codec writes one head's quantized state.
struct CodecOut {
    int8_t *codes;     // [(DK-P)][DV] by slot, or (codes_t) value-column-major, swizzled
    int codes_t;       // 1: code_off_t layout, or the packed planes of 4 / 6-bit codes (no
                       //    BF16 rows); 0: row-major by INT8 slot, one code per byte
    uint16_t *hp;      // [P][DV]
    float *m;          // [DK]
    float *s;          // [DV]
    float *ck;         // c_j at ck + j*ck_stride, [DK] each
    int ck_stride;
    float *cw;         // w_j at cw + j*cw_stride, [DV] each
    int cw_stride;
};
// With smoothing 2 the scales are fixed: the codec reads them from m and s
// (the record's, which hold them from lq_state_init on) and writes them back
// unchanged.

template <int DK, int DV>
__device__ __forceinline__ void load_cols16(const float *v, float (&o)[16]) {
    using T = Tile<DK, DV>;
    const int cg = threadIdx.x % T::CG;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 f = *reinterpret_cast<const float4 *>(v + T::col(cg, q));
        o[4 * q] = f.x; o[4 * q + 1] = f.y; o[4 * q + 2] = f.z; o[4 * q + 3] = f.w;
    }
}

// z[r] = sum_c R[r][c] w[c] for the thread's rows (w: the thread's 16 column
// values); all CG lanes of a row group end with the full sums.  Packed FP32
// FMAs over column pairs, then a transpose all-reduce over the row group.
template <int DK, int DV, int NT>
__device__ __forceinline__ void tile_rows_matvec(const float (&R)[Tile<DK, DV, NT>::RPT][16], const float (&w)[16],
                                                 float (&z)[Tile<DK, DV, NT>::RPT]) {
    using T = Tile<DK, DV, NT>;
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) {
        float2 acc = f2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc = ffma2(f2(R[r][2 * j], R[r][2 * j + 1]), f2(w[2 * j], w[2 * j + 1]), acc);
        z[r] = acc.x + acc.y;
    }
    xpose_allreduce<T::RPT, T::CG / 2, 1>(z);
}

// Sum of NW per-warp float4 partials in a fixed tree order (the same bits in
// every warp that computes it).
template <int NW>
__device__ __forceinline__ float4 sum_partials4(const float *base, int stride) {
    float4 p[NW];
#pragma unroll
    for (int w = 0; w < NW; ++w) p[w] = *reinterpret_cast<const float4 *>(base + w * stride);
#pragma unroll
    for (int h = NW / 2; h >= 1; h >>= 1)
#pragma unroll
        for (int w = 0; w < h; ++w) {
            p[w].x += p[w + h].x; p[w].y += p[w + h].y; p[w].z += p[w + h].z; p[w].w += p[w + h].w;
        }
    return p[0];
}

// Column sums of R weighted by z, reduced over the tile.  Every warp ends with
// the full vector y[DV] lane-distributed in `mine` (lane l holds y[4l .. 4l+3]
// for l < DV/4).  One barrier.
template <int DK, int DV, int NT>
__device__ __forceinline__ void tile_cols_matvec(const float (&R)[Tile<DK, DV, NT>::RPT][16],
                                                 const float (&z)[Tile<DK, DV, NT>::RPT], CodecSmem<DK, DV, NT> &cs,
                                                 int buf, float4 &mine) {
    using T = Tile<DK, DV, NT>;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5, cg = t % T::CG;
    float acc[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float2 a = f2(0.f, 0.f);
#pragma unroll
        for (int r = 0; r < T::RPT; ++r) a = ffma2(f2(R[r][2 * j], R[r][2 * j + 1]), f2(z[r], z[r]), a);
        acc[2 * j] = a.x;
        acc[2 * j + 1] = a.y;
    }
    // over the warp's row groups: lanes differing in bits 16 .. CG
    xpose_reduce<16, 16, T::CG>(acc);
    constexpr int NR = 16 >> xpose_bits<16, T::CG>();   // tile columns left per lane
    const int base = xpose_base<16, 16, T::CG>(lane);
    float *dst = &cs.red[buf][warp][T::col(cg, base / 4) + base % 4];
    if (NR == 4) *reinterpret_cast<float4 *>(dst) = make_float4(acc[0], acc[1], acc[2 % NR], acc[3 % NR]);
    else *reinterpret_cast<float2 *>(dst) = make_float2(acc[0], acc[1 % NR]);
    cbar<NT>();
    mine = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane < DV / 4) mine = sum_partials4<T::NW>(&cs.red[buf][0][4 * lane], DV);
}

// Step 1 in FP32 on the register tile: R becomes the residual.  (The window
// flush uses this path; its input is itself an FP32 result.)  With WRITE the
// compensators go to `out`.  Returns the barrier-buffer index to continue with.
//
// The power-iteration vector is normalised lazily: step k multiplies R by the
// previous, unnormalised y and scales z = R y by 1/|y| afterwards, so the norm
// (a double reduction, a square root and a reciprocal) runs alongside the next
// matrix-vector product instead of before it.  The final w_j is y_K / |y_K|.
template <int DK, int DV, bool WRITE, int NT = kThreads>
__device__ int codec_compensators_fp32(float (&R)[Tile<DK, DV, NT>::RPT][16], int r_comp, int K,
                                       CodecSmem<DK, DV, NT> &cs, const CodecOut &out) {
    using T = Tile<DK, DV, NT>;
    constexpr int RPT = T::RPT, CG = T::CG;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int cg = t % CG, rg = t / CG;
    const int row0 = rg * RPT;
    int buf = 0;
    for (int j = 0; j < r_comp; ++j) {
        float w[16];
        const float w0 = (float)(1.0 / sqrt((double)DV));
#pragma unroll
        for (int c = 0; c < 16; ++c) w[c] = w0;
        float inv = 1.0f;
        bool zero = false;   // identical in every thread: every warp reduces the same partials
        for (int it = 0; it < K; ++it) {
            float z[RPT];
            tile_rows_matvec<DK, DV, NT>(R, w, z);
#pragma unroll
            for (int r = 0; r < RPT; ++r) z[r] *= inv;
            float4 y;
            tile_cols_matvec<DK, DV, NT>(R, z, cs, buf, y);
            buf ^= 1;
            if (it + 1 < K) {
                // 1/|y| only sets the next step's length, not its direction:
                // FP32 sum and reciprocal square root while |y|^2 is
                // comfortably inside the FP32 range, else the sum again in
                // double.  A zero norm ends the extraction of this
                // compensator; the remaining steps then run on zeros / NaN and
                // are discarded.  (The sums are identical in every lane and
                // warp, so the branch is uniform.)
                if (lane < DV / 4) *reinterpret_cast<float4 *>(&cs.wv[warp][4 * lane]) = y;
                float ssf = fmaf(y.x, y.x, fmaf(y.y, y.y, fmaf(y.z, y.z, y.w * y.w)));
                ssf = warp_sum(ssf);
                if (ssf >= 0x1p-100f && ssf <= 0x1p100f) {
                    inv = rsqrtf(ssf);
                } else {
                    double ss = (double)y.x * y.x + (double)y.y * y.y + (double)y.z * y.z + (double)y.w * y.w;
                    ss = warp_sum_d(ss);
                    zero = zero || (ss == 0.0);
                    inv = (float)(1.0 / sqrt(ss));
                }
            } else {
                // The final w_j = y_K / |y_K| with the norm and the division in
                // double: unlike the per-step scales, |w_j| enters the removed
                // term c_j w_j^T = R w_j w_j^T squared, and that term can
                // exceed the residual by the ratio of the first to the
                // (r+1)-th singular value.
                double ss = (double)y.x * y.x + (double)y.y * y.y + (double)y.z * y.z + (double)y.w * y.w;
                ss = warp_sum_d(ss);
                zero = zero || (ss == 0.0);
                const double invd = 1.0 / sqrt(ss);
                if (lane < DV / 4)
                    *reinterpret_cast<float4 *>(&cs.wv[warp][4 * lane]) =
                        make_float4((float)(y.x * invd), (float)(y.y * invd), (float)(y.z * invd), (float)(y.w * invd));
            }
            __syncwarp();
            load_cols16<DK, DV>(cs.wv[warp], w);
            __syncwarp();
        }
        if (zero) {
            if (WRITE) {
                if (t < DV) out.cw[j * out.cw_stride + t] = 0.f;
                if (t < DK) out.ck[j * out.ck_stride + t] = 0.f;
            }
            continue;
        }
        float c[RPT];
        tile_rows_matvec<DK, DV, NT>(R, w, c);
        if (WRITE) {
            if (warp == 0 && lane < CG) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<float4 *>(out.cw + j * out.cw_stride + T::col(cg, q)) =
                        make_float4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
            }
            if (cg == 0) {
#pragma unroll
                for (int r = 0; r < RPT; ++r) out.ck[j * out.ck_stride + row0 + r] = c[r];
            }
        }
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float2 o = ffma2(f2(-c[r], -c[r]), f2(w[2 * q], w[2 * q + 1]), f2(R[r][2 * q], R[r][2 * q + 1]));
                R[r][2 * q] = o.x;
                R[r][2 * q + 1] = o.y;
            }
    }
    return buf;
}

// Double-precision scratch of the exact compensator extraction.
template <int DK, int DV>
struct ExactSmem {
    double R[DK][DV];
    double z[DK];
    double w[DV];
    double part[kThreads];
    double red[kWarps];
};

// Step 1 in double, as the oracle computes it: the residual lives in shared
// memory in double; z = R w / |R w|, w = R^T z / |R^T z| (K times), w and
// c = R w rounded to float when stored, R <- R - c w^T in double; the float
// residual comes back into the tile.  Used where the codec's input is an exact
// FP32 array (lq_quantize_state, lq_state_init, DAMP calibration), so that the
// compensators -- which decide every code -- agree with the oracle's to double
// rounding.
template <int DK, int DV, bool WRITE>
__device__ void codec_compensators_fp64(float (&R)[Tile<DK, DV>::RPT][16], int r_comp, int K,
                                        ExactSmem<DK, DV> &X, const CodecOut &out) {
    using T = Tile<DK, DV>;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int cg = t % T::CG, row0 = (t / T::CG) * T::RPT;
    constexpr int TPC = kThreads / DV;   // threads per column in R^T z
    constexpr int RPTC = DK / TPC;       // rows each of them sums
#pragma unroll
    for (int r = 0; r < T::RPT; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int u = 0; u < 4; ++u) X.R[row0 + r][T::col(cg, q) + u] = (double)R[r][4 * q + u];
    cbar();
    for (int j = 0; j < r_comp; ++j) {
        if (t < DV) X.w[t] = 1.0 / sqrt((double)DV);
        cbar();
        bool zero = false;
        for (int it = 0; it < K; ++it) {
            for (int i = warp; i < DK; i += kWarps) {
                double acc = 0.0;
#pragma unroll
                for (int k = 0; k < DV / 32; ++k) acc = fma(X.R[i][lane + 32 * k], X.w[lane + 32 * k], acc);
                acc = warp_sum_d(acc);
                if (lane == 0) X.z[i] = acc;
            }
            cbar();
            const double nz = sqrt(block_sum_d(t < DK ? X.z[t] * X.z[t] : 0.0, X.red));
            if (nz == 0.0) { zero = true; break; }
            if (t < DK) X.z[t] = X.z[t] / nz;
            cbar();
            {
                const int c = t % DV, h = t / DV;
                double acc = 0.0;
                for (int i = h * RPTC; i < (h + 1) * RPTC; ++i) acc = fma(X.R[i][c], X.z[i], acc);
                X.part[t] = acc;
            }
            cbar();
            if (t < DV) {
                double a = 0.0;
#pragma unroll
                for (int hh = 0; hh < TPC; ++hh) a += X.part[t + hh * DV];
                X.w[t] = a;
            }
            const double nw = sqrt(block_sum_d(t < DV ? X.w[t] * X.w[t] : 0.0, X.red));
            if (nw == 0.0) { zero = true; break; }
            if (t < DV) X.w[t] = X.w[t] / nw;
            cbar();
        }
        if (zero) {
            if (WRITE) {
                if (t < DV) out.cw[j * out.cw_stride + t] = 0.f;
                if (t < DK) out.ck[j * out.ck_stride + t] = 0.f;
            }
            cbar();
            continue;
        }
        if (t < DV) {
            const float wf = (float)X.w[t];
            X.w[t] = (double)wf;
            if (WRITE) out.cw[j * out.cw_stride + t] = wf;
        }
        cbar();
        for (int i = warp; i < DK; i += kWarps) {
            double acc = 0.0;
#pragma unroll
            for (int k = 0; k < DV / 32; ++k) acc = fma(X.R[i][lane + 32 * k], X.w[lane + 32 * k], acc);
            acc = warp_sum_d(acc);
            if (lane == 0) {
                const float cf = (float)acc;
                X.z[i] = (double)cf;
                if (WRITE) out.ck[j * out.ck_stride + i] = cf;
            }
        }
        cbar();
        for (int e = t; e < DK * DV; e += kThreads) {
            const int i = e / DV, c = e % DV;
            X.R[i][c] -= X.z[i] * X.w[c];
        }
        cbar();
    }
#pragma unroll
    for (int r = 0; r < T::RPT; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int u = 0; u < 4; ++u) R[r][4 * q + u] = (float)X.R[row0 + r][T::col(cg, q) + u];
    cbar();
}

// Steps 2-4 on the residual tile R (destroyed).  `map` is the shared row map
// (slot >= 0 for INT8 rows, -1-p for BF16 row p); with P == 0 it may be null.
// ENERGY: instead of writing codes, add sum_c (R - Deq)^2 of the residual to
// eacc[r] (DAMP calibration); in that mode nothing is written.
template <int DK, int DV, bool ENERGY, int NT = kThreads, int BITS = 8>
__device__ void codec_finish(float (&R)[Tile<DK, DV, NT>::RPT][16], int smoothing, int P, const int *map,
                             CodecSmem<DK, DV, NT> &cs, const CodecOut &out,
                             double (&eacc)[Tile<DK, DV, NT>::RPT], int buf) {
    using T = Tile<DK, DV, NT>;
    constexpr int RPT = T::RPT, CG = T::CG;
    constexpr float kQmax = (float)((1 << (BITS - 1)) - 1);   // 127, 31 or 7
    static_assert(BITS == 8 || BITS == 6 || BITS == 4, "code widths");
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int cg = t % CG, rg = t / CG;
    const int row0 = rg * RPT;

    // 2. BF16 rows and 3. smoothing scales; x = R / m in place (ENERGY keeps R).
    float m[RPT];
    uint32_t int8mask = 0;   // bit r: row row0 + r is an INT8 row
    float minabs = INFINITY;  // smallest |R| of the thread's elements
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = row0 + r;
        const int mp = (P > 0) ? map[i] : i;
        if (mp >= 0) int8mask |= 1u << r;
        if (!ENERGY && mp < 0) {
            const int p = -1 - mp;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t lo = (uint32_t)bf16_rne(R[r][4 * q]) | ((uint32_t)bf16_rne(R[r][4 * q + 1]) << 16);
                const uint32_t hi = (uint32_t)bf16_rne(R[r][4 * q + 2]) | ((uint32_t)bf16_rne(R[r][4 * q + 3]) << 16);
                *reinterpret_cast<uint2 *>(out.hp + (size_t)p * DV + T::col(cg, q)) = make_uint2(lo, hi);
            }
        }
#pragma unroll
        for (int q = 0; q < 16; ++q) minabs = fminf(minabs, fabsf(R[r][q]));
        float mi = 1.0f;
        if (smoothing == 2) {
            mi = out.m[i];   // fixed (fitted offline)
        } else {
            // row sum of squares in double over the row group's CG lanes (one
            // row at a time: few registers beside the tile)
            double ss = 0.0;
#pragma unroll
            for (int q = 0; q < 16; ++q) ss = fma((double)R[r][q], (double)R[r][q], ss);
#pragma unroll
            for (int mm = CG / 2; mm >= 1; mm >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, mm);
            if (smoothing && mp >= 0) {
                mi = (float)sqrt(ss / (double)DV);
                if (mi == 0.0f) mi = 1.0f;
            }
        }
        m[r] = mi;
    }
    if (!ENERGY && cg == 0) {
        if (RPT % 4 == 0) {
#pragma unroll
            for (int r = 0; r < RPT; r += 4)
                *reinterpret_cast<float4 *>(out.m + row0 + r) = make_float4(m[r], m[(r + 1) % RPT], m[(r + 2) % RPT], m[(r + 3) % RPT]);
        } else {
#pragma unroll
            for (int r = 0; r < RPT; ++r) out.m[row0 + r] = m[r];
        }
    }
    // x = R / m, correctly rounded (the oracle's IEEE division).  When every
    // element of the thread is at least 2^-79 in size and every row scale
    // lies in [2^-20, 2^20], the reciprocal-and-correction division (div_rn)
    // is exact for all of them -- m is 1 or the row RMS, so |x| <= sqrt(dv)
    // or the division is by 1 -- and one branch-free loop of packed
    // operations does it; otherwise the thread divides.  In place unless R
    // is still needed for the error energy.
    if (!ENERGY) {
        bool fast = minabs >= 0x1p-79f;
#pragma unroll
        for (int r = 0; r < RPT; ++r) fast = fast && m[r] >= 0x1p-20f && m[r] <= 0x1p20f;
        if (fast) {
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float ym = __frcp_rn(m[r]);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float2 x = div2_rn_unchecked(f2(R[r][2 * q], R[r][2 * q + 1]), m[r], ym);
                    R[r][2 * q] = x.x;
                    R[r][2 * q + 1] = x.y;
                }
            }
        } else {
#pragma unroll
            for (int r = 0; r < RPT; ++r)
#pragma unroll
                for (int q = 0; q < 16; ++q) R[r][q] = __fdiv_rn(R[r][q], m[r]);
        }
    }
    auto X = [&](int r, int q) -> float { return ENERGY ? __fdiv_rn(R[r][q], m[r]) : R[r][q]; };

    // 4. Column scales over INT8 rows (fixed ones with smoothing 2).
    if (smoothing == 2) {
        if (t < DV) {
            const float sc = out.s[t];
            cs.sc[t] = sc;
            cs.ysc[t] = __frcp_rn(sc);
            if (!ENERGY) out.s[t] = sc;
        }
        cbar<NT>();
    } else {
        float am[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) am[q] = 0.f;
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            if (!((int8mask >> r) & 1u)) continue;
#pragma unroll
            for (int q = 0; q < 16; ++q) am[q] = fmaxf(am[q], fabsf(X(r, q)));
        }
        xpose_reduce<16, 16, CG, true>(am);   // over the warp's row groups
        constexpr int NR = 16 >> xpose_bits<16, CG>();
        const int base = xpose_base<16, 16, CG>(lane);
        float *dst = &cs.red[buf][warp][T::col(cg, base / 4) + base % 4];
        if (NR == 4) *reinterpret_cast<float4 *>(dst) = make_float4(am[0], am[1], am[2 % NR], am[3 % NR]);
        else *reinterpret_cast<float2 *>(dst) = make_float2(am[0], am[1 % NR]);
        cbar<NT>();
        if (t < DV) {
            float a = 0.f;
#pragma unroll
            for (int w = 0; w < T::NW; ++w) a = fmaxf(a, cs.red[buf][w][t]);
            const float sc = a / kQmax;
            cs.sc[t] = sc;
            cs.ysc[t] = __frcp_rn(sc);
            if (!ENERGY) out.s[t] = sc;
        }
        cbar<NT>();
    }

    // Codes (or the error energy of the INT8 reconstruction).
    // C = clamp(rne(x / s)), the quotient correctly rounded as in the oracle.
    // For a column scale in [2^-20, 2^20] (col_fast) the reciprocal-and-
    // correction quotient is exact for |x| >= 2^-79 (|x / s| <= qmax for INT8
    // rows); below that, exact or not, it is under 2^-58 in size and rounds
    // to code 0 like the exact one: no branch per element.  Other scales (0
    // included) take IEEE division.  s and 1/s come from shared memory.
    auto col_fast = [](float sc) -> bool { return sc >= 0x1p-20f && sc <= 0x1p20f; };
    // clamp, then round half to even and convert with one FP32 add of
    // 1.5 * 2^23 (the sum's last bit is the integer, RN does the rounding) and
    // an integer subtract: no conversion-pipe instructions.  Clamping first is
    // equivalent to clamping the rounded value (qmax is an integer).
    auto clamp_code = [](float qt) -> uint32_t {
        const float cq = fminf(fmaxf(qt, -kQmax), kQmax) + 12582912.0f;
        return (uint32_t)(__float_as_int(cq) - 0x4B400000) & 0xffu;
    };
    auto code_fast = [&](float x, float sc, float ysc) -> uint32_t { return clamp_code(div_rn_unchecked(x, sc, ysc)); };
    auto code_ieee = [&](float x, float sc) -> uint32_t { return sc != 0.f ? clamp_code(__fdiv_rn(x, sc)) : 0u; };
    auto code_of = [&](float x, float sc, float ysc) -> uint32_t {
        return col_fast(sc) ? code_fast(x, sc, ysc) : code_ieee(x, sc);
    };
    if (ENERGY) {
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            if (!((int8mask >> r) & 1u)) continue;
            double e = 0.0;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const float4 s4 = *reinterpret_cast<const float4 *>(&cs.sc[T::col(cg, q4)]);
                const float4 y4 = *reinterpret_cast<const float4 *>(&cs.ysc[T::col(cg, q4)]);
                const float sa[4] = {s4.x, s4.y, s4.z, s4.w}, ya[4] = {y4.x, y4.y, y4.z, y4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int q = 4 * q4 + u;
                    const float dq = ((float)(int8_t)code_of(X(r, q), sa[u], ya[u]) * sa[u]) * m[r];
                    const double d = (double)R[r][q] - (double)dq;
                    e += d * d;
                }
            }
#pragma unroll
            for (int mm = CG / 2; mm >= 1; mm >>= 1) e += __shfl_xor_sync(0xffffffffu, e, mm);
            eacc[r] += e;
        }
    } else if (BITS < 8 && out.codes_t) {
        // packed 4 / 6-bit planes (no BF16 rows; the codes_t layout): the
        // RPT rows of one column go into the nibble / pair words of their
        // 8-row group, the 8 / RPT row groups of a code group (lanes CG
        // apart in one warp) OR their words together and the first stores.
        static_assert(RPT <= 8, "an 8-row code group spans whole row groups");
        constexpr int GT = 8 / RPT;
        unsigned char *base = reinterpret_cast<unsigned char *>(out.codes);
        const int g = row0 >> 3, k0 = row0 & 7;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const int col = T::col(cg, q / 4) + q % 4;
            const float sc = cs.sc[col], ysc = cs.ysc[col];
            uint32_t nw = 0u, pw = 0u;
            auto put = [&](int r, uint32_t b) {
                nw |= (b & 15u) << (4 * (k0 + r));
                pw |= ((b >> 4) & 3u) << (2 * (k0 + r));
            };
            if (col_fast(sc)) {   // one decision per column, as for INT8
#pragma unroll
                for (int r = 0; r < RPT; ++r) put(r, code_fast(R[r][q], sc, ysc));
            } else {
#pragma unroll
                for (int r = 0; r < RPT; ++r) put(r, code_ieee(R[r][q], sc));
            }
#pragma unroll
            for (int o = CG; o < CG * GT; o <<= 1) {
                nw |= __shfl_xor_sync(0xffffffffu, nw, o);
                if (BITS == 6) pw |= __shfl_xor_sync(0xffffffffu, pw, o);
            }
            if (k0 == 0) {
                *reinterpret_cast<uint32_t *>(base + nib_off(col, g, DK)) = nw;
                if (BITS == 6) *reinterpret_cast<uint16_t *>(base + pair_off(col, g, DK, DV)) = (uint16_t)pw;
            }
        }
    } else if (out.codes_t) {
        // value-column-major (no BF16 rows): the thread's RPT rows of one
        // column are RPT consecutive bytes; one store per column
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const int col = T::col(cg, q / 4) + q % 4;
            const float sc = cs.sc[col], ysc = cs.ysc[col];
            uint32_t lo = 0u, hi = 0u;
            if (col_fast(sc)) {
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const uint32_t b = code_fast(R[r][q], sc, ysc);
                    if (r < 4) lo |= b << (8 * r);
                    else hi |= b << (8 * (r - 4));
                }
            } else {
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const uint32_t b = code_ieee(R[r][q], sc);
                    if (r < 4) lo |= b << (8 * r);
                    else hi |= b << (8 * (r - 4));
                }
            }
            int8_t *dst = out.codes + code_off_t(col, row0, DK);
            if (RPT == 8) *reinterpret_cast<uint2 *>(dst) = make_uint2(lo, hi);
            else if (RPT == 4) *reinterpret_cast<uint32_t *>(dst) = lo;
            else if (RPT == 2) *reinterpret_cast<uint16_t *>(dst) = (uint16_t)lo;
            else *dst = (int8_t)lo;
        }
    } else {
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            if (!((int8mask >> r) & 1u)) continue;
            const int i = row0 + r;
            const int slot = (P > 0) ? map[i] : i;
            uint32_t *dst = reinterpret_cast<uint32_t *>(out.codes + (size_t)slot * DV);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const float4 s4 = *reinterpret_cast<const float4 *>(&cs.sc[T::col(cg, q4)]);
                const float4 y4 = *reinterpret_cast<const float4 *>(&cs.ysc[T::col(cg, q4)]);
                const uint32_t pk = code_of(R[r][4 * q4], s4.x, y4.x) | (code_of(R[r][4 * q4 + 1], s4.y, y4.y) << 8) |
                                    (code_of(R[r][4 * q4 + 2], s4.z, y4.z) << 16) |
                                    (code_of(R[r][4 * q4 + 3], s4.w, y4.w) << 24);
                dst[T::col(cg, q4) / 4] = pk;
            }
        }
    }
    cbar<NT>();
}

// The whole quantizer with the FP32 compensator step (window flush).
template <int DK, int DV, bool ENERGY, int NT = kThreads, int BITS = 8>
__device__ void codec_quantize(float (&R)[Tile<DK, DV, NT>::RPT][16], int r_comp, int K, int smoothing, int P,
                               const int *map, CodecSmem<DK, DV, NT> &cs, const CodecOut &out,
                               double (&eacc)[Tile<DK, DV, NT>::RPT]) {
    const int buf = codec_compensators_fp32<DK, DV, !ENERGY, NT>(R, r_comp, K, cs, out);
    codec_finish<DK, DV, ENERGY, NT, BITS>(R, smoothing, P, map, cs, out, eacc, buf);
}

// The whole quantizer with the double-precision compensator step.
template <int DK, int DV, bool ENERGY, int BITS = 8>
__device__ void codec_quantize_exact(float (&R)[Tile<DK, DV>::RPT][16], int r_comp, int K, int smoothing, int P,
                                     const int *map, CodecSmem<DK, DV> &cs, ExactSmem<DK, DV> &X,
                                     const CodecOut &out, double (&eacc)[Tile<DK, DV>::RPT]) {
    codec_compensators_fp64<DK, DV, !ENERGY>(R, r_comp, K, X, out);
    codec_finish<DK, DV, ENERGY, kThreads, BITS>(R, smoothing, P, map, cs, out, eacc, 0);
}

// Reconstruction of a head's current state into the tile, in three parts:
//   tile_dequant:      R = Deq(C, m, s) [BF16 rows widened]  (ADD: R += ...)
//   tile_add_entries:  R += sum_e ktil_e u_e^T over n entries [n][DK+DV]
//   tile_gamma:        R *= Gamma (by key row); true if every value is finite
// The arrays may live in shared or global memory: m_s [DK], s_s [DV],
// hp_s [P][DV], codes_s (layout per codes_t; BITS < 8: the packed planes),
// gam_s [DK]; sig_s [DK] (nullable) scales every key row, quantized or BF16
// (the decode kernels' decay guard).
template <int DK, int DV, int NT, bool ADD = false, int BITS = 8>
__device__ __forceinline__ void tile_dequant(float (&R)[Tile<DK, DV, NT>::RPT][16], const float *m_s,
                                             const float *s_s, const uint16_t *hp_s, const int8_t *codes_s, int P,
                                             const int *map, bool codes_t, const float *sig_s = nullptr) {
    using T = Tile<DK, DV, NT>;
    constexpr int RPT = T::RPT;
    const int t = threadIdx.x, cg = t % T::CG, rg = t / T::CG, row0 = rg * RPT;
    auto put = [&](int r, int q, float v) { R[r][q] = ADD ? R[r][q] + v : v; };
    if (BITS < 8) {
        // packed 4 / 6-bit codes: the thread's rows lie in one 8-row group,
        // unpacked to signed bytes c * 2^(8-BITS), scaled back exactly
        static_assert(RPT <= 8, "rows of a thread within one code group");
        constexpr float kInv = BITS == 4 ? 0.0625f : 0.25f;
        const unsigned char *cb = reinterpret_cast<const unsigned char *>(codes_s);
        const int g = row0 >> 3, k0 = row0 & 7;
        float sv[16];
        load_cols16<DK, DV>(s_s, sv);
        float mi[RPT];
#pragma unroll
        for (int r = 0; r < RPT; ++r) mi[r] = sig_s ? m_s[row0 + r] * sig_s[row0 + r] : m_s[row0 + r];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int col = T::col(cg, q) + u;
                const uint32_t nib = *reinterpret_cast<const uint32_t *>(cb + nib_off(col, g, DK));
                const uint32_t pr =
                    BITS == 6 ? spread_pairs(*reinterpret_cast<const uint16_t *>(cb + pair_off(col, g, DK, DV)), false)
                              : 0u;
                uint32_t lo, hi;
                unpack_group<(BITS < 8 ? BITS : 4)>(nib, pr, lo, hi);
                if (RPT == 8) {
                    float fl[4], fh[4];
                    s8x4_to_f(lo, fl);
                    s8x4_to_f(hi, fh);
#pragma unroll
                    for (int r = 0; r < RPT; ++r) {
                        const float cf = ((r & 1) ? fh[r >> 1] : fl[r >> 1]) * kInv;
                        put(r, 4 * q + u, (cf * sv[4 * q + u]) * mi[r]);
                    }
                } else {
#pragma unroll
                    for (int r = 0; r < RPT; ++r) {
                        const int k = k0 + r;
                        const uint32_t w = (k & 1) ? hi : lo;
                        const float cf = (float)(int8_t)((w >> (8 * (k >> 1))) & 0xffu) * kInv;
                        put(r, 4 * q + u, (cf * sv[4 * q + u]) * mi[r]);
                    }
                }
            }
        return;
    }
    if (codes_t && (RPT == 4 || RPT == 8)) {
        float sv[16];
        load_cols16<DK, DV>(s_s, sv);
        // value-column-major codes (no BF16 rows): the thread's RPT rows of
        // one column are RPT consecutive bytes
        float mi[RPT];
#pragma unroll
        for (int r = 0; r < RPT; ++r) mi[r] = sig_s ? m_s[row0 + r] * sig_s[row0 + r] : m_s[row0 + r];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int8_t *src = codes_s + code_off_t(T::col(cg, q) + u, row0, DK);
                uint32_t wd[2];
                if (RPT == 8) {
                    const uint2 v2 = *reinterpret_cast<const uint2 *>(src);
                    wd[0] = v2.x;
                    wd[1] = v2.y;
                } else {
                    wd[0] = *reinterpret_cast<const uint32_t *>(src);
                    wd[1] = 0u;
                }
#pragma unroll
                for (int h = 0; h < RPT / 4; ++h) {
                    float f[4];
                    s8x4_to_f(wd[h], f);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int r = 4 * h + k;
                        put(r % RPT, 4 * q + u, (f[k] * sv[4 * q + u]) * mi[r % RPT]);
                    }
                }
            }
        return;
    }
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = row0 + r;
        const int mp = (P > 0) ? map[i] : i;
        if (mp >= 0 && codes_t) {
            const float mi = sig_s ? m_s[i] * sig_s[i] : m_s[i];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 s4 = *reinterpret_cast<const float4 *>(s_s + T::col(cg, q));
                const float sq[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float cf = (float)codes_s[code_off_t(T::col(cg, q) + u, i, DK)];
                    put(r, 4 * q + u, (cf * sq[u]) * mi);
                }
            }
        } else if (mp >= 0) {
            const float mi = sig_s ? m_s[i] * sig_s[i] : m_s[i];
            const uint32_t *row = reinterpret_cast<const uint32_t *>(codes_s + (size_t)mp * DV);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 s4 = *reinterpret_cast<const float4 *>(s_s + T::col(cg, q));
                const float sq[4] = {s4.x, s4.y, s4.z, s4.w};
                float f[4];
                s8x4_to_f(row[T::col(cg, q) / 4], f);
#pragma unroll
                for (int u = 0; u < 4; ++u) put(r, 4 * q + u, (f[u] * sq[u]) * mi);
            }
        } else {
            const int p = -1 - mp;
            const float sg = sig_s ? sig_s[i] : 1.0f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint2 h = *reinterpret_cast<const uint2 *>(hp_s + (size_t)p * DV + T::col(cg, q));
                put(r, 4 * q, bf16_to_f((uint16_t)(h.x & 0xffff)) * sg);
                put(r, 4 * q + 1, bf16_to_f((uint16_t)(h.x >> 16)) * sg);
                put(r, 4 * q + 2, bf16_to_f((uint16_t)(h.y & 0xffff)) * sg);
                put(r, 4 * q + 3, bf16_to_f((uint16_t)(h.y >> 16)) * sg);
            }
        }
    }
}

template <int DK, int DV, int NT>
__device__ __forceinline__ void tile_add_entries(float (&R)[Tile<DK, DV, NT>::RPT][16], const float *ent, int n) {
    using T = Tile<DK, DV, NT>;
    constexpr int RPT = T::RPT;
    const int row0 = (threadIdx.x / T::CG) * RPT;
    for (int e = 0; e < n; ++e) {
        const float *kt = ent + (size_t)e * (DK + DV);
        float kv[RPT];
        if (RPT % 4 == 0) {
#pragma unroll
            for (int r = 0; r < RPT; r += 4) {
                const float4 k4 = *reinterpret_cast<const float4 *>(kt + row0 + r);
                kv[r] = k4.x; kv[(r + 1) % RPT] = k4.y; kv[(r + 2) % RPT] = k4.z; kv[(r + 3) % RPT] = k4.w;
            }
        } else {
#pragma unroll
            for (int r = 0; r < RPT; ++r) kv[r] = kt[row0 + r];
        }
        float uv[16];
        load_cols16<DK, DV>(kt + DK, uv);
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float2 o = ffma2(f2(kv[r], kv[r]), f2(uv[2 * q], uv[2 * q + 1]), f2(R[r][2 * q], R[r][2 * q + 1]));
                R[r][2 * q] = o.x;
                R[r][2 * q + 1] = o.y;
            }
    }
}

// Gamma, and a finiteness check that costs one packed FMA per pair: x * 0 is
// NaN exactly when x is not finite, and NaN propagates.
template <int DK, int DV, int NT>
__device__ __forceinline__ bool tile_gamma(float (&R)[Tile<DK, DV, NT>::RPT][16], const float *gam_s) {
    using T = Tile<DK, DV, NT>;
    const int row0 = (threadIdx.x / T::CG) * T::RPT;
    float2 chk = f2(0.f, 0.f);
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) {
        const float g = gam_s[row0 + r];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float2 o = __fmul2_rn(f2(g, g), f2(R[r][2 * q], R[r][2 * q + 1]));
            R[r][2 * q] = o.x;
            R[r][2 * q + 1] = o.y;
            chk = ffma2(o, f2(0.f, 0.f), chk);
        }
    }
    return chk.x == 0.f && chk.y == 0.f;
}

// Tile <-> row-major [DK][DV] global arrays.
template <int DK, int DV, int NT = kThreads>
__device__ __forceinline__ void tile_load_global(float (&R)[Tile<DK, DV, NT>::RPT][16], const float *src) {
    using T = Tile<DK, DV, NT>;
    const int t = threadIdx.x, cg = t % T::CG, row0 = (t / T::CG) * T::RPT;
#pragma unroll
    for (int r = 0; r < T::RPT; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 f = __ldg(reinterpret_cast<const float4 *>(src + (size_t)(row0 + r) * DV + T::col(cg, q)));
            R[r][4 * q] = f.x; R[r][4 * q + 1] = f.y; R[r][4 * q + 2] = f.z; R[r][4 * q + 3] = f.w;
        }
}

template <int DK, int DV, int NT = kThreads>
__device__ __forceinline__ void tile_store_global(const float (&R)[Tile<DK, DV, NT>::RPT][16], float *dst) {
    using T = Tile<DK, DV, NT>;
    const int t = threadIdx.x, cg = t % T::CG, row0 = (t / T::CG) * T::RPT;
#pragma unroll
    for (int r = 0; r < T::RPT; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q)
            *reinterpret_cast<float4 *>(dst + (size_t)(row0 + r) * DV + T::col(cg, q)) =
                make_float4(R[r][4 * q], R[r][4 * q + 1], R[r][4 * q + 2], R[r][4 * q + 3]);
}

}  // namespace lq
