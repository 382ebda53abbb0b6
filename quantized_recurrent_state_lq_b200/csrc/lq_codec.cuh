// lq_codec.cuh -- the window-boundary quantizer on one head's FP32 state held
// in registers across the 256 compute threads of a CTA.
//
// Steps (LeapQuant project page: Compensator Tokens paragraph, then the
// smoothing paragraph; STEPQuant article for key-row / value-column scales;
// DAMP abstract for the BF16 rows):
//   1. r compensators by deflated power iteration on the residual R:
//      w = 1/sqrt(dv); K times { w = R^T (R w), normalised };  c = R w;
//      R <- R - c w^T.  (R^T R w normalised is the oracle's z = Rw/|Rw|,
//      w = R^T z/|R^T z| without the intermediate scaling, which only changes
//      rounding; norms are accumulated in double.)
//   2. BF16 rows: bf16_rne(R_i) for the head's listed key rows.
//   3. m_i = sqrt(mean_c R_ic^2) (double accumulation), 1 if zero or if
//      smoothing is off;  x = R / m.
//   4. s_c = max_i |x_ic| / 127 over INT8 rows;  C = clamp(rne(x / s), +-127).
//
// Tile layout: a thread owns RPT consecutive key rows and 16 value columns, in
// four groups of four adjacent columns spaced CG*4 apart:
//   cols(cg, q, u) = 4*cg + 4*CG*q + u,  q, u in [0, 4),
// with CG = dv/16 column groups and thread t in column group t % CG, row group
// t / CG.  The CG threads sharing rows are adjacent lanes, so every 16-byte
// shared-memory access of a column group touches consecutive words (no bank
// conflicts) and code rows leave as 32-byte contiguous segments.
#pragma once

#include "lq_common.cuh"

namespace lq {

template <int DK, int DV>
struct Tile {
    static constexpr int CG = DV / 16;
    static constexpr int RG = kThreads / CG;
    static constexpr int RPT = DK / RG;
    static constexpr int RGW = 32 / CG;  // row groups per warp
    static_assert(RPT >= 1 && RG * RPT == DK, "tile shape");
    static_assert(CG <= 32 && (32 % CG) == 0, "column groups per warp");
    __device__ static int col(int cg, int q) { return 4 * cg + 4 * CG * q; }
};

template <int DK, int DV>
struct CodecSmem {
    float red[2][kWarps][DV];   // cross-warp partial column sums (double-buffered)
    float wv[kWarps][DV];       // per-warp copy of the current power-iteration vector
    float sc[DV];
    double dred[kWarps];
};

// Where the codec writes one head's quantized state.
struct CodecOut {
    int8_t *codes;     // [(DK-P)][DV] by slot, or (codes_t) value-column-major, swizzled
    int codes_t;       // 1: code_off_t layout (no BF16 rows); 0: row-major by INT8 slot
    uint16_t *hp;      // [P][DV]
    float *m;          // [DK]
    float *s;          // [DV]
    float *ck;         // c_j at ck + j*ck_stride, [DK] each
    int ck_stride;
    float *cw;         // w_j at cw + j*cw_stride, [DV] each
    int cw_stride;
};

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
template <int DK, int DV>
__device__ __forceinline__ void tile_rows_matvec(const float (&R)[Tile<DK, DV>::RPT][16], const float (&w)[16],
                                                 float (&z)[Tile<DK, DV>::RPT]) {
    using T = Tile<DK, DV>;
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) {
        float2 acc = f2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc = ffma2(f2(R[r][2 * j], R[r][2 * j + 1]), f2(w[2 * j], w[2 * j + 1]), acc);
        z[r] = acc.x + acc.y;
    }
    xpose_allreduce<T::RPT, T::CG / 2, 1>(z);
}

// Column sums of R weighted by z, reduced over the tile.  Each warp ends with
// the full vector y[DV] in its own wv[warp] (and lane-distributed in `mine`:
// lane l holds y[4l .. 4l+3] for l < DV/4).  One barrier.
template <int DK, int DV>
__device__ __forceinline__ void tile_cols_matvec(const float (&R)[Tile<DK, DV>::RPT][16],
                                                 const float (&z)[Tile<DK, DV>::RPT], CodecSmem<DK, DV> &cs,
                                                 int buf, float4 &mine) {
    using T = Tile<DK, DV>;
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
    cbar();
    mine = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane < DV / 4) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float4 p = *reinterpret_cast<const float4 *>(&cs.red[buf][w][4 * lane]);
            mine.x += p.x; mine.y += p.y; mine.z += p.z; mine.w += p.w;
        }
    }
}

// Step 1 in FP32 on the register tile: R becomes the residual.  (The window
// flush uses this path; its input is itself an FP32 result.)  With WRITE the
// compensators go to `out`.  Returns the barrier-buffer index to continue with.
template <int DK, int DV, bool WRITE>
__device__ int codec_compensators_fp32(float (&R)[Tile<DK, DV>::RPT][16], int r_comp, int K,
                                       CodecSmem<DK, DV> &cs, const CodecOut &out) {
    using T = Tile<DK, DV>;
    constexpr int RPT = T::RPT, CG = T::CG;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int cg = t % CG, rg = t / CG;
    const int row0 = rg * RPT;
    constexpr bool ENERGY = !WRITE;
    int buf = 0;
    for (int j = 0; j < r_comp; ++j) {
        float w[16];
        const float w0 = (float)(1.0 / sqrt((double)DV));
#pragma unroll
        for (int c = 0; c < 16; ++c) w[c] = w0;
        bool zero = false;
        for (int it = 0; it < K; ++it) {
            float z[RPT];
            tile_rows_matvec<DK, DV>(R, w, z);
            float4 y;
            tile_cols_matvec<DK, DV>(R, z, cs, buf, y);
            buf ^= 1;
            // |y|^2 accumulated in double (no overflow for any finite y); only
            // the reciprocal of the norm is taken in FP32: it sets w's length,
            // not its direction, and the next step normalises again.
            double ss = (double)y.x * y.x + (double)y.y * y.y + (double)y.z * y.z + (double)y.w * y.w;
            ss = warp_sum_d(ss);   // identical in every warp
            if (ss == 0.0) { zero = true; break; }
            const float inv = 1.0f / (float)sqrt(ss);
            if (lane < DV / 4)
                *reinterpret_cast<float4 *>(&cs.wv[warp][4 * lane]) =
                    make_float4(y.x * inv, y.y * inv, y.z * inv, y.w * inv);
            __syncwarp();
            load_cols16<DK, DV>(cs.wv[warp], w);
            __syncwarp();
        }
        if (zero) {
            if (!ENERGY) {
                if (t < DV) out.cw[j * out.cw_stride + t] = 0.f;
                if (t < DK) out.ck[j * out.ck_stride + t] = 0.f;
            }
            continue;
        }
        float c[RPT];
        tile_rows_matvec<DK, DV>(R, w, c);
        if (!ENERGY) {
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
template <int DK, int DV, bool ENERGY>
__device__ void codec_finish(float (&R)[Tile<DK, DV>::RPT][16], int smoothing, int P, const int *map,
                             CodecSmem<DK, DV> &cs, const CodecOut &out, double (&eacc)[Tile<DK, DV>::RPT],
                             int buf) {
    using T = Tile<DK, DV>;
    constexpr int RPT = T::RPT, CG = T::CG;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int cg = t % CG, rg = t / CG;
    const int row0 = rg * RPT;

    // 2. BF16 rows and 3. smoothing scales; x = R / m in place (ENERGY keeps R).
    float m[RPT];
    bool int8row[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = row0 + r;
        const int mp = (P > 0) ? map[i] : i;
        int8row[r] = mp >= 0;
        if (!ENERGY && mp < 0) {
            const int p = -1 - mp;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t lo = (uint32_t)bf16_rne(R[r][4 * q]) | ((uint32_t)bf16_rne(R[r][4 * q + 1]) << 16);
                const uint32_t hi = (uint32_t)bf16_rne(R[r][4 * q + 2]) | ((uint32_t)bf16_rne(R[r][4 * q + 3]) << 16);
                *reinterpret_cast<uint2 *>(out.hp + (size_t)p * DV + T::col(cg, q)) = make_uint2(lo, hi);
            }
        }
        double ss = 0.0;
#pragma unroll
        for (int q = 0; q < 16; ++q) ss += (double)R[r][q] * (double)R[r][q];
#pragma unroll
        for (int mm = CG / 2; mm >= 1; mm >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, mm);
        float mi = 1.0f;
        if (smoothing && int8row[r]) {
            mi = (float)sqrt(ss / (double)DV);
            if (mi == 0.0f) mi = 1.0f;
        }
        m[r] = mi;
        if (!ENERGY && cg == 0) out.m[i] = mi;
    }
    // x = R / m (IEEE division, as the oracle); in place unless R is still
    // needed for the error energy.
    if (!ENERGY) {
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int q = 0; q < 16; ++q) R[r][q] = R[r][q] / m[r];
    }
    auto X = [&](int r, int q) -> float { return ENERGY ? R[r][q] / m[r] : R[r][q]; };

    // 4. Column scales over INT8 rows.
    {
        float am[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) am[q] = 0.f;
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            if (!int8row[r]) continue;
#pragma unroll
            for (int q = 0; q < 16; ++q) am[q] = fmaxf(am[q], fabsf(X(r, q)));
        }
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            float a = am[q];
#pragma unroll
            for (int mm = CG; mm < 32; mm <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, mm));
            am[q] = a;
        }
        if (lane < CG) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<float4 *>(&cs.red[buf][warp][T::col(cg, q)]) =
                    make_float4(am[4 * q], am[4 * q + 1], am[4 * q + 2], am[4 * q + 3]);
        }
        cbar();
        if (t < DV) {
            float a = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) a = fmaxf(a, cs.red[buf][w][t]);
            const float sc = a / 127.0f;
            cs.sc[t] = sc;
            if (!ENERGY) out.s[t] = sc;
        }
        cbar();
    }

    // Codes (or the error energy of the INT8 reconstruction).
    float sv[16];
    load_cols16<DK, DV>(cs.sc, sv);
    uint32_t tpk[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) tpk[c] = 0u;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        if (!int8row[r]) continue;
        const int i = row0 + r;
        uint32_t pk[4] = {0u, 0u, 0u, 0u};
        double e = 0.0;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            float code = 0.f;
            if (sv[q] != 0.f) code = fminf(fmaxf(rintf(X(r, q) / sv[q]), -127.f), 127.f);
            if (ENERGY) {
                const float dq = (code * sv[q]) * m[r];
                const double d = (double)R[r][q] - (double)dq;
                e += d * d;
            } else {
                pk[q >> 2] |= ((uint32_t)((int)code & 0xff)) << (8 * (q & 3));
            }
        }
        if (ENERGY) {
#pragma unroll
            for (int mm = CG / 2; mm >= 1; mm >>= 1) e += __shfl_xor_sync(0xffffffffu, e, mm);
            eacc[r] += e;
        } else if (out.codes_t) {
            // value-column-major: gather this thread's RPT consecutive rows of each column
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int u = 0; u < 4; ++u) tpk[4 * q + u] |= ((pk[q] >> (8 * u)) & 0xffu) << (8 * r);
        } else {
            const int slot = (P > 0) ? map[i] : i;
            uint32_t *dst = reinterpret_cast<uint32_t *>(out.codes + (size_t)slot * DV);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[T::col(cg, q) / 4] = pk[q];
        }
    }
    if (!ENERGY && out.codes_t) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                int8_t *dst = out.codes + code_off_t(T::col(cg, q) + u, row0, DK);
                if (RPT == 4) {
                    *reinterpret_cast<uint32_t *>(dst) = tpk[4 * q + u];
                } else {
#pragma unroll
                    for (int r = 0; r < RPT; ++r) dst[r] = (int8_t)((tpk[4 * q + u] >> (8 * r)) & 0xffu);
                }
            }
    }
    cbar();
}

// The whole quantizer with the FP32 compensator step (window flush).
template <int DK, int DV, bool ENERGY>
__device__ void codec_quantize(float (&R)[Tile<DK, DV>::RPT][16], int r_comp, int K, int smoothing, int P,
                               const int *map, CodecSmem<DK, DV> &cs, const CodecOut &out,
                               double (&eacc)[Tile<DK, DV>::RPT]) {
    const int buf = codec_compensators_fp32<DK, DV, !ENERGY>(R, r_comp, K, cs, out);
    codec_finish<DK, DV, ENERGY>(R, smoothing, P, map, cs, out, eacc, buf);
}

// The whole quantizer with the double-precision compensator step.
template <int DK, int DV, bool ENERGY>
__device__ void codec_quantize_exact(float (&R)[Tile<DK, DV>::RPT][16], int r_comp, int K, int smoothing, int P,
                                     const int *map, CodecSmem<DK, DV> &cs, ExactSmem<DK, DV> &X,
                                     const CodecOut &out, double (&eacc)[Tile<DK, DV>::RPT]) {
    codec_compensators_fp64<DK, DV, !ENERGY>(R, r_comp, K, X, out);
    codec_finish<DK, DV, ENERGY>(R, smoothing, P, map, cs, out, eacc, 0);
}

// Reconstruct a head's current state into the tile:
// R = Gamma * ( Deq(C, m, s) [or BF16 rows] + sum_{e<E} ktil_e u_e^T ).
// The arrays may live in shared or global memory: m_s [DK], s_s [DV],
// hp_s [P][DV], codes_s [DK-P][DV], ent [E][DK+DV], gam_s [DK].
// Returns true if every value is finite.
template <int DK, int DV>
__device__ __forceinline__ bool tile_reconstruct(float (&R)[Tile<DK, DV>::RPT][16], const float *m_s,
                                                 const float *s_s, const uint16_t *hp_s, const int8_t *codes_s,
                                                 const float *ent, int P, const int *map, int E,
                                                 const float *gam_s, bool codes_t) {
    using T = Tile<DK, DV>;
    constexpr int RPT = T::RPT;
    const int t = threadIdx.x, cg = t % T::CG, rg = t / T::CG, row0 = rg * RPT;
    float sv[16];
    load_cols16<DK, DV>(s_s, sv);
    if (codes_t && RPT == 4) {
        // value-column-major codes (no BF16 rows): the thread's 4 rows of one
        // column are 4 consecutive bytes
        float mi[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) mi[r] = m_s[row0 + r];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t w4 = *reinterpret_cast<const uint32_t *>(codes_s + code_off_t(T::col(cg, q) + u, row0, DK));
                float f[4];
                s8x4_to_f(w4, f);
#pragma unroll
                for (int r = 0; r < 4; ++r) R[r % RPT][4 * q + u] = (f[r] * sv[4 * q + u]) * mi[r];
            }
    } else {
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int i = row0 + r;
            const int mp = (P > 0) ? map[i] : i;
            if (mp >= 0 && codes_t) {
                const float mi = m_s[i];
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float cf = (float)codes_s[code_off_t(T::col(cg, q) + u, i, DK)];
                        R[r][4 * q + u] = (cf * sv[4 * q + u]) * mi;
                    }
            } else if (mp >= 0) {
                const float mi = m_s[i];
                const uint32_t *row = reinterpret_cast<const uint32_t *>(codes_s + (size_t)mp * DV);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float f[4];
                    s8x4_to_f(row[T::col(cg, q) / 4], f);
#pragma unroll
                    for (int u = 0; u < 4; ++u) R[r][4 * q + u] = (f[u] * sv[4 * q + u]) * mi;
                }
            } else {
                const int p = -1 - mp;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint2 h = *reinterpret_cast<const uint2 *>(hp_s + (size_t)p * DV + T::col(cg, q));
                    R[r][4 * q] = bf16_to_f((uint16_t)(h.x & 0xffff));
                    R[r][4 * q + 1] = bf16_to_f((uint16_t)(h.x >> 16));
                    R[r][4 * q + 2] = bf16_to_f((uint16_t)(h.y & 0xffff));
                    R[r][4 * q + 3] = bf16_to_f((uint16_t)(h.y >> 16));
                }
            }
        }
    }
    // buffered entries: R += ktil_e u_e^T, two columns per packed FMA
    for (int e = 0; e < E; ++e) {
        const float *kt = ent + (size_t)e * (DK + DV);
        float kv[RPT];
        if (RPT == 4) {
            const float4 k4 = *reinterpret_cast<const float4 *>(kt + row0);
            kv[0] = k4.x; kv[1 % RPT] = k4.y; kv[2 % RPT] = k4.z; kv[3 % RPT] = k4.w;
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
    // Gamma, and a finiteness check that costs one packed FMA per pair:
    // x * 0 is NaN exactly when x is not finite, and NaN propagates.
    float2 chk = f2(0.f, 0.f);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
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
template <int DK, int DV>
__device__ __forceinline__ void tile_load_global(float (&R)[Tile<DK, DV>::RPT][16], const float *src) {
    using T = Tile<DK, DV>;
    const int t = threadIdx.x, cg = t % T::CG, row0 = (t / T::CG) * T::RPT;
#pragma unroll
    for (int r = 0; r < T::RPT; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 f = __ldg(reinterpret_cast<const float4 *>(src + (size_t)(row0 + r) * DV + T::col(cg, q)));
            R[r][4 * q] = f.x; R[r][4 * q + 1] = f.y; R[r][4 * q + 2] = f.z; R[r][4 * q + 3] = f.w;
        }
}

template <int DK, int DV>
__device__ __forceinline__ void tile_store_global(const float (&R)[Tile<DK, DV>::RPT][16], float *dst) {
    using T = Tile<DK, DV>;
    const int t = threadIdx.x, cg = t % T::CG, row0 = (t / T::CG) * T::RPT;
#pragma unroll
    for (int r = 0; r < T::RPT; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q)
            *reinterpret_cast<float4 *>(dst + (size_t)(row0 + r) * DV + T::col(cg, q)) =
                make_float4(R[r][4 * q], R[r][4 * q + 1], R[r][4 * q + 2], R[r][4 * q + 3]);
}

}  // namespace lq
