// lq_codec.cuh -- the window-boundary quantizer on one head's FP32 state held
// in registers across a 256-thread CTA.
//
// Steps (LeapQuant project page: Compensator Tokens paragraph, then the
// smoothing paragraph; STEPQuant article for key-row / value-column scales;
// DAMP abstract for the BF16 rows):
//   1. r compensators by deflated power iteration on the residual R:
//      w = 1/sqrt(dv); K times { z = R w / |R w| ; w = R^T z / |R^T z| };
//      c = R w;  R <- R - c w^T.   (norms accumulated in double)
//   2. BF16 rows: bf16_rne(R_i) for the head's listed key rows.
//   3. m_i = sqrt(mean_c R_ic^2) (double accumulation), 1 if zero or if
//      smoothing is off;  x = R / m.
//   4. s_c = max_i |x_ic| / 127 over INT8 rows;  C = clamp(rne(x / s), +-127).
//
// Tile layout: a thread owns RPT consecutive key rows x 16 consecutive value
// columns; CG = dv/16 column groups, RG = 256/CG row groups; thread t has
// column group t % CG and row group t / CG, so the CG threads sharing rows are
// adjacent lanes and the codes of one row segment leave as one 16-byte store.
#pragma once

#include "lq_common.cuh"

namespace lq {

template <int DK, int DV>
struct Tile {
    static constexpr int CG = DV / 16;
    static constexpr int RG = kThreads / CG;
    static constexpr int RPT = DK / RG;
    static_assert(RPT >= 1 && RG * RPT == DK, "tile shape");
    static_assert(CG <= 32 && (32 % CG) == 0, "column groups per warp");
};

template <int DK, int DV>
struct CodecSmem {
    float w[DV];
    float red[kWarps][DV];
    float sc[DV];
    double dred[kWarps];
};

// Where the codec writes one head's quantized state.
struct CodecOut {
    int8_t *codes;     // [(DK-P)][DV]
    uint16_t *hp;      // [P][DV]
    float *m;          // [DK]
    float *s;          // [DV]
    float *ck;         // c_j at ck + j*ck_stride, [DK] each
    int ck_stride;
    float *cw;         // w_j at cw + j*cw_stride, [DV] each
    int cw_stride;
};

// z[r] = sum_c R[r][c] w[c] for the thread's rows; all CG lanes of a row group
// end with the full sums.
template <int DK, int DV>
__device__ __forceinline__ void tile_rows_matvec(const float (&R)[Tile<DK, DV>::RPT][16], const float *w_s,
                                                 float (&z)[Tile<DK, DV>::RPT]) {
    using T = Tile<DK, DV>;
    const int cg = threadIdx.x % T::CG;
    float wv[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 f = reinterpret_cast<const float4 *>(w_s + cg * 16)[q];
        wv[4 * q] = f.x; wv[4 * q + 1] = f.y; wv[4 * q + 2] = f.z; wv[4 * q + 3] = f.w;
    }
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) {
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < 16; ++c) acc = fmaf(R[r][c], wv[c], acc);
        z[r] = shfl_xor_sum<T::CG>(acc);
    }
}

// out_s[c] = sum_i R[i][c] z[i] over the whole tile.  Barrier at the end.
template <int DK, int DV>
__device__ __forceinline__ void tile_cols_matvec(const float (&R)[Tile<DK, DV>::RPT][16],
                                                 const float (&z)[Tile<DK, DV>::RPT], float (*red)[DV],
                                                 float *out_s) {
    using T = Tile<DK, DV>;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5, cg = t % T::CG;
    float acc[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        float a = 0.f;
#pragma unroll
        for (int r = 0; r < T::RPT; ++r) a = fmaf(R[r][c], z[r], a);
#pragma unroll
        for (int m = T::CG; m < 32; m <<= 1) a += __shfl_xor_sync(0xffffffffu, a, m);
        acc[c] = a;
    }
    if (lane < T::CG) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
            reinterpret_cast<float4 *>(&red[warp][cg * 16])[q] =
                make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
    }
    __syncthreads();
    if (t < DV) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += red[w][t];
        out_s[t] = s;
    }
    __syncthreads();
}

// Full codec on the register tile R (destroyed).  `map` is the shared row map
// (slot >= 0 for INT8 rows, -1-p for BF16 row p); with P == 0 it may be null.
// ENERGY: instead of writing codes, add sum_c (R - Deq)^2 of the residual to
// eacc[r] (DAMP calibration); in that mode only m/s/compensators are computed.
template <int DK, int DV, bool ENERGY>
__device__ void codec_quantize(float (&R)[Tile<DK, DV>::RPT][16], int r_comp, int K, int smoothing, int P,
                               const int *map, CodecSmem<DK, DV> &cs, const CodecOut &out,
                               double (&eacc)[Tile<DK, DV>::RPT]) {
    using T = Tile<DK, DV>;
    constexpr int RPT = T::RPT, CG = T::CG;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int cg = t % CG, rg = t / CG;
    const int row0 = rg * RPT;

    // 1. Compensator tokens.
    for (int j = 0; j < r_comp; ++j) {
        if (t < DV) cs.w[t] = (float)(1.0 / sqrt((double)DV));
        __syncthreads();
        bool zero = false;
        for (int it = 0; it < K; ++it) {
            float z[RPT];
            tile_rows_matvec<DK, DV>(R, cs.w, z);
            double ss = 0.0;
            if (cg == 0) {
#pragma unroll
                for (int r = 0; r < RPT; ++r) ss += (double)z[r] * (double)z[r];
            }
            const double nz = sqrt(block_sum_d(ss, cs.dred));
            if (nz == 0.0) { zero = true; break; }
#pragma unroll
            for (int r = 0; r < RPT; ++r) z[r] = (float)((double)z[r] / nz);
            tile_cols_matvec<DK, DV>(R, z, cs.red, cs.w);
            const double sw = (t < DV) ? (double)cs.w[t] * (double)cs.w[t] : 0.0;
            const double nw = sqrt(block_sum_d(sw, cs.dred));
            if (nw == 0.0) { zero = true; break; }
            if (t < DV) cs.w[t] = (float)((double)cs.w[t] / nw);
            __syncthreads();
        }
        if (zero) {
            if (!ENERGY) {
                if (t < DV) out.cw[j * out.cw_stride + t] = 0.f;
                if (t < DK) out.ck[j * out.ck_stride + t] = 0.f;
            }
            __syncthreads();
            continue;
        }
        float c[RPT];
        tile_rows_matvec<DK, DV>(R, cs.w, c);
        if (!ENERGY) {
            if (t < DV) out.cw[j * out.cw_stride + t] = cs.w[t];
            if (cg == 0) {
#pragma unroll
                for (int r = 0; r < RPT; ++r) out.ck[j * out.ck_stride + row0 + r] = c[r];
            }
        }
        float wv[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) wv[q] = cs.w[cg * 16 + q];
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int q = 0; q < 16; ++q) R[r][q] = fmaf(-c[r], wv[q], R[r][q]);
        __syncthreads();
    }

    // 2. BF16 rows and 3. smoothing scales.
    float m[RPT];
    bool int8row[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = row0 + r;
        const int mp = (P > 0) ? map[i] : i;
        int8row[r] = mp >= 0;
        if (!ENERGY && mp < 0) {
            const int p = -1 - mp;
            uint32_t pk[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                pk[q] = (uint32_t)bf16_rne(R[r][2 * q]) | ((uint32_t)bf16_rne(R[r][2 * q + 1]) << 16);
            uint4 *dst = reinterpret_cast<uint4 *>(out.hp + (size_t)p * DV + cg * 16);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
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

    // 4. Column scales over INT8 rows.
    {
        float am[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) am[q] = 0.f;
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            if (!int8row[r]) continue;
#pragma unroll
            for (int q = 0; q < 16; ++q) am[q] = fmaxf(am[q], fabsf(R[r][q] / m[r]));
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
            for (int q = 0; q < 16; ++q) cs.red[warp][cg * 16 + q] = am[q];
        }
        __syncthreads();
        if (t < DV) {
            float a = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) a = fmaxf(a, cs.red[w][t]);
            const float sc = a / 127.0f;
            cs.sc[t] = sc;
            if (!ENERGY) out.s[t] = sc;
        }
        __syncthreads();
    }

    // Codes (or the error energy of the INT8 reconstruction).
    float sv[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) sv[q] = cs.sc[cg * 16 + q];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        if (!int8row[r]) continue;
        const int i = row0 + r;
        uint32_t pk[4] = {0u, 0u, 0u, 0u};
        double e = 0.0;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const float x = R[r][q] / m[r];
            float code = 0.f;
            if (sv[q] != 0.f) code = fminf(fmaxf(rintf(x / sv[q]), -127.f), 127.f);
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
        } else {
            const int slot = (P > 0) ? map[i] : i;
            *reinterpret_cast<uint4 *>(out.codes + (size_t)slot * DV + cg * 16) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
    }
    __syncthreads();
}

// Reconstruct a head's current state into the tile from a staged record:
// R = Gamma * ( Deq(C, m, s) [or BF16 rows] + sum_{e<E} ktil_e u_e^T ).
// stage points at the record prefix in shared memory; gam_s holds Gamma per
// key row (shared memory, DK floats).  Returns true if every value is finite.
template <int DK, int DV>
__device__ __forceinline__ bool tile_from_stage(float (&R)[Tile<DK, DV>::RPT][16], const unsigned char *stage,
                                                const Layout &L, int P, const int *map, int E,
                                                const float *gam_s) {
    using T = Tile<DK, DV>;
    constexpr int RPT = T::RPT;
    const int t = threadIdx.x, cg = t % T::CG, rg = t / T::CG, row0 = rg * RPT;
    const float *m_s = reinterpret_cast<const float *>(stage + L.off_m);
    const float *s_s = reinterpret_cast<const float *>(stage + L.off_s);
    const uint16_t *hp_s = reinterpret_cast<const uint16_t *>(stage + L.off_hp);
    const float *ent = reinterpret_cast<const float *>(stage + L.off_ent);
    float sv[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 f = reinterpret_cast<const float4 *>(s_s + cg * 16)[q];
        sv[4 * q] = f.x; sv[4 * q + 1] = f.y; sv[4 * q + 2] = f.z; sv[4 * q + 3] = f.w;
    }
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = row0 + r;
        const int mp = (P > 0) ? map[i] : i;
        if (mp >= 0) {
            const uint4 w = *reinterpret_cast<const uint4 *>(stage + (size_t)mp * DV + cg * 16);
            const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
            const float mi = m_s[i];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float f[4];
                s8x4_to_f(wd[q], f);
#pragma unroll
                for (int u = 0; u < 4; ++u) R[r][4 * q + u] = (f[u] * sv[4 * q + u]) * mi;
            }
        } else {
            const int p = -1 - mp;
#pragma unroll
            for (int q = 0; q < 16; ++q) R[r][q] = bf16_to_f(hp_s[(size_t)p * DV + cg * 16 + q]);
        }
    }
    for (int e = 0; e < E; ++e) {
        const float *kt = ent + (size_t)e * (DK + DV);
        const float *ut = kt + DK;
        float kv[RPT];
#pragma unroll
        for (int r = 0; r < RPT; ++r) kv[r] = kt[row0 + r];
        float uv[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 f = reinterpret_cast<const float4 *>(ut + cg * 16)[q];
            uv[4 * q] = f.x; uv[4 * q + 1] = f.y; uv[4 * q + 2] = f.z; uv[4 * q + 3] = f.w;
        }
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int q = 0; q < 16; ++q) R[r][q] = fmaf(kv[r], uv[q], R[r][q]);
    }
    bool finite = true;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const float g = gam_s[row0 + r];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            R[r][q] *= g;
            finite = finite && isfinite(R[r][q]);
        }
    }
    return finite;
}

}  // namespace lq
