// lq_codec.cu -- stateless codec kernels: quantize an FP32 state (window-start
// quantizer of the LeapQuant project page, with the DAMP BF16 rows),
// dequantize it, copy a quantized state between the workspace record and plain
// arrays, and the DAMP channel-risk selection.  One CTA of 256 threads per head.
#include "lq_codec.cuh"
#include "lq_kernels.h"

namespace lq {

template <int DK, int DV>
struct QSmem {
    CodecSmem<DK, DV> cs;
    int map[DK];
    int wscr[kWarps];
};

__device__ __forceinline__ CodecOut codec_out_of(const QPtrs &q, int head) {
    CodecOut o{};
    o.codes = reinterpret_cast<int8_t *>(q.codes + (size_t)head * q.codes_hs);
    o.codes_t = q.codes_t;
    o.hp = reinterpret_cast<uint16_t *>(q.hp ? q.hp + (size_t)head * q.hp_hs : nullptr);
    o.m = reinterpret_cast<float *>(q.m + (size_t)head * q.m_hs);
    o.s = reinterpret_cast<float *>(q.s + (size_t)head * q.s_hs);
    o.ck = reinterpret_cast<float *>(q.ck ? q.ck + (size_t)head * q.ck_hs : nullptr);
    o.ck_stride = q.ck_js;
    o.cw = reinterpret_cast<float *>(q.cw ? q.cw + (size_t)head * q.cw_hs : nullptr);
    o.cw_stride = q.cw_js;
    return o;
}

template <int DK, int DV, int BITS>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const CodecArgs a) {
    __shared__ QSmem<DK, DV> sm;
    extern __shared__ __align__(16) unsigned char dyn[];
    ExactSmem<DK, DV> &X = *reinterpret_cast<ExactSmem<DK, DV> *>(dyn);
    using T = Tile<DK, DV>;
    const int head = blockIdx.x, h = head % a.H;
    if (a.P > 0) build_row_map<DK>(a.hp_rows + (size_t)h * a.P, a.P, sm.map, sm.wscr);
    float R[T::RPT][16];
    tile_load_global<DK, DV>(R, a.S_in + (size_t)head * DK * DV);
    const CodecOut out = codec_out_of(a.q, head);
    if (a.smoothing == 2) {   // the fixed scales, read back by the codec
        const float *ms = a.static_ms + (size_t)h * (DK + DV);
        for (int i = threadIdx.x; i < DK; i += kThreads) out.m[i] = ms[i];
        for (int c = threadIdx.x; c < DV; c += kThreads) out.s[c] = ms[DK + c];
        __syncthreads();
    }
    double eacc[T::RPT];
    codec_quantize_exact<DK, DV, false, BITS>(R, a.r, a.K, a.smoothing, a.P, a.P > 0 ? sm.map : nullptr, sm.cs, X,
                                              out, eacc);
    if (a.q.gam) {
        float *g = reinterpret_cast<float *>(a.q.gam + (size_t)head * a.q.gam_hs);
        for (int i = threadIdx.x; i < a.q.gam_n; i += kThreads) g[i] = 1.0f;
    }
}

// S = Deq(C, m, s) [BF16 rows widened] + sum_j c_j w_j^T.
template <int DK, int DV>
__global__ void __launch_bounds__(kThreads) dequantize_kernel(const CodecArgs a) {
    __shared__ QSmem<DK, DV> sm;
    using T = Tile<DK, DV>;
    const int head = blockIdx.x, h = head % a.H;
    const int t = threadIdx.x, cg = t % T::CG, row0 = (t / T::CG) * T::RPT;
    if (a.P > 0) build_row_map<DK>(a.hp_rows + (size_t)h * a.P, a.P, sm.map, sm.wscr);
    const QPtrs &q = a.q;
    const int8_t *codes = reinterpret_cast<const int8_t *>(q.codes + (size_t)head * q.codes_hs);
    const uint16_t *hp = q.hp ? reinterpret_cast<const uint16_t *>(q.hp + (size_t)head * q.hp_hs) : nullptr;
    const float *m = reinterpret_cast<const float *>(q.m + (size_t)head * q.m_hs);
    const float *s = reinterpret_cast<const float *>(q.s + (size_t)head * q.s_hs);
    float R[T::RPT][16];
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) {
        const int i = row0 + r;
        const int mp = a.P > 0 ? sm.map[i] : i;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int col = T::col(cg, qq) + u;
                R[r][4 * qq + u] = mp >= 0 ? ((float)codes[(size_t)mp * DV + col] * s[col]) * m[i]
                                           : bf16_to_f(hp[(size_t)(-1 - mp) * DV + col]);
            }
    }
    for (int j = 0; j < a.r; ++j) {
        const float *ck = reinterpret_cast<const float *>(q.ck + (size_t)head * q.ck_hs) + (size_t)j * q.ck_js;
        const float *cw = reinterpret_cast<const float *>(q.cw + (size_t)head * q.cw_hs) + (size_t)j * q.cw_js;
        float wv[16];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq)
#pragma unroll
            for (int u = 0; u < 4; ++u) wv[4 * qq + u] = cw[T::col(cg, qq) + u];
#pragma unroll
        for (int r = 0; r < T::RPT; ++r) {
            const float c = ck[row0 + r];
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) R[r][cc] = fmaf(c, wv[cc], R[r][cc]);
        }
    }
    tile_store_global<DK, DV>(R, a.S_out + (size_t)head * DK * DV);
}

// Copy a quantized state from q to q2 (same head numbering), setting q2's
// Gamma to 1 when it has one.  Row-major (view) codes are one per byte; a
// record's 4 / 6-bit codes are packed (an 8-row group per thread), and codes
// entering one are saturated to +-qmax.
template <int DK, int DV>
__global__ void __launch_bounds__(kThreads) qcopy_kernel(const CodecArgs a) {
    const int head = blockIdx.x, t = threadIdx.x;
    const QPtrs &x = a.q, &y = a.q2;
    const int P = a.P;
    if (a.bits < 8 && x.codes_t != y.codes_t) {
        const int qmax = (1 << (a.bits - 1)) - 1;
        const int8_t *src = reinterpret_cast<const int8_t *>(x.codes + (size_t)head * x.codes_hs);
        int8_t *dst = reinterpret_cast<int8_t *>(y.codes + (size_t)head * y.codes_hs);
        for (int e = t; e < (DK / 8) * DV; e += kThreads) {
            const int g = e / DV, c = e % DV;
            if (x.codes_t) {   // record -> view
                const unsigned char *pk = reinterpret_cast<const unsigned char *>(src);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    dst[(size_t)(8 * g + k) * DV + c] = (int8_t)packed_code(pk, c, 8 * g + k, DK, DV, a.bits);
            } else {           // view -> record
                uint32_t nw = 0u, pw = 0u;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int v = max(-qmax, min(qmax, (int)src[(size_t)(8 * g + k) * DV + c]));
                    nw |= ((uint32_t)v & 15u) << (4 * k);
                    pw |= (((uint32_t)v >> 4) & 3u) << (2 * k);
                }
                unsigned char *pk = reinterpret_cast<unsigned char *>(dst);
                *reinterpret_cast<uint32_t *>(pk + nib_off(c, g, DK)) = nw;
                if (a.bits == 6) *reinterpret_cast<uint16_t *>(pk + pair_off(c, g, DK, DV)) = (uint16_t)pw;
            }
        }
    } else if (x.codes_t == y.codes_t) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x.codes + (size_t)head * x.codes_hs);
        uint4 *dst = reinterpret_cast<uint4 *>(y.codes + (size_t)head * y.codes_hs);
        const int n16 = (DK - P) * DV / 16;
        for (int e = t; e < n16; e += kThreads) dst[e] = src[e];
    } else {   // row-major view <-> column-major swizzled record (P == 0)
        const int8_t *src = reinterpret_cast<const int8_t *>(x.codes + (size_t)head * x.codes_hs);
        int8_t *dst = reinterpret_cast<int8_t *>(y.codes + (size_t)head * y.codes_hs);
        for (int e = t; e < DK * DV; e += kThreads) {
            const int i = e / DV, c = e % DV;
            const int rm = i * DV + c, cm = code_off_t(c, i, DK);
            dst[y.codes_t ? cm : rm] = src[x.codes_t ? cm : rm];
        }
    }
    if (P > 0) {
        const uint16_t *src = reinterpret_cast<const uint16_t *>(x.hp + (size_t)head * x.hp_hs);
        uint16_t *dst = reinterpret_cast<uint16_t *>(y.hp + (size_t)head * y.hp_hs);
        for (int e = t; e < P * DV; e += kThreads) dst[e] = src[e];
    }
    {
        const float *src = reinterpret_cast<const float *>(x.m + (size_t)head * x.m_hs);
        float *dst = reinterpret_cast<float *>(y.m + (size_t)head * y.m_hs);
        for (int e = t; e < DK; e += kThreads) dst[e] = src[e];
        src = reinterpret_cast<const float *>(x.s + (size_t)head * x.s_hs);
        dst = reinterpret_cast<float *>(y.s + (size_t)head * y.s_hs);
        for (int e = t; e < DV; e += kThreads) dst[e] = src[e];
    }
    for (int j = 0; j < a.r; ++j) {
        const float *sk = reinterpret_cast<const float *>(x.ck + (size_t)head * x.ck_hs) + (size_t)j * x.ck_js;
        float *dk_ = reinterpret_cast<float *>(y.ck + (size_t)head * y.ck_hs) + (size_t)j * y.ck_js;
        for (int e = t; e < DK; e += kThreads) dk_[e] = sk[e];
        const float *sw = reinterpret_cast<const float *>(x.cw + (size_t)head * x.cw_hs) + (size_t)j * x.cw_js;
        float *dw = reinterpret_cast<float *>(y.cw + (size_t)head * y.cw_hs) + (size_t)j * y.cw_js;
        for (int e = t; e < DV; e += kThreads) dw[e] = sw[e];
    }
    if (y.gam) {
        float *g = reinterpret_cast<float *>(y.gam + (size_t)head * y.gam_hs);
        for (int i = t; i < y.gam_n; i += kThreads) g[i] = 1.0f;
    }
}

// DAMP channel risk: per head, sum over the calibration states of the per-row
// INT8 error energy, times the row's persistence 1 / (1 - mean decay); keep the
// top P rows (ties to the lower index), listed in increasing order.
template <int DK, int DV>
__global__ void __launch_bounds__(kThreads) damp_select_kernel(const CodecArgs a) {
    __shared__ CodecSmem<DK, DV> cs;
    extern __shared__ __align__(16) unsigned char dyn[];
    ExactSmem<DK, DV> &X = *reinterpret_cast<ExactSmem<DK, DV> *>(dyn);
    __shared__ double score[DK];
    __shared__ int sel[DK];
    using T = Tile<DK, DV>;
    const int h = blockIdx.x, t = threadIdx.x;
    const int cg = t % T::CG, row0 = (t / T::CG) * T::RPT;
    double eacc[T::RPT];
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) eacc[r] = 0.0;
    CodecOut none{};
    for (int n = 0; n < a.n_states; ++n) {
        float R[T::RPT][16];
        tile_load_global<DK, DV>(R, a.S_in + ((size_t)n * a.H + h) * DK * DV);
        codec_quantize_exact<DK, DV, true>(R, a.r, a.K, a.smoothing, 0, nullptr, cs, X, none, eacc);
    }
    if (cg == 0) {
#pragma unroll
        for (int r = 0; r < T::RPT; ++r) score[row0 + r] = eacc[r];
    }
    cbar();
    if (t < DK) {
        const double E = score[t];
        a.energy[(size_t)h * DK + t] = E;
        double mean = 0.0;
        const int ga = a.gate_per_channel ? DK : 1;
        const int col = a.gate_per_channel ? t : 0;
        for (int sidx = 0; sidx < a.n_gate_samples; ++sidx)
            mean += (double)a.gates[((size_t)sidx * a.H + h) * ga + col];
        mean /= (double)a.n_gate_samples;
        score[t] = E * (1.0 / (1.0 - mean));
    }
    __syncthreads();
    if (t < DK) {
        const double mine = score[t];
        int rank = 0;
        for (int j = 0; j < DK; ++j) {
            const double o = score[j];
            rank += (o > mine) || (o == mine && j < t);
        }
        sel[t] = rank < a.P;
    }
    __syncthreads();
    if (t < DK && sel[t]) {
        int pos = 0;
        for (int j = 0; j < t; ++j) pos += sel[j];
        a.rows_out[(size_t)h * a.P + pos] = t;
    }
}

// ---------------------------------------------------------------------------
// Static key-row / value-column scales fitted offline (STEPQuant article: the
// scales are fitted jointly from the state distribution and each key row's
// impact on the output error).  Reading: per head, on the residuals of n
// calibration states after the r compensators, minimise
//   sum_states sum_i sum_c w_i (R_ic - (clamp(rne((R_ic / m_i) / s_c)) s_c) m_i)^2
// by kFitRounds rounds of coordinate descent from m_i = RMS of row i over all
// states (1 if 0) and s_c = max |R_ic / m_i| / qmax: every column takes the
// best of s_c0 (1 - j/16), j < 12, then every row the best of m_i0 x
// kFitRowGrid (first best kept).  Errors in double, states outer, then rows
// (column step) or columns (row step); explicit roundings (no contraction).
// ---------------------------------------------------------------------------
constexpr int kFitRounds = 3;
constexpr int kFitNCol = 12;
constexpr int kFitNRow = 9;
__constant__ float kFitRowGrid[kFitNRow] = {0.5f, 0.625f, 0.75f, 0.875f, 1.0f, 1.25f, 1.5f, 1.75f, 2.0f};

// Residual of one calibration state after the compensators (FP64 extraction),
// float, to the scratch array [n][H][DK][DV].
template <int DK, int DV>
__global__ void __launch_bounds__(kThreads) fit_residual_kernel(const CodecArgs a) {
    extern __shared__ __align__(16) unsigned char dyn[];
    ExactSmem<DK, DV> &X = *reinterpret_cast<ExactSmem<DK, DV> *>(dyn);
    using T = Tile<DK, DV>;
    const size_t idx = blockIdx.x;   // state * H + head
    float R[T::RPT][16];
    tile_load_global<DK, DV>(R, a.S_in + idx * DK * DV);
    CodecOut none{};
    codec_compensators_fp64<DK, DV, false>(R, a.r, a.K, X, none);
    tile_store_global<DK, DV>(R, a.S_out + idx * DK * DV);
}

__device__ __forceinline__ double fit_err(float R, float m, float s, float qmax) {
    float dq = 0.0f;
    if (s != 0.0f) {
        const float x = __fdiv_rn(R, m);
        const float rq = fminf(fmaxf(rintf(__fdiv_rn(x, s)), -qmax), qmax);
        dq = __fmul_rn(__fmul_rn(rq, s), m);
    }
    const double d = __dsub_rn((double)R, (double)dq);
    return __dmul_rn(d, d);
}

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads) fit_static_kernel(const CodecArgs a, const float *res, int n,
                                                              float *m_out, float *s_out) {
    __shared__ float m0[DK], m[DK], s0[DV], s[DV];
    __shared__ double w[DK];
    __shared__ double err[kFitNRow > kFitNCol ? kFitNRow : kFitNCol][DK > DV ? DK : DV];
    const int h = blockIdx.x, t = threadIdx.x, H = a.H;
    const float qmax = (float)((1 << (a.bits - 1)) - 1);
    auto Rv = [&](int st, int i, int c) -> float { return res[(((size_t)st * H + h) * DK + i) * DV + c]; };
    if (t < DK) {
        // row weight: the decay persistence 1 / (1 - mean calibration decay)
        // of the row's channel (KDA) or of the head (GDN), as DAMP scores rows
        double wt = 1.0;
        if (a.gates) {
            const int ga = a.gate_per_channel ? DK : 1;
            const int col = a.gate_per_channel ? t : 0;
            double mean = 0.0;
            for (int sidx = 0; sidx < a.n_gate_samples; ++sidx)
                mean += (double)a.gates[((size_t)sidx * a.H + h) * ga + col];
            mean /= (double)a.n_gate_samples;
            wt = 1.0 / (1.0 - mean);
        }
        w[t] = wt;
        double ss = 0.0;
        for (int st = 0; st < n; ++st)
            for (int c = 0; c < DV; ++c) {
                const double r = (double)Rv(st, t, c);
                ss = __dadd_rn(ss, __dmul_rn(r, r));
            }
        float mi = (float)sqrt(__ddiv_rn(ss, (double)n * DV));
        if (mi == 0.0f) mi = 1.0f;
        m0[t] = m[t] = mi;
    }
    __syncthreads();
    if (t < DV) {
        float amax = 0.0f;
        for (int st = 0; st < n; ++st)
            for (int i = 0; i < DK; ++i) amax = fmaxf(amax, fabsf(__fdiv_rn(Rv(st, i, t), m[i])));
        s0[t] = s[t] = __fdiv_rn(amax, qmax);
    }
    __syncthreads();
    for (int round = 0; round < kFitRounds; ++round) {
        // columns: every (column, candidate) pair by one thread
        for (int p = t; p < DV * kFitNCol; p += kThreads) {
            const int c = p % DV, j = p / DV;
            const float sc = __fmul_rn(s0[c], 1.0f - (float)j / 16.0f);
            double e = 0.0;
            for (int st = 0; st < n; ++st)
                for (int i = 0; i < DK; ++i) e = __dadd_rn(e, __dmul_rn(w[i], fit_err(Rv(st, i, c), m[i], sc, qmax)));
            err[j][c] = e;
        }
        __syncthreads();
        if (t < DV) {
            double best = INFINITY;
            float sb = s[t];
            for (int j = 0; j < kFitNCol; ++j)
                if (err[j][t] < best) {
                    best = err[j][t];
                    sb = __fmul_rn(s0[t], 1.0f - (float)j / 16.0f);
                }
            s[t] = sb;
        }
        __syncthreads();
        // rows
        for (int p = t; p < DK * kFitNRow; p += kThreads) {
            const int i = p % DK, j = p / DK;
            const float mi = __fmul_rn(m0[i], kFitRowGrid[j]);
            double e = 0.0;
            for (int st = 0; st < n; ++st)
                for (int c = 0; c < DV; ++c) e = __dadd_rn(e, fit_err(Rv(st, i, c), mi, s[c], qmax));
            err[j][i] = e;
        }
        __syncthreads();
        if (t < DK) {
            double best = INFINITY;
            float mb = m[t];
            for (int j = 0; j < kFitNRow; ++j)
                if (err[j][t] < best) {
                    best = err[j][t];
                    mb = __fmul_rn(m0[t], kFitRowGrid[j]);
                }
            m[t] = mb;
        }
        __syncthreads();
    }
    if (t < DK) m_out[(size_t)h * DK + t] = m[t];
    if (t < DV) s_out[(size_t)h * DV + t] = s[t];
}

#define LQ_PICK(dk, dv, KERN)                          \
    (((dk) == 128 && (dv) == 128)  ? KERN<128, 128>    \
     : ((dk) == 64 && (dv) == 64)  ? KERN<64, 64>      \
     : ((dk) == 64 && (dv) == 128) ? KERN<64, 128>     \
                                   : KERN<128, 64>)

static size_t exact_bytes(int dk, int dv) {
    if (dk == 64 && dv == 64) return sizeof(ExactSmem<64, 64>);
    if (dk == 64 && dv == 128) return sizeof(ExactSmem<64, 128>);
    if (dk == 128 && dv == 64) return sizeof(ExactSmem<128, 64>);
    return sizeof(ExactSmem<128, 128>);
}

template <typename K>
static cudaError_t allow_smem(K kern, size_t bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

using CodecKernel = void (*)(const CodecArgs);

template <int BITS>
static CodecKernel pick_quantize(int dk, int dv) {
    if (dk == 128 && dv == 128) return quantize_kernel<128, 128, BITS>;
    if (dk == 64 && dv == 64) return quantize_kernel<64, 64, BITS>;
    if (dk == 64 && dv == 128) return quantize_kernel<64, 128, BITS>;
    return quantize_kernel<128, 64, BITS>;
}

cudaError_t launch_quantize(const CodecArgs &a, int dk, int dv, int heads, cudaStream_t s) {
    auto kern = a.bits == 4 ? pick_quantize<4>(dk, dv) : a.bits == 6 ? pick_quantize<6>(dk, dv) : pick_quantize<8>(dk, dv);
    const size_t sm = exact_bytes(dk, dv);
    cudaError_t e = allow_smem(kern, sm);
    if (e != cudaSuccess) return e;
    kern<<<heads, kThreads, sm, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_dequantize(const CodecArgs &a, int dk, int dv, int heads, cudaStream_t s) {
    LQ_PICK(dk, dv, dequantize_kernel)<<<heads, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_qcopy(const CodecArgs &a, int dk, int dv, int heads, cudaStream_t s) {
    LQ_PICK(dk, dv, qcopy_kernel)<<<heads, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_damp_select(const CodecArgs &a, int dk, int dv, cudaStream_t s) {
    auto kern = LQ_PICK(dk, dv, damp_select_kernel);
    const size_t sm = exact_bytes(dk, dv);
    cudaError_t e = allow_smem(kern, sm);
    if (e != cudaSuccess) return e;
    kern<<<a.H, kThreads, sm, s>>>(a);
    return cudaGetLastError();
}

template <int DK, int DV>
static cudaError_t fit_static_t(const CodecArgs &a, int n, float *m, float *sc, cudaStream_t s) {
    float *res = nullptr;
    const size_t nb = (size_t)n * a.H * DK * DV * sizeof(float);
    cudaError_t e = cudaMallocAsync(reinterpret_cast<void **>(&res), nb, s);
    if (e != cudaSuccess) return e;
    auto rk = fit_residual_kernel<DK, DV>;
    const size_t sm = sizeof(ExactSmem<DK, DV>);
    e = allow_smem(rk, sm);
    CodecArgs b = a;
    b.S_out = res;
    if (e == cudaSuccess) {
        rk<<<n * a.H, kThreads, sm, s>>>(b);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        fit_static_kernel<DK, DV><<<a.H, kThreads, 0, s>>>(a, res, n, m, sc);
        e = cudaGetLastError();
    }
    const cudaError_t f = cudaFreeAsync(res, s);
    return e != cudaSuccess ? e : f;
}

cudaError_t launch_fit_static(const CodecArgs &a, int dk, int dv, int n, float *m, float *sc, cudaStream_t s) {
    if (dk == 128 && dv == 128) return fit_static_t<128, 128>(a, n, m, sc, s);
    if (dk == 64 && dv == 64) return fit_static_t<64, 64>(a, n, m, sc, s);
    if (dk == 64 && dv == 128) return fit_static_t<64, 128>(a, n, m, sc, s);
    return fit_static_t<128, 64>(a, n, m, sc, s);
}

// The codec's division routine beside IEEE division (lq_selftest_division).
__global__ void div_selftest_kernel(const float *a, const float *b, float *fast, float *pair, float *ieee, int n) {
    const int j = blockIdx.x * blockDim.x + threadIdx.x;   // pair index
    if (2 * j >= n) return;
    const int i0 = 2 * j, i1 = 2 * j + 1;
    fast[i0] = div_rn(a[i0], b[i0], __frcp_rn(b[i0]));
    fast[i1] = div_rn(a[i1], b[i1], __frcp_rn(b[i1]));
    const float2 p = div2_rn(f2(a[i0], a[i1]), b[i0], __frcp_rn(b[i0]));
    pair[i0] = p.x;
    pair[i1] = p.y;
    ieee[i0] = __fdiv_rn(a[i0], b[i0]);
    ieee[i1] = __fdiv_rn(a[i1], b[i1]);
}

cudaError_t launch_div_selftest(const float *a, const float *b, float *fast, float *pair, float *ieee, int n,
                                cudaStream_t s) {
    const int pairs = n / 2;
    if (pairs == 0) return cudaSuccess;
    div_selftest_kernel<<<(pairs + 255) / 256, 256, 0, s>>>(a, b, fast, pair, ieee, n);
    return cudaGetLastError();
}

// The bounded wait of the staging copies, made to run out: the mbarrier is
// armed for 32 bytes and receives one 16-byte copy, so its phase never
// completes; mbar_wait_bounded gives up after limit_ns, raises the timeout
// status bit and returns (the copy itself has landed by then).
__global__ void __launch_bounds__(32) wait_selftest_kernel(const unsigned char *src, int *status,
                                                           unsigned long long limit_ns) {
    __shared__ __align__(16) unsigned char buf[16];
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&bar, 32u);
        bulk_g2s(buf, src, 16u, &bar);
        mbar_wait_bounded(&bar, 0, status, limit_ns);
    }
}

cudaError_t launch_wait_selftest(const unsigned char *src, int *status, unsigned long long limit_ns,
                                 cudaStream_t s) {
    wait_selftest_kernel<<<1, 32, 0, s>>>(src, status, limit_ns);
    return cudaGetLastError();
}

}  // namespace lq
