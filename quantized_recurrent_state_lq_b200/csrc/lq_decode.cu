// lq_decode.cu -- decode-step kernels.
//
// Windowed INT8 decode (LeapQuant project page, window paragraph): within a
// window the INT8 state is read, never written.  With Gamma_t the product of
// the decays since the window start, ktil_tau = k_tau / Gamma_tau and the
// compensators (c_j, w_j) treated as buffer entries with ktil = c_j, u = w_j
// (Compensator Tokens paragraph), the recurrence of the LinQuant appendix
// Table 3 unrolls to
//   S_t = Gamma_t [ Deq + sum_j c_j w_j^T + sum_{tau<=t} ktil_tau u_tau^T ],
// so with x = Gamma_t * k_t (and Gamma_t * q_t):
//   y_x = diag(s) C^T (m * x)  +  sum_e u_e (ktil_e . x)
//   u_t = beta_t (v_t - y_k),   o_t = y_q + u_t (k_t . q_t),
// and (k_t / Gamma_t, u_t) is appended to the buffer.
//
// One CTA per (batch, head).  Thread 0 stages the head's record prefix (codes,
// BF16 rows, m, s and the r + n buffered entries -- one contiguous range) into
// shared memory with a single cp.async.bulk; meanwhile the other threads load
// q, k, v, beta, alpha and form Gamma_t.  The codes are consumed as one 32-bit
// word (4 columns) per lane and row, a warp covering whole 128-byte rows.
#include "lq_codec.cuh"
#include "lq_kernels.h"

namespace lq {

template <int DK, int DV>
struct DecSmem {
    float2 x2[DK];     // (Gamma*k, Gamma*q)
    float2 a2[DK];     // (m*Gamma*k, m*Gamma*q) by INT8 slot
    float k[DK];
    float gam[DK];
    float v[DV];
    float2 red[kWarps * (128 / DV)][DV];
    int map[DK];
    int wscr[kWarps];
    float kqw[kWarps];
    CodecSmem<DK, DV> cs;
    uint64_t mbar;
};

template <int DK, int DV>
__host__ __device__ constexpr size_t dec_fixed_bytes() {
    return (sizeof(DecSmem<DK, DV>) + 15) / 16 * 16;
}

size_t decode_smem_bytes(int dk, int dv, const Layout &L) {
    size_t fixed = 0;
    if (dk == 64 && dv == 64) fixed = dec_fixed_bytes<64, 64>();
    if (dk == 64 && dv == 128) fixed = dec_fixed_bytes<64, 128>();
    if (dk == 128 && dv == 64) fixed = dec_fixed_bytes<128, 64>();
    if (dk == 128 && dv == 128) fixed = dec_fixed_bytes<128, 128>();
    const size_t stage = (size_t)align_up(L.off_ent + (L.r + L.W) * (L.dk + L.dv) * 4, 16);
    const size_t dots = (size_t)(L.r + L.W + 1) * sizeof(float2);
    return stage + fixed + align_up((int)dots, 16);
}

// Decode one token of one head; FLUSH also ends the window in the same launch.
template <int DK, int DV, bool KDA, bool FLUSH, bool DAMP>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const Layout &L = a.L;
    const int head = blockIdx.x;
    const int b = head / a.H, h = head - b * a.H;
    const int g = (h * a.Hk) / a.H;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int P = DAMP ? L.P : 0;
    const int NI = DK - P;
    const int E = L.r + a.n;  // entries present before this token
    const size_t stage_bytes = (size_t)align_up(L.off_ent + (L.r + L.W) * (DK + DV) * 4, 16);
    unsigned char *stage = smem;
    DecSmem<DK, DV> &S = *reinterpret_cast<DecSmem<DK, DV> *>(smem + stage_bytes);
    float2 *dots = reinterpret_cast<float2 *>(smem + stage_bytes + dec_fixed_bytes<DK, DV>());
    unsigned char *rec = a.rec + (size_t)head * L.rec_bytes;
    float *rec_ent = reinterpret_cast<float *>(rec + L.off_ent);
    float *rec_gam = reinterpret_cast<float *>(rec + L.off_gam);

    if (t == 0) {
        mbar_init(&S.mbar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (t == 0) {
        const uint32_t bytes = (uint32_t)(L.off_ent + E * (DK + DV) * 4);
        mbar_arrive_expect_tx(&S.mbar, bytes);
        bulk_g2s(stage, rec, bytes, &S.mbar);
    }

    // Step inputs and the cumulative gate while the stage is in flight.
    const size_t hv = (size_t)b * a.H + h;
    const size_t qk = ((size_t)b * a.Hk + g) * DK;
    float kqp = 0.f;
    if (t < DK) {
        const float kk = a.k[qk + t], qq = a.q[qk + t];
        const float al = KDA ? a.alpha[hv * DK + t] : a.alpha[hv];
        float gp = 1.0f;
        if (a.n > 0) gp = KDA ? rec_gam[t] : rec_gam[0];
        const float gt = al * gp;
        S.k[t] = kk;
        S.gam[t] = gt;
        S.x2[t] = make_float2(gt * kk, gt * qq);
        kqp = kk * qq;
    }
    if (t < DV) S.v[t] = a.v[hv * DV + t];
    kqp = warp_sum(kqp);
    if (lane == 0) S.kqw[warp] = kqp;
    if (DAMP) build_row_map<DK>(a.hp_rows + (size_t)h * P, P, S.map, S.wscr);
    __syncthreads();
    float kq = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) kq += S.kqw[w];

    const bool ok = mbar_wait_bounded(&S.mbar, 0, a.status);
    if (__syncthreads_or(!ok)) return;

    const float *m_s = reinterpret_cast<const float *>(stage + L.off_m);
    const float *s_s = reinterpret_cast<const float *>(stage + L.off_s);
    const uint16_t *hp_s = reinterpret_cast<const uint16_t *>(stage + L.off_hp);
    const float *ent = reinterpret_cast<const float *>(stage + L.off_ent);

    if (t < DK) {
        const int j = DAMP ? S.map[t] : t;
        if (j >= 0) {
            const float mi = m_s[t];
            const float2 x = S.x2[t];
            S.a2[j] = make_float2(mi * x.x, mi * x.y);
        }
    }
    __syncthreads();

    // Dual GEMV over the INT8 rows.
    constexpr int LPR = DV / 4;    // lanes per row
    constexpr int RPP = 32 / LPR;  // rows per warp pass
    {
        const int cq = lane % LPR, rsub = lane / LPR;
        float ak[4] = {0.f, 0.f, 0.f, 0.f}, aq[4] = {0.f, 0.f, 0.f, 0.f};
        for (int j = warp * RPP + rsub; j < NI; j += kWarps * RPP) {
            const uint32_t w = *reinterpret_cast<const uint32_t *>(stage + (size_t)j * DV + cq * 4);
            float f[4];
            s8x4_to_f(w, f);
            const float2 av = S.a2[j];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                ak[u] = fmaf(f[u], av.x, ak[u]);
                aq[u] = fmaf(f[u], av.y, aq[u]);
            }
        }
        float2 *red = S.red[warp * RPP + rsub];
#pragma unroll
        for (int u = 0; u < 4; ++u) red[cq * 4 + u] = make_float2(ak[u], aq[u]);
    }
    // Buffer / compensator dot products, one warp per entry.
    for (int e = warp; e < E; e += kWarps) {
        const float *kt = ent + (size_t)e * (DK + DV);
        float dk_ = 0.f, dq_ = 0.f;
#pragma unroll
        for (int i = lane; i < DK; i += 32) {
            const float kv = kt[i];
            const float2 x = S.x2[i];
            dk_ = fmaf(kv, x.x, dk_);
            dq_ = fmaf(kv, x.y, dq_);
        }
        dk_ = warp_sum(dk_);
        dq_ = warp_sum(dq_);
        if (lane == 0) dots[e] = make_float2(dk_, dq_);
    }
    __syncthreads();

    // Per value column: finish y_k, y_q; output; the new buffer entry.
    const int En = E;  // slot of the new entry
    if (t < DV) {
        float yk = 0.f, yq = 0.f;
#pragma unroll
        for (int sl = 0; sl < kWarps * RPP; ++sl) {
            const float2 p = S.red[sl][t];
            yk += p.x;
            yq += p.y;
        }
        const float sc = s_s[t];
        yk *= sc;
        yq *= sc;
        if (DAMP) {
            for (int p = 0; p < P; ++p) {
                const int i = a.hp_rows[(size_t)h * P + p];
                const float bv = bf16_to_f(hp_s[(size_t)p * DV + t]);
                const float2 x = S.x2[i];
                yk = fmaf(bv, x.x, yk);
                yq = fmaf(bv, x.y, yq);
            }
        }
        for (int e = 0; e < E; ++e) {
            const float u = ent[(size_t)e * (DK + DV) + DK + t];
            const float2 d = dots[e];
            yk = fmaf(u, d.x, yk);
            yq = fmaf(u, d.y, yq);
        }
        const float beta = a.beta[hv];
        const float ut = beta * (S.v[t] - yk);
        const float o = fmaf(ut, kq, yq);
        a.o[hv * DV + t] = o;
        if (!isfinite(o) || !isfinite(ut)) atomicOr(a.status, kStatusNonFinite);
        if (FLUSH) {
            reinterpret_cast<float *>(stage + L.off_ent)[(size_t)En * (DK + DV) + DK + t] = ut;
        } else {
            rec_ent[(size_t)En * (DK + DV) + DK + t] = ut;
        }
    }
    if (t < DK) {
        const float kt = S.k[t] / S.gam[t];
        if (FLUSH) {
            reinterpret_cast<float *>(stage + L.off_ent)[(size_t)En * (DK + DV) + t] = kt;
        } else {
            rec_ent[(size_t)En * (DK + DV) + t] = kt;
            if (KDA) rec_gam[t] = S.gam[t];
            else if (t == 0) rec_gam[0] = S.gam[0];
        }
    }
    if (!FLUSH) return;

    // ---- window end: reconstruct, re-extract compensators, smooth, pack ----
    __syncthreads();
    using T = Tile<DK, DV>;
    float R[T::RPT][16];
    const bool fin = tile_from_stage<DK, DV>(R, stage, L, P, DAMP ? S.map : nullptr, E + 1, S.gam);
    if (!fin) atomicOr(a.status, kStatusNonFinite);
    CodecOut out;
    out.codes = reinterpret_cast<int8_t *>(rec);
    out.hp = reinterpret_cast<uint16_t *>(rec + L.off_hp);
    out.m = reinterpret_cast<float *>(rec + L.off_m);
    out.s = reinterpret_cast<float *>(rec + L.off_s);
    out.ck = rec_ent;
    out.ck_stride = DK + DV;
    out.cw = rec_ent + DK;
    out.cw_stride = DK + DV;
    double eacc[T::RPT];
    codec_quantize<DK, DV, false>(R, L.r, a.K, a.smoothing, P, DAMP ? S.map : nullptr, S.cs, out, eacc);
    if (KDA) {
        if (t < DK) rec_gam[t] = 1.0f;
    } else if (t == 0) {
        rec_gam[0] = 1.0f;
    }
}

// Stage a head's record prefix with E entries (used by flush / export).
template <int DK, int DV>
__device__ inline bool stage_record(unsigned char *stage, const unsigned char *rec, const Layout &L, int E,
                                    uint64_t *mbar, int *status) {
    if (threadIdx.x == 0) {
        mbar_init(mbar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t bytes = (uint32_t)(L.off_ent + E * (DK + DV) * 4);
        mbar_arrive_expect_tx(mbar, bytes);
        bulk_g2s(stage, rec, bytes, mbar);
    }
    const bool ok = mbar_wait_bounded(mbar, 0, status);
    return !__syncthreads_or(!ok);
}

// End a window (n >= 1 tokens buffered), or (EXPORT) write the current state.
template <int DK, int DV, bool KDA, bool DAMP, bool EXPORT>
__global__ void __launch_bounds__(kThreads) flush_kernel(const DecodeArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const Layout &L = a.L;
    const int head = blockIdx.x;
    const int h = head % a.H;
    const int t = threadIdx.x;
    const int P = DAMP ? L.P : 0;
    const int E = L.r + a.n;
    const size_t stage_bytes = (size_t)align_up(L.off_ent + (L.r + L.W) * (DK + DV) * 4, 16);
    unsigned char *stage = smem;
    DecSmem<DK, DV> &S = *reinterpret_cast<DecSmem<DK, DV> *>(smem + stage_bytes);
    unsigned char *rec = a.rec + (size_t)head * L.rec_bytes;
    float *rec_ent = reinterpret_cast<float *>(rec + L.off_ent);
    float *rec_gam = reinterpret_cast<float *>(rec + L.off_gam);
    if (t < DK) S.gam[t] = (a.n == 0) ? 1.0f : (KDA ? rec_gam[t] : rec_gam[0]);
    if (DAMP) build_row_map<DK>(a.hp_rows + (size_t)h * P, P, S.map, S.wscr);
    if (!stage_record<DK, DV>(stage, rec, L, E, &S.mbar, a.status)) return;
    using T = Tile<DK, DV>;
    float R[T::RPT][16];
    const bool fin = tile_from_stage<DK, DV>(R, stage, L, P, DAMP ? S.map : nullptr, E, S.gam);
    if (!fin) atomicOr(a.status, kStatusNonFinite);
    if (EXPORT) {
        const int cg = t % T::CG, row0 = (t / T::CG) * T::RPT;
        float *dst = a.S_out + (size_t)head * DK * DV;
#pragma unroll
        for (int r = 0; r < T::RPT; ++r)
#pragma unroll
            for (int q = 0; q < 4; ++q)
                reinterpret_cast<float4 *>(dst + (size_t)(row0 + r) * DV + cg * 16)[q] =
                    make_float4(R[r][4 * q], R[r][4 * q + 1], R[r][4 * q + 2], R[r][4 * q + 3]);
        return;
    }
    CodecOut out;
    out.codes = reinterpret_cast<int8_t *>(rec);
    out.hp = reinterpret_cast<uint16_t *>(rec + L.off_hp);
    out.m = reinterpret_cast<float *>(rec + L.off_m);
    out.s = reinterpret_cast<float *>(rec + L.off_s);
    out.ck = rec_ent;
    out.ck_stride = DK + DV;
    out.cw = rec_ent + DK;
    out.cw_stride = DK + DV;
    double eacc[T::RPT];
    codec_quantize<DK, DV, false>(R, L.r, a.K, a.smoothing, P, DAMP ? S.map : nullptr, S.cs, out, eacc);
    if (KDA) {
        if (t < DK) rec_gam[t] = 1.0f;
    } else if (t == 0) {
        rec_gam[0] = 1.0f;
    }
}

// FP32-state reference step: S' = D S; y = S'^T k; u = beta (v - y);
// S = S' + k u^T; o = S'^T q + u (k . q).  One CTA per head; the state is read
// once into registers (a warp covers whole rows with 16-byte loads) and
// written once.
template <int DK, int DV, bool KDA>
__global__ void __launch_bounds__(kThreads) fp32_step_kernel(const Fp32Args a) {
    constexpr int LPR = DV / 4, RPP = 32 / LPR, ROWS = DK / (kWarps * RPP);
    __shared__ float k_s[DK], q_s[DK], d_s[DK];
    __shared__ float2 red[kWarps * RPP][DV];
    __shared__ float kqw[kWarps];
    const int head = blockIdx.x;
    const int b = head / a.H, h = head - b * a.H, g = (h * a.Hk) / a.H;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int cq = lane % LPR, rsub = lane / LPR;
    const size_t hv = (size_t)b * a.H + h;
    const size_t qk = ((size_t)b * a.Hk + g) * DK;
    float *Sh = a.S + (size_t)head * DK * DV;

    float4 Sv[ROWS];
#pragma unroll
    for (int p = 0; p < ROWS; ++p) {
        const int i = (warp * RPP + rsub) + p * kWarps * RPP;
        Sv[p] = __ldcs(reinterpret_cast<const float4 *>(Sh + (size_t)i * DV) + cq);
    }
    float kqp = 0.f;
    if (t < DK) {
        const float kk = a.k[qk + t], qq = a.q[qk + t];
        k_s[t] = kk;
        q_s[t] = qq;
        d_s[t] = KDA ? a.alpha[hv * DK + t] : a.alpha[hv];
        kqp = kk * qq;
    }
    kqp = warp_sum(kqp);
    if (lane == 0) kqw[warp] = kqp;
    __syncthreads();
    float yk[4] = {0.f, 0.f, 0.f, 0.f}, yq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int p = 0; p < ROWS; ++p) {
        const int i = (warp * RPP + rsub) + p * kWarps * RPP;
        const float d = d_s[i], kk = k_s[i], qq = q_s[i];
        Sv[p].x *= d; Sv[p].y *= d; Sv[p].z *= d; Sv[p].w *= d;
        yk[0] = fmaf(kk, Sv[p].x, yk[0]); yk[1] = fmaf(kk, Sv[p].y, yk[1]);
        yk[2] = fmaf(kk, Sv[p].z, yk[2]); yk[3] = fmaf(kk, Sv[p].w, yk[3]);
        yq[0] = fmaf(qq, Sv[p].x, yq[0]); yq[1] = fmaf(qq, Sv[p].y, yq[1]);
        yq[2] = fmaf(qq, Sv[p].z, yq[2]); yq[3] = fmaf(qq, Sv[p].w, yq[3]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) red[warp * RPP + rsub][cq * 4 + u] = make_float2(yk[u], yq[u]);
    __syncthreads();
    __shared__ float u_s[DV];
    if (t < DV) {
        float a_k = 0.f, a_q = 0.f;
#pragma unroll
        for (int sl = 0; sl < kWarps * RPP; ++sl) {
            a_k += red[sl][t].x;
            a_q += red[sl][t].y;
        }
        float kq = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) kq += kqw[w];
        const float ut = a.beta[hv] * (a.v[hv * DV + t] - a_k);
        u_s[t] = ut;
        const float o = fmaf(ut, kq, a_q);
        a.o[hv * DV + t] = o;
        if (!isfinite(o)) atomicOr(a.status, kStatusNonFinite);
    }
    __syncthreads();
    const float4 uv = reinterpret_cast<const float4 *>(u_s)[cq];
#pragma unroll
    for (int p = 0; p < ROWS; ++p) {
        const int i = (warp * RPP + rsub) + p * kWarps * RPP;
        const float kk = k_s[i];
        float4 o = Sv[p];
        o.x = fmaf(kk, uv.x, o.x); o.y = fmaf(kk, uv.y, o.y);
        o.z = fmaf(kk, uv.z, o.z); o.w = fmaf(kk, uv.w, o.w);
        __stcs(reinterpret_cast<float4 *>(Sh + (size_t)i * DV) + cq, o);
    }
}

// ---------------------------------------------------------------------------
// Host-side launchers (called from the C ABI).
// ---------------------------------------------------------------------------
// Raise a kernel's dynamic shared memory limit when a launch first needs more
// than it was set to.  `done` must be distinct for every kernel, so each
// launcher below keeps its own.
template <typename K>
static cudaError_t set_smem(K kern, size_t bytes, size_t &done) {
    if (bytes <= done) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) done = bytes;
    return e;
}

template <int DK, int DV, bool KDA, bool FLUSH, bool DAMP>
static cudaError_t launch_decode_t(const DecodeArgs &a, int heads, cudaStream_t s) {
    const size_t sm = decode_smem_bytes(DK, DV, a.L);
    auto kern = decode_kernel<DK, DV, KDA, FLUSH, DAMP>;
    static size_t done = 0;  // one per instantiation of this launcher
    cudaError_t e = set_smem(kern, sm, done);
    if (e != cudaSuccess) return e;
    kern<<<heads, kThreads, sm, s>>>(a);
    return cudaGetLastError();
}

template <int DK, int DV, bool KDA, bool DAMP, bool EXPORT>
static cudaError_t launch_flush_t(const DecodeArgs &a, int heads, cudaStream_t s) {
    const size_t sm = decode_smem_bytes(DK, DV, a.L);
    auto kern = flush_kernel<DK, DV, KDA, DAMP, EXPORT>;
    static size_t done = 0;  // one per instantiation of this launcher
    cudaError_t e = set_smem(kern, sm, done);
    if (e != cudaSuccess) return e;
    kern<<<heads, kThreads, sm, s>>>(a);
    return cudaGetLastError();
}

#define LQ_DISPATCH_DKDV(dk, dv, FN)                   \
    (((dk) == 128 && (dv) == 128)  ? FN<128, 128>      \
     : ((dk) == 64 && (dv) == 64)  ? FN<64, 64>        \
     : ((dk) == 64 && (dv) == 128) ? FN<64, 128>       \
                                   : FN<128, 64>)

template <int DK, int DV>
static cudaError_t decode_dispatch(const DecodeArgs &a, int heads, bool kda, bool flush, bool damp,
                                   cudaStream_t s) {
    if (kda) {
        if (flush) return damp ? launch_decode_t<DK, DV, true, true, true>(a, heads, s)
                               : launch_decode_t<DK, DV, true, true, false>(a, heads, s);
        return damp ? launch_decode_t<DK, DV, true, false, true>(a, heads, s)
                    : launch_decode_t<DK, DV, true, false, false>(a, heads, s);
    }
    if (flush) return damp ? launch_decode_t<DK, DV, false, true, true>(a, heads, s)
                           : launch_decode_t<DK, DV, false, true, false>(a, heads, s);
    return damp ? launch_decode_t<DK, DV, false, false, true>(a, heads, s)
                : launch_decode_t<DK, DV, false, false, false>(a, heads, s);
}

template <int DK, int DV>
static cudaError_t flush_dispatch(const DecodeArgs &a, int heads, bool kda, bool damp, bool exp,
                                  cudaStream_t s) {
    if (exp) {
        if (kda) return damp ? launch_flush_t<DK, DV, true, true, true>(a, heads, s)
                             : launch_flush_t<DK, DV, true, false, true>(a, heads, s);
        return damp ? launch_flush_t<DK, DV, false, true, true>(a, heads, s)
                    : launch_flush_t<DK, DV, false, false, true>(a, heads, s);
    }
    if (kda) return damp ? launch_flush_t<DK, DV, true, true, false>(a, heads, s)
                         : launch_flush_t<DK, DV, true, false, false>(a, heads, s);
    return damp ? launch_flush_t<DK, DV, false, true, false>(a, heads, s)
                : launch_flush_t<DK, DV, false, false, false>(a, heads, s);
}

template <int DK, int DV>
static cudaError_t fp32_dispatch(const Fp32Args &a, int heads, bool kda, cudaStream_t s) {
    if (kda) fp32_step_kernel<DK, DV, true><<<heads, kThreads, 0, s>>>(a);
    else fp32_step_kernel<DK, DV, false><<<heads, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool flush, bool damp,
                          cudaStream_t s) {
    return LQ_DISPATCH_DKDV(dk, dv, decode_dispatch)(a, heads, kda, flush, damp, s);
}

cudaError_t launch_flush(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool damp, bool exp,
                         cudaStream_t s) {
    return LQ_DISPATCH_DKDV(dk, dv, flush_dispatch)(a, heads, kda, damp, exp, s);
}

cudaError_t launch_fp32_step(const Fp32Args &a, int dk, int dv, int heads, bool kda, cudaStream_t s) {
    return LQ_DISPATCH_DKDV(dk, dv, fp32_dispatch)(a, heads, kda, s);
}

}  // namespace lq
