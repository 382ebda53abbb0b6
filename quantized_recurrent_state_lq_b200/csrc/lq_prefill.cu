// lq_prefill.cu -- chunked prefill of the recurrence (the step before the
// windowed decode): T tokens of S_t = (I - b k k^T) D_t S_{t-1} + b k v^T,
// o_t = S_t^T q_t (LinQuant appendix Table 3, key-rows form; decay first,
// then the delta projection) from an FP32 state, in chunks of kChunk tokens.
//
// Within a chunk starting from state S, with g_t the cumulative log2 decay of
// tokens 1..t of the chunk (per key channel for KDA, one value for GDN) and
// Gamma_t = 2^g_t, the state after token t is
//   S_t = diag(Gamma_t) S + sum_{i<=t} diag(Gamma_t / Gamma_i) k_i u_i^T
// (the WY form of the product of the chunk's rank-one updates), where the
// pseudo-values u_t follow from the rank-one form u_t = b_t (v_t - (D_t
// S_{t-1})^T k_t) by forward substitution:
//   u_t = b_t (v_t - S^T (Gamma_t k_t)) - sum_{i<t} A_ti u_i,
//   A_ti = b_t sum_c k_tc k_ic Gamma_tc / Gamma_ic,
// the outputs are
//   o_t = S^T (Gamma_t q_t) + sum_{i<=t} P_ti u_i,  P_ti = sum_c q_tc k_ic Gamma_tc / Gamma_ic,
// and the chunk ends with S <- diag(Gamma_C) S + sum_i diag(Gamma_C / Gamma_i) k_i u_i^T.
// Every decay factor is 2^(g_t - g_i) with i <= t, or 2^g_t: never above 1
// for gates in (0, 1], so nothing overflows however strong the decay.
//
// One CTA of 2 dv threads per head (two per SM): thread (c, half) holds key
// rows half * dk/2 .. + dk/2 of value column c of the state in registers for
// the whole run; the chunk's keys, queries and decays are staged in shared memory
// and read as broadcasts.  FP32 arithmetic (FMA), the products ordered as
// written above.
#include "lq_common.cuh"
#include "lq_prefill.h"

namespace lq {

constexpr int kChunk = 16;

template <int DK, int DV, bool KDA>
struct PrefillSmem {
    static constexpr int GC = KDA ? DK : 1;   // decay channels
    static constexpr int CP = kChunk + 1;     // padded row: column access free of bank conflicts
    float kg_t[DK][kChunk];   // (Gamma_t k_t)^T, rows read as float4
    float qg_t[DK][kChunk];   // (Gamma_t q_t)^T
    float kh_t[DK][kChunk];   // (Gamma_C / Gamma_t k_t)^T
    float k[DK][CP];          // k^T, q^T as staged
    float q[DK][CP];
    float g[GC][CP];          // cumulative log2 decay within the chunk, per channel
    float v[kChunk][DV];
    float beta[kChunk];
    float A[kChunk][kChunk];
    float P[kChunk][kChunk];
    float yp[2][kChunk][DV];  // per row half: S^T (Gamma_t k_t)
    float op[2][kChunk][DV];  // per row half: S^T (Gamma_t q_t)
    float glast[DK];          // Gamma_C per key row
};

template <int DK, int DV>
size_t prefill_smem_bytes_t(bool kda) {
    return kda ? sizeof(PrefillSmem<DK, DV, true>) : sizeof(PrefillSmem<DK, DV, false>);
}

template <int DK, int DV, bool KDA>
__global__ void __launch_bounds__(2 * DV, 2) prefill_kernel(const PrefillArgs a) {
    constexpr int NT = 2 * DV, RH = DK / 2, C = kChunk;
    using Sm = PrefillSmem<DK, DV, KDA>;
    constexpr int GC = Sm::GC;
    (void)GC;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Sm &S = *reinterpret_cast<Sm *>(smem_raw);
    const int head = blockIdx.x;
    const int b = head / a.H, h = head - b * a.H, g = (h * a.Hk) / a.H;
    const int t = threadIdx.x, c = t % DV, half = t / DV, r0 = half * RH;
    const size_t state_off = (size_t)head * DK * DV;

    float Sr[RH];
#pragma unroll
    for (int j = 0; j < RH; ++j) Sr[j] = a.S0 ? a.S0[state_off + (size_t)(r0 + j) * DV + c] : 0.0f;

    const int nchunks = (a.T + C - 1) / C;
    for (int ch = 0; ch < nchunks; ++ch) {
        const int t0 = ch * C;
        // (0) the chunk's inputs; tokens past T are identity steps (b = 0,
        // decay 1, zero vectors) and write nothing
        for (int e = t; e < C * DK; e += NT) {
            const int tt = e / DK, r = e % DK, tok = t0 + tt;
            float kv = 0.f, qv = 0.f, gl = 0.f;
            if (tok < a.T) {
                const size_t qk = (((size_t)tok * a.B + b) * a.Hk + g) * DK + r;
                kv = a.k[qk];
                qv = a.q[qk];
                if (KDA) gl = fmaxf(log2f(a.alpha[(((size_t)tok * a.B + b) * a.H + h) * DK + r]), -150.0f);
            }
            S.k[r][tt] = kv;
            S.q[r][tt] = qv;
            if (KDA) S.g[r][tt] = gl;
        }
        for (int e = t; e < C * DV; e += NT) {
            const int tt = e / DV, cc = e % DV, tok = t0 + tt;
            S.v[tt][cc] = tok < a.T ? a.v[(((size_t)tok * a.B + b) * a.H + h) * DV + cc] : 0.f;
        }
        if (t < C) {
            const int tok = t0 + t;
            const size_t bh = ((size_t)tok * a.B + b) * a.H + h;
            S.beta[t] = tok < a.T ? a.beta[bh] : 0.f;
            if (!KDA) S.g[0][t] = tok < a.T ? fmaxf(log2f(a.alpha[bh]), -150.0f) : 0.f;
        }
        __syncthreads();
        // (1) cumulative log2 decay per channel
        if (t < GC) {
            float acc = 0.f;
#pragma unroll
            for (int tt = 0; tt < C; ++tt) {
                acc += S.g[t][tt];
                S.g[t][tt] = acc;
            }
            S.glast[KDA ? t : 0] = exp2f(acc);
        }
        __syncthreads();
        if (!KDA && t < DK && t > 0) S.glast[t] = S.glast[0];
        // (2) decayed keys / queries, and the chunk's pair matrices
        for (int e = t; e < C * DK; e += NT) {
            const int tt = e % C, r = e / C;
            const float gt = S.g[KDA ? r : 0][tt], gC = S.g[KDA ? r : 0][C - 1];
            const float et = exp2f(gt);
            S.kg_t[r][tt] = S.k[r][tt] * et;
            S.qg_t[r][tt] = S.q[r][tt] * et;
            S.kh_t[r][tt] = S.k[r][tt] * exp2f(gC - gt);
        }
        for (int pr = t; pr < C * C; pr += NT) {
            const int ti = pr / C, ii = pr % C;
            float dkk = 0.f, dqk = 0.f;
            if (ii <= ti) {
                if (KDA) {
#pragma unroll 8
                    for (int r = 0; r < DK; ++r) {
                        const float f = exp2f(S.g[r][ti] - S.g[r][ii]) * S.k[r][ii];
                        dkk = fmaf(S.k[r][ti], f, dkk);
                        dqk = fmaf(S.q[r][ti], f, dqk);
                    }
                } else {
#pragma unroll 8
                    for (int r = 0; r < DK; ++r) {
                        dkk = fmaf(S.k[r][ti], S.k[r][ii], dkk);
                        dqk = fmaf(S.q[r][ti], S.k[r][ii], dqk);
                    }
                    const float f = exp2f(S.g[0][ti] - S.g[0][ii]);
                    dkk *= f;
                    dqk *= f;
                }
            }
            S.A[ti][ii] = ii < ti ? S.beta[ti] * dkk : 0.f;
            S.P[ti][ii] = ii <= ti ? dqk : 0.f;
        }
        __syncthreads();
        // (3) S^T (Gamma_t k_t) and S^T (Gamma_t q_t) over this thread's rows,
        // one product at a time (few accumulators beside the state)
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
            float y[C];
#pragma unroll
            for (int tt = 0; tt < C; ++tt) y[tt] = 0.f;
            const float(*xt)[C] = which ? S.qg_t : S.kg_t;
#pragma unroll
            for (int jj = 0; jj < RH; ++jj) {
                const float s = Sr[jj];
                const float4 *xr = reinterpret_cast<const float4 *>(xt[r0 + jj]);
#pragma unroll
                for (int u = 0; u < C / 4; ++u) {
                    const float4 xv = xr[u];
                    y[4 * u] = fmaf(xv.x, s, y[4 * u]);
                    y[4 * u + 1] = fmaf(xv.y, s, y[4 * u + 1]);
                    y[4 * u + 2] = fmaf(xv.z, s, y[4 * u + 2]);
                    y[4 * u + 3] = fmaf(xv.w, s, y[4 * u + 3]);
                }
            }
            float(*dst)[DV] = which ? S.op[half] : S.yp[half];
#pragma unroll
            for (int tt = 0; tt < C; ++tt) dst[tt][c] = y[tt];
        }
        __syncthreads();
        // (4) pseudo-values by forward substitution (both halves of a column
        // compute them), outputs (half 0)
        float u[C];
#pragma unroll
        for (int tt = 0; tt < C; ++tt) {
            float x = S.beta[tt] * (S.v[tt][c] - (S.yp[0][tt][c] + S.yp[1][tt][c]));
#pragma unroll
            for (int i = 0; i < tt; ++i) x = fmaf(-S.A[tt][i], u[i], x);
            u[tt] = x;
        }
        if (half == 0 && a.o) {
#pragma unroll
            for (int tt = 0; tt < C; ++tt) {
                const int tok = t0 + tt;
                float x = S.op[0][tt][c] + S.op[1][tt][c];
#pragma unroll
                for (int i = 0; i <= tt; ++i) x = fmaf(S.P[tt][i], u[i], x);
                if (tok < a.T) a.o[(((size_t)tok * a.B + b) * a.H + h) * DV + c] = x;
            }
        }
        // (5) the state after the chunk
#pragma unroll
        for (int j = 0; j < RH; ++j) {
            const float4 *kr = reinterpret_cast<const float4 *>(S.kh_t[r0 + j]);
            float s = S.glast[r0 + j] * Sr[j];
#pragma unroll
            for (int uu = 0; uu < C / 4; ++uu) {
                const float4 kv = kr[uu];
                s = fmaf(kv.x, u[4 * uu], s);
                s = fmaf(kv.y, u[4 * uu + 1], s);
                s = fmaf(kv.z, u[4 * uu + 2], s);
                s = fmaf(kv.w, u[4 * uu + 3], s);
            }
            Sr[j] = s;
        }
        __syncthreads();
    }
    bool fin = true;
#pragma unroll
    for (int j = 0; j < RH; ++j) {
        fin = fin && isfinite(Sr[j]);
        a.S_out[state_off + (size_t)(r0 + j) * DV + c] = Sr[j];
    }
    if (!fin && a.status) atomicOr(a.status, kStatusNonFinite);
}

template <int DK, int DV>
static cudaError_t prefill_dispatch(const PrefillArgs &a, int heads, bool kda, cudaStream_t s) {
    const size_t sm = prefill_smem_bytes_t<DK, DV>(kda);
    auto kern = kda ? prefill_kernel<DK, DV, true> : prefill_kernel<DK, DV, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    kern<<<heads, 2 * DV, sm, s>>>(a);
    return cudaGetLastError();
}

size_t prefill_smem_bytes(int dk, int dv, bool kda) {
    if (dk == 128 && dv == 128) return prefill_smem_bytes_t<128, 128>(kda);
    if (dk == 64 && dv == 64) return prefill_smem_bytes_t<64, 64>(kda);
    if (dk == 64 && dv == 128) return prefill_smem_bytes_t<64, 128>(kda);
    return prefill_smem_bytes_t<128, 64>(kda);
}

cudaError_t launch_prefill(const PrefillArgs &a, int dk, int dv, int heads, bool kda, cudaStream_t s) {
    if (dk == 128 && dv == 128) return prefill_dispatch<128, 128>(a, heads, kda, s);
    if (dk == 64 && dv == 64) return prefill_dispatch<64, 64>(a, heads, kda, s);
    if (dk == 64 && dv == 128) return prefill_dispatch<64, 128>(a, heads, kda, s);
    return prefill_dispatch<128, 64>(a, heads, kda, s);
}

}  // namespace lq
