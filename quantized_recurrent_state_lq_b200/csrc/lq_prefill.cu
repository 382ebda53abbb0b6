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
// One CTA of 2 dv threads per head (two per SM), the state in registers for
// the whole run (below); the chunk's keys, queries and decays are staged in
// shared memory.  The three d_k x d_v products run on the tensor cores in
// three TF32 passes (FP32-level accuracy); the pair matrices, the forward
// substitution and the outputs in FP32.
#include "lq_common.cuh"
#include "lq_prefill.h"
#include "lq_tc.cuh"

namespace lq {

constexpr int kChunk = 16;

// ---------------------------------------------------------------------------
// The chunk step on the tensor cores.  Warp w owns value columns
// 16w .. 16w+15 and keeps S^T for them in registers as mma.sync m16n8k8
// accumulator tiles (M = 16 columns, N = 8 key rows per tile): thread (g, q)
// of a tile holds S[8nb+2q][c0+g], S[8nb+2q+1][c0+g], S[8nb+2q][c0+g+8],
// S[8nb+2q+1][c0+g+8].  Read with the key rows of each 8-row block ordered
// 0, 2, 4, 6, 1, 3, 5, 7, the same registers are the A operand (M = columns,
// K = rows) of S^T (Gamma k)^T, so the products need no data movement:
//   Y^T = S^T Kg^T, Oi^T = S^T Qg^T   (M = 16 columns, N = 8 tokens, K = rows)
//   S^T <- Gamma_C S^T + U^T Kh        (M = 16 columns, N = 8 rows, K = tokens)
// Every product is three TF32 MMAs (big x big + big x small + small x big of
// the operands' split, FP32-level accuracy).  Each warp holds all key rows of
// its columns, so no product needs a reduction across warps; the forward
// substitution of the pseudo-values runs one column per lane of the warp.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D += A B in three TF32 passes; A given split, B as two floats.
__device__ __forceinline__ void mma3(float (&d)[4], const uint32_t (&ab)[4], const uint32_t (&as)[4], float b0,
                                     float b1) {
    uint32_t bb0, bs0, bb1, bs1;
    tf32_split(b0, bb0, bs0);
    tf32_split(b1, bb1, bs1);
    mma_tf32_16x8x8(d, as, bb0, bb1);
    mma_tf32_16x8x8(d, ab, bs0, bs1);
    mma_tf32_16x8x8(d, ab, bb0, bb1);
}

template <int DK, int DV, bool KDA>
struct PrefillTcSmem {
    static constexpr int GC = KDA ? DK : 1;
    static constexpr int CP = kChunk + 1;   // transposed rows, padded
    static constexpr int KP = DK + 8;       // token rows of the MMA operands, padded
    static constexpr int VP = DV + 8;       // u: A-fragment reads free of bank conflicts
    static constexpr int YP = DV + 4;       // y, oi: fragment stores free of bank conflicts
    alignas(16) float kg[kChunk][KP];       // Gamma_t k_t (read as float2)
    alignas(16) float qg[kChunk][KP];       // Gamma_t q_t
    float kh[kChunk][KP];                   // Gamma_C / Gamma_t k_t
    float y[kChunk][YP], oi[kChunk][YP];    // S^T (Gamma k), S^T (Gamma q)
    float u[kChunk][VP];                    // pseudo-values
    float v[kChunk][DV];
    float kT[DK][CP], qT[DK][CP];           // raw k^T, q^T (pair matrices)
    float g[GC][CP];                        // cumulative log2 decay
    float beta[kChunk];
    float A[kChunk][kChunk], P[kChunk][kChunk];
    float glast[DK];
};

template <int DK, int DV, bool KDA>
__global__ void __launch_bounds__(2 * DV, 2) prefill_tc_kernel(const PrefillArgs a) {
    constexpr int NT = 2 * DV, C = kChunk, NB = DK / 8;
    using Sm = PrefillTcSmem<DK, DV, KDA>;
    constexpr int GC = Sm::GC;
    (void)GC;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Sm &S = *reinterpret_cast<Sm *>(smem_raw);
    const int head = blockIdx.x;
    const int b = head / a.H, h = head - b * a.H, gk = (h * a.Hk) / a.H;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int gq = lane >> 2, tq = lane & 3, c0 = 16 * warp;
    const size_t state_off = (size_t)head * DK * DV;

    // S^T tiles: st[nb][0..3] = S[8nb+2tq][c0+gq], S[8nb+2tq+1][c0+gq],
    //                           S[8nb+2tq][c0+gq+8], S[8nb+2tq+1][c0+gq+8]
    float st[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        const int r = 8 * nb + 2 * tq;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int rr = r + (e & 1), cc = c0 + gq + 8 * (e >> 1);
            st[nb][e] = a.S0 ? a.S0[state_off + (size_t)rr * DV + cc] : 0.0f;
        }
    }

    const int nchunks = (a.T + C - 1) / C;
    for (int ch = 0; ch < nchunks; ++ch) {
        const int t0 = ch * C;
        // (0) inputs; tokens past T are identity steps
        for (int e = t; e < C * DK; e += NT) {
            const int tt = e / DK, r = e % DK, tok = t0 + tt;
            float kv = 0.f, qv = 0.f, gl = 0.f;
            if (tok < a.T) {
                const size_t qk = (((size_t)tok * a.B + b) * a.Hk + gk) * DK + r;
                kv = a.k[qk];
                qv = a.q[qk];
                if (KDA) gl = fmaxf(log2f(a.alpha[(((size_t)tok * a.B + b) * a.H + h) * DK + r]), -150.0f);
            }
            S.kT[r][tt] = kv;
            S.qT[r][tt] = qv;
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
        // the next chunk's input lines into L2 while this chunk computes: per
        // token k, q (one q/k head), v and a per-channel gate, 128-byte lines
        {
            constexpr int LK = DK / 32, LV = DV / 32;          // lines per vector
            constexpr int LT = 2 * LK + LV + (KDA ? LK : 0);   // lines per token
            const int tok = t0 + C + t / LT, l = t % LT;
            if (t < C * LT && tok < a.T) {
                const float *p;
                const size_t qk = (((size_t)tok * a.B + b) * a.Hk + gk) * DK;
                const size_t hv = ((size_t)tok * a.B + b) * a.H + h;
                if (l < LK) p = a.k + qk + 32 * l;
                else if (l < 2 * LK) p = a.q + qk + 32 * (l - LK);
                else if (l < 2 * LK + LV) p = a.v + hv * DV + 32 * (l - 2 * LK);
                else p = a.alpha + hv * DK + 32 * (l - 2 * LK - LV);
                asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
            }
        }
        // (1) cumulative log2 decay
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
        // (2) decayed operands (token-major) and the pair matrices
        for (int e = t; e < C * DK; e += NT) {
            const int r = e % DK, tt = e / DK;
            const float gt = S.g[KDA ? r : 0][tt], gC = S.g[KDA ? r : 0][C - 1];
            const float et = exp2f(gt);
            S.kg[tt][r] = S.kT[r][tt] * et;
            S.qg[tt][r] = S.qT[r][tt] * et;
            S.kh[tt][r] = S.kT[r][tt] * exp2f(gC - gt);
        }
        for (int pr = t; pr < C * C; pr += NT) {
            const int ti = pr / C, ii = pr % C;
            float dkk = 0.f, dqk = 0.f;
            if (ii <= ti) {
                if (KDA) {
#pragma unroll 8
                    for (int r = 0; r < DK; ++r) {
                        const float f = exp2f(S.g[r][ti] - S.g[r][ii]) * S.kT[r][ii];
                        dkk = fmaf(S.kT[r][ti], f, dkk);
                        dqk = fmaf(S.qT[r][ti], f, dqk);
                    }
                } else {
#pragma unroll 8
                    for (int r = 0; r < DK; ++r) {
                        dkk = fmaf(S.kT[r][ti], S.kT[r][ii], dkk);
                        dqk = fmaf(S.qT[r][ti], S.kT[r][ii], dqk);
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
        // (3) Y^T = S^T Kg^T and Oi^T = S^T Qg^T on the tensor cores
        {
            float dy[2][4] = {}, dq[2][4] = {};
#pragma unroll
            for (int kb = 0; kb < NB; ++kb) {
                uint32_t ab[4], as[4];
                // A: rows 8kb+2tq (k = tq) and 8kb+2tq+1 (k = tq+4)
                tf32_split(st[kb][0], ab[0], as[0]);
                tf32_split(st[kb][2], ab[1], as[1]);
                tf32_split(st[kb][1], ab[2], as[2]);
                tf32_split(st[kb][3], ab[3], as[3]);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const float2 kv = *reinterpret_cast<const float2 *>(&S.kg[8 * nt + gq][8 * kb + 2 * tq]);
                    const float2 qv = *reinterpret_cast<const float2 *>(&S.qg[8 * nt + gq][8 * kb + 2 * tq]);
                    mma3(dy[nt], ab, as, kv.x, kv.y);
                    mma3(dq[nt], ab, as, qv.x, qv.y);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int tt = 8 * nt + 2 * tq;
                S.y[tt][c0 + gq] = dy[nt][0];
                S.y[tt + 1][c0 + gq] = dy[nt][1];
                S.y[tt][c0 + gq + 8] = dy[nt][2];
                S.y[tt + 1][c0 + gq + 8] = dy[nt][3];
                S.oi[tt][c0 + gq] = dq[nt][0];
                S.oi[tt + 1][c0 + gq] = dq[nt][1];
                S.oi[tt][c0 + gq + 8] = dq[nt][2];
                S.oi[tt + 1][c0 + gq + 8] = dq[nt][3];
            }
        }
        __syncwarp();
        // (4) pseudo-values by forward substitution and the outputs, a column per lane
        if (lane < 16) {
            const int cc = c0 + lane;
            float u[C];
#pragma unroll
            for (int tt = 0; tt < C; ++tt) {
                float x = S.beta[tt] * (S.v[tt][cc] - S.y[tt][cc]);
#pragma unroll
                for (int i = 0; i < tt; ++i) x = fmaf(-S.A[tt][i], u[i], x);
                u[tt] = x;
                S.u[tt][cc] = x;
            }
            if (a.o) {
#pragma unroll
                for (int tt = 0; tt < C; ++tt) {
                    const int tok = t0 + tt;
                    float x = S.oi[tt][cc];
#pragma unroll
                    for (int i = 0; i <= tt; ++i) x = fmaf(S.P[tt][i], u[i], x);
                    if (tok < a.T) a.o[(((size_t)tok * a.B + b) * a.H + h) * DV + cc] = x;
                }
            }
        }
        __syncwarp();
        // (5) S^T <- Gamma_C S^T + U^T Kh on the tensor cores
        {
            uint32_t ub[2][4], us[2][4];
#pragma unroll
            for (int kt = 0; kt < 2; ++kt) {
                const int tt = 8 * kt + tq;
                tf32_split(S.u[tt][c0 + gq], ub[kt][0], us[kt][0]);
                tf32_split(S.u[tt][c0 + gq + 8], ub[kt][1], us[kt][1]);
                tf32_split(S.u[tt + 4][c0 + gq], ub[kt][2], us[kt][2]);
                tf32_split(S.u[tt + 4][c0 + gq + 8], ub[kt][3], us[kt][3]);
            }
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int r = 8 * nb + 2 * tq;
                const float g0 = S.glast[r], g1 = S.glast[r + 1];
                st[nb][0] *= g0;
                st[nb][1] *= g1;
                st[nb][2] *= g0;
                st[nb][3] *= g1;
#pragma unroll
                for (int kt = 0; kt < 2; ++kt)
                    mma3(st[nb], ub[kt], us[kt], S.kh[8 * kt + tq][8 * nb + gq], S.kh[8 * kt + tq + 4][8 * nb + gq]);
            }
        }
        __syncthreads();
    }
    bool fin = true;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        const int r = 8 * nb + 2 * tq;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int rr = r + (e & 1), cc = c0 + gq + 8 * (e >> 1);
            fin = fin && isfinite(st[nb][e]);
            a.S_out[state_off + (size_t)rr * DV + cc] = st[nb][e];
        }
    }
    if (!fin && a.status) atomicOr(a.status, kStatusNonFinite);
}

template <int DK, int DV>
size_t prefill_smem_bytes_t(bool kda) {
    return kda ? sizeof(PrefillTcSmem<DK, DV, true>) : sizeof(PrefillTcSmem<DK, DV, false>);
}

template <int DK, int DV>
static cudaError_t prefill_dispatch(const PrefillArgs &a, int heads, bool kda, cudaStream_t s) {
    const size_t sm = prefill_smem_bytes_t<DK, DV>(kda);
    auto kern = kda ? prefill_tc_kernel<DK, DV, true> : prefill_tc_kernel<DK, DV, false>;
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
