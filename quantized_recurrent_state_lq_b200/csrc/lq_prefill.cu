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
// Two kernels, one CTA per head, products in three TF32 passes on the tensor
// cores (FP32-level accuracy), substitutions in FP32:
//   prefill_umma_kernel (d_k = d_v = 128, 16-byte aligned rows): the state in
//     tensor memory, the products as tcgen05.mma chains issued by a
//     tensor-memory warpgroup while eight other warps prepare the next chunk
//     (GDN's pair matrices there on mma.sync, KDA's in FP32); inputs by TMA
//     tensor copies;
//   prefill_tc_kernel (other shapes, other rows): the state in registers as
//     mma.sync accumulator tiles, the chunk's inputs staged by plain loads.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "lq_common.cuh"
#include "lq_prefill.h"
#include "lq_tc.cuh"

namespace lq {

constexpr int kChunk = 16;

// The hardware base-2 exponential and logarithm (MUFU, ~2 ulp like exp2f /
// log2f), results below 2^-126 flushed to zero: the decay factors they form
// multiply keys and states of size <= 1, so a flushed factor changes a value
// by less than 2^-126.
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float lg2_ftz(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

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
                if (KDA) gl = fmaxf(lg2_ftz(a.alpha[(((size_t)tok * a.B + b) * a.H + h) * DK + r]), -150.0f);
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
            if (!KDA) S.g[0][t] = tok < a.T ? fmaxf(lg2_ftz(a.alpha[bh]), -150.0f) : 0.f;
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
            S.glast[KDA ? t : 0] = ex2_ftz(acc);
        }
        __syncthreads();
        if (!KDA && t < DK && t > 0) S.glast[t] = S.glast[0];
        // (2) decayed operands (token-major) and the pair matrices
        for (int e = t; e < C * DK; e += NT) {
            const int r = e % DK, tt = e / DK;
            const float gt = S.g[KDA ? r : 0][tt], gC = S.g[KDA ? r : 0][C - 1];
            const float et = ex2_ftz(gt);
            S.kg[tt][r] = S.kT[r][tt] * et;
            S.qg[tt][r] = S.qT[r][tt] * et;
            S.kh[tt][r] = S.kT[r][tt] * ex2_ftz(gC - gt);
        }
        for (int pr = t; pr < C * C; pr += NT) {
            const int ti = pr / C, ii = pr % C;
            float dkk = 0.f, dqk = 0.f;
            if (ii <= ti) {
                if (KDA) {
#pragma unroll 8
                    for (int r = 0; r < DK; ++r) {
                        const float f = ex2_ftz(S.g[r][ti] - S.g[r][ii]) * S.kT[r][ii];
                        dkk = fmaf(S.kT[r][ti], f, dkk);
                        dqk = fmaf(S.qT[r][ti], f, dqk);
                    }
                } else {
#pragma unroll 8
                    for (int r = 0; r < DK; ++r) {
                        dkk = fmaf(S.kT[r][ti], S.kT[r][ii], dkk);
                        dqk = fmaf(S.qT[r][ti], S.kT[r][ii], dqk);
                    }
                    const float f = ex2_ftz(S.g[0][ti] - S.g[0][ii]);
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


// ---------------------------------------------------------------------------
// d_k = d_v = 128: the chunk step on the fifth-generation tensor cores, in
// chunks of kUChunk = 16 tokens, one CTA per head (one per SM: the state's
// tensor memory) of a tensor-memory warpgroup and an 8-warp preparation
// group.  The chunk's pseudo-values are solved without the state first: with
// A the strictly lower pair matrix above,
//   (I + A) W = diag(b) Kg,   (I + A) Ut = diag(b) V     (rows = tokens)
// by forward substitution (a key or value column per thread), so that
//   U = Ut - W S,   O = Qg S + P U,   S <- diag(Gamma_C) S + Kh^T U
// are products only, all on the tensor cores with the state in tensor memory
// as S^T [d_v lanes x d_k columns] (FP32, the update's accumulator):
//   group 1:  [Oi^T | U'^T] = S^T [Qg; -W]^T        (M = d_v, N = 32, K = d_k;
//             A = S^T's TF32 big and small parts, also in tensor memory; the
//             big part times both parts of B in one N = 64 MMA)
//   group 2:  [S^T | O^T] += U^T [Kh; P]^T           (N = d_k + 16, K = 16
//             tokens; A = U^T from shared memory, U = Ut + U')
// each product in three TF32 passes (big x big + big x small + small x big);
// stacking the two right-hand sides of each group makes it one MMA chain.
// The tensor-memory warpgroup (warps 0-3, a value column per thread) splits
// the state, issues both groups and forms U^T and the outputs; everything that
// does not need the state -- the next chunk's decays, pair matrices,
// substitution and operand splits -- runs meanwhile on the preparation group
// (warps 4-11), the two handing buffers over by mbarriers.  The inputs arrive
// by tensor copies two chunks ahead (two input slots); the buffers a chunk
// reads after its group 1 (Ut, Gamma_C, [Kh; P]) have two slots.  Tensor
// memory: S^T columns 0-127; group 1's three passes as three [Oi^T | U'^T]
// partials at 128, 160, 192 (their sum is the product; group 2 adds U^T P^T
// onto the first); S^T's big and small parts 256-383 and 384-511.
// ---------------------------------------------------------------------------
constexpr int kUChunk = 16;
constexpr int kUPrep = 256;               // the preparation group (warps 4-11)
constexpr int kUThreads = 128 + kUPrep;   // after the tensor-memory warpgroup (warps 0-3)

template <bool KDA>
struct alignas(128) PrefillUIn {   // one chunk's inputs (token rows padded against bank conflicts;
                                   // tensor-copy destinations 128-byte aligned)
    static constexpr int D = 128, C = kUChunk, RP = D + 4;
    alignas(128) float k[C][RP];
    alignas(128) float q[C][RP];
    alignas(128) float g[KDA ? C : 1][KDA ? RP : C];   // decays -> cumulative log2 decay
    alignas(128) float v[C][D];
    float beta[C];
};

template <bool KDA>
struct PrefillUSmem {
    static constexpr int D = 128, C = kUChunk, RP = D + 4;
    // MMA operands, TF32 big [0] and small [1], K-major core matrices: word
    // (row x, k) at (k / 4) rows 4 + (x / 8) 32 + (x % 8) 4 + k % 4
    alignas(128) uint32_t qw[4 * C * D];            // B of group 1: [Qg; -W] big, then small: [N = 4C][K = D key rows]
    alignas(128) uint32_t khp[2][2][(D + C) * C];   // [slot]: B of group 2: [Kh; P] [N = D + C][K = C tokens]
    alignas(128) uint32_t ut[2][D * C];             // A of group 2: U^T [M = D value columns][K = C tokens]
    alignas(16) float ud[2][C][D];           // [slot]: Ut
    alignas(16) float wst[C][RP];            // -W before its split
    alignas(16) float fac[KDA ? 24 : 1][RP]; // KDA: the decay-factored pair operands (below)
    PrefillUIn<KDA> in[2];                   // input slots: chunk c in slot c % 2
    alignas(16) float A[C][C + 4];           // rows read as float4 (the last 4 columns unused)
    alignas(16) float P[2][C][C + 4];        // [chunk % 2]: read by the tensor-memory warpgroup
    float gC[2][D];                          // [slot]: Gamma over the whole chunk, per key row
    float bg[C];                             // GDN: b_t Gamma_t of the chunk being prepared
    uint64_t mbar_in[2];       // input slot filled
    uint64_t mbar_ops;         // a chunk's operands written (preparation group -> tensor-memory warpgroup)
    uint64_t mbar_yo;          // group 1 complete
    uint64_t mbar_up[2];       // group 2 of an even / odd chunk complete
    uint32_t tmem_base;
};

__device__ __forceinline__ int umma_word(int rows, int x, int k) {
    return (k >> 2) * rows * 4 + (x >> 3) * 32 + (x & 7) * 4 + (k & 3);
}

__device__ __forceinline__ void split4(float4 f, uint4 &big, uint4 &small) {
    tf32_split(f.x, big.x, small.x);
    tf32_split(f.y, big.y, small.y);
    tf32_split(f.z, big.z, small.z);
    tf32_split(f.w, big.w, small.w);
}

// Tensor maps of the token-major inputs [T][B][heads][D], one box = 16 token
// rows of one head: k and q (of the q/k head), the KDA decays 132 floats wide
// (the padded shared-memory rows; the 4 floats past D are out of bounds and
// arrive as zeros), v 128 wide.  Rows past T arrive as zeros.
struct alignas(64) PrefillMaps {
    CUtensorMap k, q, v, g;
};

template <bool KDA>
constexpr uint32_t prefill_load_bytes() {
    return (uint32_t)(kUChunk * (PrefillUIn<KDA>::RP * 4 * (KDA ? 3 : 2) + 128 * 4));
}

__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, int x, int y, int z, int w,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5}], [%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
        : "memory");
}

// Named barrier of the preparation group (warps 4-11), and its OR form.
__device__ __forceinline__ void ubar() { asm volatile("bar.sync 1, %0;" ::"n"(kUPrep) : "memory"); }

__device__ __forceinline__ bool ubar_or(bool v) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.s32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\t"
        "selp.s32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((int)v), "n"(kUPrep)
        : "memory");
    return r != 0;
}

// Named barrier of the tensor-memory warpgroup (warps 0-3), and its OR form.
__device__ __forceinline__ void tbar() { asm volatile("bar.sync 2, 128;" ::: "memory"); }

__device__ __forceinline__ bool tbar_or(bool v) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.s32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 2, 128, p;\n\t"
        "selp.s32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((int)v)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <bool KDA>
__global__ void __launch_bounds__(kUThreads, 1) prefill_umma_kernel(const PrefillArgs a,
                                                                      const __grid_constant__ PrefillMaps mp) {
    constexpr int D = 128, C = kUChunk, NT = kUPrep;
    using Sm = PrefillUSmem<KDA>;
    using In = PrefillUIn<KDA>;
    extern __shared__ __align__(128) unsigned char smem_u[];
    Sm &S = *reinterpret_cast<Sm *>(smem_u);
    const int head = blockIdx.x;
    const int b = head / a.H, h = head - b * a.H, gk = (h * a.Hk) / a.H;
    const int lane = threadIdx.x & 31;
    const size_t state_off = (size_t)head * D * D;
    const int nchunks = (a.T + C - 1) / C;
    // group 1 in two MMAs a K-block: S_big [Qg; -W]_big|small (N = 64) into
    // cO .. cO+63 and S_small [Qg; -W]_big (N = 32) into cO+64 .. cO+95: three
    // [Oi | U'] partials at cO, cO+32, cO+64; group 2 accumulates onto the first
    constexpr uint32_t cS = 0, cO = 128, cU = 144, cSb = 256, cSs = 384;
    constexpr uint32_t IDESC_G1W = umma_idesc_tf32(128, 4 * C), IDESC_G1 = umma_idesc_tf32(128, 2 * C);
    constexpr uint32_t IDESC_G2 = umma_idesc_tf32(128, D + C);
    const bool want_o = a.o != nullptr;

    if (threadIdx.x == 0) {
        mbar_init(&S.mbar_in[0], 1);
        mbar_init(&S.mbar_in[1], 1);
        mbar_init(&S.mbar_ops, 1);
        mbar_init(&S.mbar_yo, 1);
        mbar_init(&S.mbar_up[0], 1);
        mbar_init(&S.mbar_up[1], 1);
        fence_mbar_init();
    }
    if (threadIdx.x < 32) {
        tmem_alloc(&S.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    if (threadIdx.x < 128) {
        // The tensor-memory warpgroup: thread t = value column t = tensor-memory
        // lane t.  Per chunk: wait for the preparation group's operands, the
        // previous chunk's outputs, the state split, group 1, U^T, group 2.
        const int t = threadIdx.x, col = t;
        const uint32_t trow = tmem + ((uint32_t)(t & ~31) << 16);   // this warp's 32 lanes
        // S^T lane col = column col of S0
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t w[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
                w[j] = __float_as_uint(a.S0 ? a.S0[state_off + (size_t)(c0 + j) * D + col] : 0.0f);
            tmem_st_32x32b_x32(trow + cS + c0, w);
        }
        tmem_st_wait();
        // the outputs of chunk c from O^T in tensor memory
        auto store_outputs = [&](int c) {
            uint32_t w0[16], w1[16], w2[16];
            tmem_ld_32x32b<16>(trow + cO, w0);
            tmem_ld_32x32b<16>(trow + cO + 32, w1);
            tmem_ld_32x32b<16>(trow + cO + 64, w2);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < C; ++j) {
                const int tok = c * C + j;
                const float o = __uint_as_float(w0[j]) + (__uint_as_float(w1[j]) + __uint_as_float(w2[j]));
                if (tok < a.T) a.o[(((size_t)tok * a.B + b) * a.H + h) * D + col] = o;
            }
        };
        bool ok = true;
#pragma unroll 1
        for (int ch = 0; ch < nchunks; ++ch) {
            const int sl = ch & 1;
            {   // chunk ch's operands, and the previous chunk's group 2
                bool okw = mbar_wait_bounded(&S.mbar_ops, (uint32_t)(ch & 1), a.status);
                if (ch > 0 && okw)
                    okw = mbar_wait_bounded(&S.mbar_up[(ch - 1) & 1], (uint32_t)(((ch - 1) >> 1) & 1), a.status);
                if (tbar_or(!okw)) {
                    ok = false;
                    break;
                }
            }
            tc_fence_after();
            if (ch > 0 && want_o) store_outputs(ch - 1);
            // S^T split into group 1's A operand and scaled by this chunk's Gamma
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t w[32], wb[32], ws[32];
                tmem_ld_32x32b<32>(trow + cS + (uint32_t)c0, w);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float x = __uint_as_float(w[j]);
                    tf32_split(x, wb[j], ws[j]);
                    w[j] = __float_as_uint(x * S.gC[sl][KDA ? c0 + j : 0]);
                }
                tmem_st_32x32b_x32(trow + cSb + (uint32_t)c0, wb);
                tmem_st_32x32b_x32(trow + cSs + (uint32_t)c0, ws);
                tmem_st_32x32b_x32(trow + cS + (uint32_t)c0, w);
            }
            tmem_st_wait();
            tc_fence_before();
            tbar();
            if (t == 0) {   // group 1: 16 K-blocks of 8 key rows, two MMAs each
                tc_fence_after();
                // [4C rows][D]: a K-block is 8 x 4C x 4 bytes (2 KB); its first 2C
                // rows are the big parts
                const uint64_t dq = umma_smem_desc(&S.qw[0], 4 * C * 16, 128);
#pragma unroll 1
                for (int kb = 0; kb < D / 8; ++kb) {
                    const uint32_t ab = tmem + cSb + 8u * kb, as = tmem + cSs + 8u * kb;
                    const uint64_t off = (uint64_t)(kb * 8 * 4 * C * 4) >> 4;
                    const uint32_t acc = kb > 0 ? 1u : 0u;
                    umma_tf32_ta(tmem + cO, ab, dq + off, IDESC_G1W, acc);
                    umma_tf32_ta(tmem + cO + 64, as, dq + off, IDESC_G1, acc);
                }
                umma_commit(&S.mbar_yo);
            }
            __syncwarp();
            if (t >= 32) {   // while lane 0 issues: [Kh; P] of this chunk from its input slot
                In &I = S.in[sl];
                const int u = t - 32;   // 96 threads
                for (int e = u; e < D * C / 4; e += 96) {   // Kh: key row e % D, tokens 4 (e / D) ..
                    const int r = e % D, t4 = 4 * (e / D);
                    const float glast = KDA ? I.g[C - 1][r] : I.g[0][C - 1];
                    float kh[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float gt = KDA ? I.g[t4 + j][r] : I.g[0][t4 + j];
                        kh[j] = I.k[t4 + j][r] * ex2_ftz(glast - gt);
                    }
                    uint4 bb, bs;
                    split4(make_float4(kh[0], kh[1], kh[2], kh[3]), bb, bs);
                    const int wd = umma_word(D + C, r, t4);
                    *reinterpret_cast<uint4 *>(&S.khp[sl][0][wd]) = bb;
                    *reinterpret_cast<uint4 *>(&S.khp[sl][1][wd]) = bs;
                }
                if (u < C * C / 4) {   // P: token u % C, columns 4 (u / C) ..
                    const int tt = u % C, i4 = 4 * (u / C);
                    uint4 bb, bs;
                    split4(*reinterpret_cast<const float4 *>(&S.P[sl][tt][i4]), bb, bs);
                    const int wd = umma_word(D + C, D + tt, i4);
                    *reinterpret_cast<uint4 *>(&S.khp[sl][0][wd]) = bb;
                    *reinterpret_cast<uint4 *>(&S.khp[sl][1][wd]) = bs;
                }
                fence_async_smem();
            }
            tbar();
            if (t == 0 && ch + 2 < nchunks) {   // the slot's next contents: chunk ch + 2
                In &I = S.in[sl];
                const int t0 = (ch + 2) * C;
                uint64_t *bar = &S.mbar_in[sl];
                mbar_arrive_expect_tx(bar, prefill_load_bytes<KDA>());
                tma_load_4d(&I.k[0][0], &mp.k, 0, gk, b, t0, bar);
                tma_load_4d(&I.q[0][0], &mp.q, 0, gk, b, t0, bar);
                tma_load_4d(&I.v[0][0], &mp.v, 0, h, b, t0, bar);
                if (KDA) tma_load_4d(&I.g[0][0], &mp.g, 0, h, b, t0, bar);
            }
            {
                const bool okw = mbar_wait_bounded(&S.mbar_yo, (uint32_t)(ch & 1), a.status);
                if (tbar_or(!okw)) {
                    ok = false;
                    break;
                }
            }
            tc_fence_after();
            {   // U = Ut + U' (the three passes' sum) into group 2's A operand
                uint32_t w0[16], w1[16], w2[16];
                tmem_ld_32x32b<16>(trow + cU, w0);
                tmem_ld_32x32b<16>(trow + cU + 32, w1);
                tmem_ld_32x32b<16>(trow + cU + 64, w2);
                tmem_ld_wait();
                float w[16];
#pragma unroll
                for (int j = 0; j < C; ++j)
                    w[j] = __uint_as_float(w0[j]) + (__uint_as_float(w1[j]) + __uint_as_float(w2[j]));
#pragma unroll
                for (int j4 = 0; j4 < C / 4; ++j4) {
                    const int tt = 4 * j4;
                    float4 u;
                    u.x = S.ud[sl][tt][col] + w[tt];
                    u.y = S.ud[sl][tt + 1][col] + w[tt + 1];
                    u.z = S.ud[sl][tt + 2][col] + w[tt + 2];
                    u.w = S.ud[sl][tt + 3][col] + w[tt + 3];
                    uint4 bb, bs;
                    split4(u, bb, bs);
                    const int wd = umma_word(D, col, tt);
                    *reinterpret_cast<uint4 *>(&S.ut[0][wd]) = bb;
                    *reinterpret_cast<uint4 *>(&S.ut[1][wd]) = bs;
                }
            }
            fence_async_smem();
            tc_fence_before();
            tbar();
            if (t == 0) {   // group 2: 2 K-blocks of 8 tokens, three passes each
                tc_fence_after();
                const uint64_t ub = umma_smem_desc(&S.ut[0][0], D * 16, 128);
                const uint64_t us = umma_smem_desc(&S.ut[1][0], D * 16, 128);
                const uint64_t hb = umma_smem_desc(&S.khp[sl][0][0], (D + C) * 16, 128);
                const uint64_t hs = umma_smem_desc(&S.khp[sl][1][0], (D + C) * 16, 128);
#pragma unroll
                for (int kb = 0; kb < C / 8; ++kb) {
                    const uint64_t ou = (uint64_t)(kb * 8 * D * 4) >> 4;
                    const uint64_t oh = (uint64_t)(kb * 8 * (D + C) * 4) >> 4;
                    umma_tf32(tmem + cS, ub + ou, hb + oh, IDESC_G2, 1u);
                    umma_tf32(tmem + cS, ub + ou, hs + oh, IDESC_G2, 1u);
                    umma_tf32(tmem + cS, us + ou, hb + oh, IDESC_G2, 1u);
                }
                umma_commit(&S.mbar_up[sl]);
            }
            __syncwarp();
        }
        // the last chunk's group 2, its outputs and the final state
        if (ok && nchunks > 0) {
            const bool okw =
                mbar_wait_bounded(&S.mbar_up[(nchunks - 1) & 1], (uint32_t)(((nchunks - 1) >> 1) & 1), a.status);
            ok = !tbar_or(!okw);
            tc_fence_after();
            if (ok && want_o) store_outputs(nchunks - 1);
        }
        if (ok) {
            bool fin = true;
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t w[32];
                tmem_ld_32x32b<32>(trow + cS + (uint32_t)c0, w);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float x = __uint_as_float(w[j]);
                    fin = fin && isfinite(x);
                    a.S_out[state_off + (size_t)(c0 + j) * D + col] = x;
                }
            }
            if (!fin && a.status) atomicOr(a.status, kStatusNonFinite);
        }
    } else {
        // The preparation group (warps 4-11; t, warp: its own thread and warp
        // index): per chunk the decays, pair matrices, substitution and operand
        // splits, into the buffers the tensor-memory warpgroup has finished
        // with, then one arrival on mbar_ops.
        const int t = threadIdx.x - 128, warp = t >> 5;
        // Chunk c's token rows into input slot c % 2: one tensor copy per array
        // (rows past T: zeros), completing on mbar_in[c % 2].  Starts with a
        // barrier (the slot's previous contents have been read).
        auto issue_load = [&](int c) {
            In &I = S.in[c & 1];
            const int t0 = c * C;
            ubar();
            if (t == 0) {
                uint64_t *bar = &S.mbar_in[c & 1];
                mbar_arrive_expect_tx(bar, prefill_load_bytes<KDA>());
                tma_load_4d(&I.k[0][0], &mp.k, 0, gk, b, t0, bar);
                tma_load_4d(&I.q[0][0], &mp.q, 0, gk, b, t0, bar);
                tma_load_4d(&I.v[0][0], &mp.v, 0, h, b, t0, bar);
                if (KDA) tma_load_4d(&I.g[0][0], &mp.g, 0, h, b, t0, bar);
            }
        };

        // b_t (and GDN's decay, as log2) of chunk c's token t, loaded ahead of use
        auto load_scalars = [&](int c, float &bet, float &gl) {
            bet = 0.f;
            gl = 0.f;
            if (t < C && c * C + t < a.T) {
                const size_t bh = ((size_t)(c * C + t) * a.B + b) * a.H + h;
                bet = __ldg(a.beta + bh);
                if (!KDA) gl = __ldg(a.alpha + bh);
            }
        };

        // Chunk c, part 1 (no operand that a group may be reading): decays, pair
        // matrices, and the substitution into -W (wst) and Ut (ud[c % 2]).
        auto prep_solve = [&](int c, float bet, float gl) -> bool {
            In &I = S.in[c & 1];
            const int sl = c & 1;
            const bool okw = mbar_wait_bounded(&S.mbar_in[sl], (uint32_t)((c >> 1) & 1), a.status);
            if (ubar_or(!okw)) return false;
            if (t < C) {
                I.beta[t] = bet;
                if (!KDA) {
                    // log2 decay, floored at -150 (a decay of 0 wipes the
                    // state), 0 past T; then its cumulative sum within the
                    // chunk as a shuffle scan over lanes 0-15, and Gamma_C
                    float l = (c * C + t < a.T) ? fmaxf(lg2_ftz(gl), -150.0f) : 0.f;
#pragma unroll
                    for (int o = 1; o < C; o <<= 1) {
                        const float v = __shfl_up_sync(0x0000ffffu, l, o);
                        if (t >= o) l += v;
                    }
                    I.g[0][t] = l;
                    if (t == C - 1) S.gC[sl][0] = ex2_ftz(l);
                }
            }
            if (KDA) {   // decays -> log2, floored at -150 (a decay of 0 wipes the state); 0 past T
#pragma unroll
                for (int j = 0; j < C * D / NT; ++j) {
                    const int e = t + j * NT;
                    float &x = I.g[e / D][e % D];
                    x = c * C + e / D < a.T ? fmaxf(lg2_ftz(x), -150.0f) : 0.f;
                }
            }
            ubar();
            // KDA: cumulative log2 decay within the chunk per key channel, Gamma_C
            if (KDA) {
                if (t < D) {
                    float acc = 0.f;
#pragma unroll
                    for (int tt = 0; tt < C; ++tt) {
                        acc += I.g[tt][t];
                        I.g[tt][t] = acc;
                    }
                    S.gC[sl][t] = ex2_ftz(acc);
                }
                ubar();
            }
            if (!KDA) {
                // pair matrices, one decay factor per pair: the products
                // [K; Q] K^T (32 x 16, over the D key channels) on the tensor
                // cores, mma.sync m16n8k8 in three TF32 passes (FP32-level
                // accuracy).  Warp w takes the output tile of rows 16 (w / 2 % 2)
                // .. (K for 0, Q for 1) and columns 8 (w % 2) .. over key
                // channels 64 (w / 4) ..; the two halves' partial sums meet in
                // wst (free until the substitution), then every thread
                // finishes one entry.
                float *part = &S.wst[0][0];   // [kind][channel half][16][16]
                {
                    const int mt = (warp >> 1) & 1, nt = warp & 1, kh = warp >> 2;
                    const int gi = lane >> 2, tq = lane & 3;
                    const float(*X)[In::RP] = mt ? I.q : I.k;
                    const float *kr = &I.k[8 * nt + gi][0];
                    float d[4][4] = {};   // four accumulators (k-steps mod 4): shorter MMA chains
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const int k0 = (D / 2) * kh + 8 * ks + tq;
                        uint32_t ab[4], as[4];
                        tf32_split(X[gi][k0], ab[0], as[0]);
                        tf32_split(X[gi + 8][k0], ab[1], as[1]);
                        tf32_split(X[gi][k0 + 4], ab[2], as[2]);
                        tf32_split(X[gi + 8][k0 + 4], ab[3], as[3]);
                        mma3(d[ks & 3], ab, as, kr[k0], kr[k0 + 4]);
                    }
                    float e[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) e[j] = (d[0][j] + d[1][j]) + (d[2][j] + d[3][j]);
                    float *pp = part + (2 * mt + kh) * 256 + 8 * nt + 2 * tq;
                    *reinterpret_cast<float2 *>(pp + gi * 16) = make_float2(e[0], e[1]);
                    *reinterpret_cast<float2 *>(pp + (gi + 8) * 16) = make_float2(e[2], e[3]);
                }
                ubar();
                {   // entry (ti, ii) = (t / 16, t % 16)
                    const int ti = t >> 4, ii = t & 15;
                    const float f = ex2_ftz(fminf(I.g[0][ti] - I.g[0][ii], 0.f));
                    const float dkk = (part[t] + part[256 + t]) * f;
                    const float dqk = (part[512 + t] + part[768 + t]) * f;
                    S.A[ti][ii] = ii < ti ? -I.beta[ti] * dkk : 0.f;   // stored negated (the substitution adds)
                    S.P[sl][ti][ii] = ii <= ti ? dqk : 0.f;
                    if (t < C) S.bg[t] = I.beta[t] * ex2_ftz(I.g[0][t]);   // the substitution's key scale
                }
            } else {
                // KDA: per-channel factors 2^(g_t - g_i).  Across the two
                // 8-token halves (t >= 8 > 7 >= i) they factor through token 7,
                // 2^(g_t - g_7) 2^(g_7 - g_i), both <= 1: rows 0-7 of fac hold
                // k_i 2^(g_7 - g_i), rows 8-15 k_t 2^(g_t - g_7), rows 16-23
                // q_t 2^(g_t - g_7) (t = 8 ..); within a half the factor is
                // formed per pair.
#pragma unroll
                for (int j = 0; j < 24 * D / 4 / NT; ++j) {
                    const int e = t + j * NT, row = e / (D / 4), r = 4 * (e % (D / 4));
                    const float4 g7 = *reinterpret_cast<const float4 *>(&I.g[7][r]);
                    const int tr = row < 16 ? row : row - 8;
                    const float4 gr = *reinterpret_cast<const float4 *>(&I.g[tr][r]);
                    const float4 x = *reinterpret_cast<const float4 *>(row < 16 ? &I.k[tr][r] : &I.q[tr][r]);
                    float4 d = row < 8 ? make_float4(g7.x - gr.x, g7.y - gr.y, g7.z - gr.z, g7.w - gr.w)
                                       : make_float4(gr.x - g7.x, gr.y - g7.y, gr.z - g7.z, gr.w - g7.w);
                    *reinterpret_cast<float4 *>(&S.fac[row][r]) =
                        make_float4(x.x * ex2_ftz(d.x), x.y * ex2_ftz(d.y), x.z * ex2_ftz(d.z), x.w * ex2_ftz(d.w));
                }
                ubar();
                // warps 0-3: the two 8 x 8 diagonal blocks (4 rows x 8 columns
                // a warp); 4-5: rows 8-15 x columns 0-7 from fac; 6-7: rows 0-7
                // x columns 8-15, zero
                int ti, ii;
                float dkk = 0.f, dqk = 0.f;
                if (warp < 4) {
                    const int blk = 8 * (warp >> 1);
                    ti = blk + 4 * (warp & 1) + (lane >> 3);
                    ii = blk + (lane & 7);
                    float2 ak0 = f2(0.f, 0.f), ak1 = ak0, aq0 = ak0, aq1 = ak0;
#pragma unroll 4
                    for (int r4 = 0; r4 < D / 4; ++r4) {
                        const float4 kt = *reinterpret_cast<const float4 *>(&I.k[ti][4 * r4]);
                        const float4 qt = *reinterpret_cast<const float4 *>(&I.q[ti][4 * r4]);
                        float4 ki = *reinterpret_cast<const float4 *>(&I.k[ii][4 * r4]);
                        const float4 gt = *reinterpret_cast<const float4 *>(&I.g[ti][4 * r4]);
                        const float4 gi = *reinterpret_cast<const float4 *>(&I.g[ii][4 * r4]);
                        // at most 1 where used (ii <= ti); clamped past the diagonal
                        ki.x *= ex2_ftz(fminf(gt.x - gi.x, 0.f));
                        ki.y *= ex2_ftz(fminf(gt.y - gi.y, 0.f));
                        ki.z *= ex2_ftz(fminf(gt.z - gi.z, 0.f));
                        ki.w *= ex2_ftz(fminf(gt.w - gi.w, 0.f));
                        ak0 = ffma2(f2(kt.x, kt.y), f2(ki.x, ki.y), ak0);
                        ak1 = ffma2(f2(kt.z, kt.w), f2(ki.z, ki.w), ak1);
                        aq0 = ffma2(f2(qt.x, qt.y), f2(ki.x, ki.y), aq0);
                        aq1 = ffma2(f2(qt.z, qt.w), f2(ki.z, ki.w), aq1);
                    }
                    dkk = (ak0.x + ak0.y) + (ak1.x + ak1.y);
                    dqk = (aq0.x + aq0.y) + (aq1.x + aq1.y);
                } else if (warp < 6) {
                    ti = 8 + 4 * (warp - 4) + (lane >> 3);
                    ii = lane & 7;
                    float2 ak0 = f2(0.f, 0.f), ak1 = ak0, aq0 = ak0, aq1 = ak0;
#pragma unroll 4
                    for (int r4 = 0; r4 < D / 4; ++r4) {
                        const float4 kt = *reinterpret_cast<const float4 *>(&S.fac[ti][4 * r4]);
                        const float4 qt = *reinterpret_cast<const float4 *>(&S.fac[ti + 8][4 * r4]);
                        const float4 ki = *reinterpret_cast<const float4 *>(&S.fac[ii][4 * r4]);
                        ak0 = ffma2(f2(kt.x, kt.y), f2(ki.x, ki.y), ak0);
                        ak1 = ffma2(f2(kt.z, kt.w), f2(ki.z, ki.w), ak1);
                        aq0 = ffma2(f2(qt.x, qt.y), f2(ki.x, ki.y), aq0);
                        aq1 = ffma2(f2(qt.z, qt.w), f2(ki.z, ki.w), aq1);
                    }
                    dkk = (ak0.x + ak0.y) + (ak1.x + ak1.y);
                    dqk = (aq0.x + aq0.y) + (aq1.x + aq1.y);
                } else {
                    ti = 4 * (warp - 6) + (lane >> 3);
                    ii = 8 + (lane & 7);
                }
                S.A[ti][ii] = ii < ti ? -I.beta[ti] * dkk : 0.f;   // stored negated (the substitution adds)
                S.P[sl][ti][ii] = ii <= ti ? dqk : 0.f;
            }
            ubar();
            // forward substitution, one column per thread: threads 0-127 the key
            // column t of W (right side b Gamma k), 128-255 the value column of Ut
            {
                const int cc = t & (D - 1);
                float x[C];
#pragma unroll
                for (int tt = 0; tt < C; ++tt) {   // the right-hand sides first (independent loads)
                    if (t < D) x[tt] = KDA ? I.beta[tt] * (I.k[tt][cc] * ex2_ftz(I.g[tt][cc])) : S.bg[tt] * I.k[tt][cc];
                    else x[tt] = I.beta[tt] * I.v[tt][cc];
                }
                // x_t += sum_{i<t} (-A_ti) x_i, two terms per packed FMA (the
                // entries past the diagonal are zero)
#pragma unroll
                for (int tt = 1; tt < C; ++tt) {
                    float2 acc = f2(x[tt], 0.f);
#pragma unroll
                    for (int j = 0; 4 * j < tt; ++j) {
                        const float4 a4 = *reinterpret_cast<const float4 *>(&S.A[tt][4 * j]);
                        acc = ffma2(f2(a4.x, a4.y), f2(x[4 * j], 4 * j + 1 < tt ? x[4 * j + 1] : 0.f), acc);
                        if (4 * j + 2 < tt)
                            acc = ffma2(f2(a4.z, a4.w), f2(x[4 * j + 2], 4 * j + 3 < tt ? x[4 * j + 3] : 0.f), acc);
                    }
                    x[tt] = acc.x + acc.y;
                }
                if (t < D) {
#pragma unroll
                    for (int tt = 0; tt < C; ++tt) S.wst[tt][cc] = -x[tt];
                } else {
#pragma unroll
                    for (int tt = 0; tt < C; ++tt) S.ud[sl][tt][cc] = x[tt];
                }
            }
            return true;
        };

        // Chunk c, part 2: the split of [Qg; -W] (single; the caller guarantees
        // that group 1 of the previous chunk is complete).  [Kh; P] and the
        // reload of the input slot follow on the tensor-memory warpgroup.
        auto prep_operands = [&](int c) {
            In &I = S.in[c & 1];
            const int sl = c & 1;
            ubar();
            for (int e = t; e < C * D / 4; e += NT) {   // Qg, -W: token e % C, key rows 4 (e / C) ..
                const int tt = e % C, r = 4 * (e / C);
                // rows: Qg big tt, -W big C + tt, Qg small 2C + tt, -W small 3C + tt
                const int wq = umma_word(4 * C, tt, r), ww = umma_word(4 * C, C + tt, r);
                const int sq = umma_word(4 * C, 2 * C + tt, r), sw = umma_word(4 * C, 3 * C + tt, r);
                uint4 bb, bs;
                split4(*reinterpret_cast<const float4 *>(&S.wst[tt][r]), bb, bs);
                *reinterpret_cast<uint4 *>(&S.qw[ww]) = bb;
                *reinterpret_cast<uint4 *>(&S.qw[sw]) = bs;
                float4 qv = *reinterpret_cast<const float4 *>(&I.q[tt][r]);
                float4 ev;
                if (KDA) {
                    const float4 gv = *reinterpret_cast<const float4 *>(&I.g[tt][r]);
                    ev = make_float4(ex2_ftz(gv.x), ex2_ftz(gv.y), ex2_ftz(gv.z), ex2_ftz(gv.w));
                } else {
                    const float ee = ex2_ftz(I.g[0][tt]);
                    ev = make_float4(ee, ee, ee, ee);
                }
                qv = make_float4(qv.x * ev.x, qv.y * ev.y, qv.z * ev.z, qv.w * ev.w);
                split4(qv, bb, bs);
                *reinterpret_cast<uint4 *>(&S.qw[wq]) = bb;
                *reinterpret_cast<uint4 *>(&S.qw[sq]) = bs;
            }
            fence_async_smem();
        };

        bool ok = true;
        float bet = 0.f, gl = 0.f, bet_n = 0.f, gl_n = 0.f;
        if (nchunks > 0) {
            load_scalars(0, bet, gl);
            issue_load(0);
            if (nchunks > 1) issue_load(1);
        }
#pragma unroll 1
        for (int c = 0; ok && c < nchunks; ++c) {
            if (c + 1 < nchunks) load_scalars(c + 1, bet_n, gl_n);
            // ud, gC and P of c % 2 were last read by chunk c - 2
            if (c >= 2) {
                const bool okw = mbar_wait_bounded(&S.mbar_up[c & 1], (uint32_t)(((c - 2) >> 1) & 1), a.status);
                if (ubar_or(!okw)) {
                    ok = false;
                    break;
                }
            }
            if (!prep_solve(c, bet, gl)) {
                ok = false;
                break;
            }
            // [Qg; -W] was last read by chunk c - 1's group 1
            if (c >= 1) {
                const bool okw = mbar_wait_bounded(&S.mbar_yo, (uint32_t)((c - 1) & 1), a.status);
                if (ubar_or(!okw)) {
                    ok = false;
                    break;
                }
            }
            prep_operands(c);
            ubar();
            if (t == 0) mbar_arrive(&S.mbar_ops);
            bet = bet_n;
            gl = gl_n;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int DK, int DV>
size_t prefill_smem_bytes_t(bool kda) {
    if (DK == 128 && DV == 128) return kda ? sizeof(PrefillUSmem<true>) : sizeof(PrefillUSmem<false>);
    return kda ? sizeof(PrefillTcSmem<DK, DV, true>) : sizeof(PrefillTcSmem<DK, DV, false>);
}

// cuTensorMapEncodeTiled from the driver, looked up once.
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        tried = true;
    }
    return fn;
}

// Token rows [T][B][NH][D] (FP32) as a 4-D map with boxes of `rows` tokens x
// `width` floats of one (b, head).
static bool encode_rows(CUtensorMap *m, const float *base, int T, int B, int NH, int D, int width, int rows) {
    const auto enc = tensor_map_encoder();
    if (!enc || !base) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)NH, (cuuint64_t)B, (cuuint64_t)(T > 0 ? T : 1)};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 4, (cuuint64_t)NH * D * 4, (cuuint64_t)B * NH * D * 4};
    const cuuint32_t box[4] = {(cuuint32_t)width, 1, 1, (cuuint32_t)rows};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK, int DV>
static cudaError_t prefill_dispatch(const PrefillArgs &a, int heads, bool kda, cudaStream_t s) {
    // the tensor-memory kernel reads token rows by tensor copies: 16-byte
    // aligned k, q, v (and KDA's decays) and encodable maps; otherwise the
    // register-state kernel
    const uintptr_t al = reinterpret_cast<uintptr_t>(a.q) | reinterpret_cast<uintptr_t>(a.k) |
                         reinterpret_cast<uintptr_t>(a.v) | (kda ? reinterpret_cast<uintptr_t>(a.alpha) : 0);
    if constexpr (DK == 128 && DV == 128) {
        PrefillMaps mp{};
        bool maps = al % 16 == 0 && a.T > 0;
        if (maps) {
            constexpr int RP = PrefillUIn<true>::RP;
            maps = encode_rows(&mp.k, a.k, a.T, a.B, a.Hk, DK, RP, kUChunk) &&
                   encode_rows(&mp.q, a.q, a.T, a.B, a.Hk, DK, RP, kUChunk) &&
                   encode_rows(&mp.v, a.v, a.T, a.B, a.H, DV, DV, kUChunk) &&
                   (!kda || encode_rows(&mp.g, a.alpha, a.T, a.B, a.H, DK, RP, kUChunk));
        }
        if (!maps && a.T > 0) {
            const size_t sm = kda ? sizeof(PrefillTcSmem<DK, DV, true>) : sizeof(PrefillTcSmem<DK, DV, false>);
            auto kern = kda ? prefill_tc_kernel<DK, DV, true> : prefill_tc_kernel<DK, DV, false>;
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
            if (e != cudaSuccess) return e;
            kern<<<heads, 2 * DV, sm, s>>>(a);
            return cudaGetLastError();
        }
        const size_t sm = kda ? sizeof(PrefillUSmem<true>) : sizeof(PrefillUSmem<false>);
        auto kern = kda ? prefill_umma_kernel<true> : prefill_umma_kernel<false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        kern<<<heads, kUThreads, sm, s>>>(a, mp);
        return cudaGetLastError();
    } else {
        const size_t sm = prefill_smem_bytes_t<DK, DV>(kda);
        auto kern = kda ? prefill_tc_kernel<DK, DV, true> : prefill_tc_kernel<DK, DV, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        kern<<<heads, 2 * DV, sm, s>>>(a);
        return cudaGetLastError();
    }
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
