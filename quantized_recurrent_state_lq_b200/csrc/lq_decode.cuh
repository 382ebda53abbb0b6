// lq_decode.cuh -- decode-step kernels (templates; instantiated per code width
// by lq_decode_b8.cu, lq_decode_b6.cu and lq_decode_b4.cu).
//
// Windowed INT8 (or bit-packed 6 / 4-bit) decode (LeapQuant project page,
// window paragraph): within a window the quantized state is read, never
// written.  With Gamma_t the product of
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
// Buffering steps run decode_buffer_kernel (one CTA per head, seven per SM: the
// codes staged by one bulk copy and multiplied on the int8 tensor cores, the
// buffered entries streamed from global memory);
// the step that ends a window runs decode_flush_kernel (one CTA per head,
// state rebuilt in registers and requantized).
#pragma once

#include "lq_codec.cuh"
#include "lq_tc.cuh"
#include "lq_kernels.h"

namespace lq {

// Tokens batch entry b holds in its current window, and whether its window
// ends at this step (always false without window phases: the caller decides).
struct EntryPos {
    int n;
    bool ends;
};
__device__ __forceinline__ EntryPos entry_pos(const DecodeArgs &a, int b) {
    if (!a.phase) return {a.n, false};
    int p = a.nmod + __ldg(a.phase + b);
    if (p >= a.L.W) p -= a.L.W;
    return {p < a.n ? p : a.n, p == a.L.W - 1};
}


// ---------------------------------------------------------------------------
// Buffering step: one CTA of 4 warps per head, small enough (<= 72 registers,
// ~27 KB of shared memory at d = 128) for seven CTAs per SM, so that the
// phases of seven heads interleave on each SM:
//   * thread 0 stages the record head [m | s | BF16 rows | codes] (17 KB at
//     d = 128 with INT8 codes, 13 / 9 KB with 6 / 4-bit) with one
//     cp.async.bulk; every warp loads the first pair of its
//     buffered entries into registers; the small step vectors are read.
//   (a) x = Gamma_t (k, q), a = m * x; the per-vector maxima of |a|.   barrier
//   (b) a_k, a_q as exact signed base-256 digits (4 each): the B operand.  barrier
//   (c) codes: int8 tensor-core MMA (m16n8k32) of the value-column-major code
//       tile with the digits, one warp per 16 value columns -- while the
//       entry pairs are still arriving (packed codes are unpacked to signed
//       bytes c * 2^(8-b) in registers first).  (With BF16 rows: SIMT, a
//       warp per row.)
//   (d) entries: pairs of entries per warp, the next pair prefetched, dot
//       products reduced by a transpose-reduce butterfly.
//   (e) per-warp partial column sums combined; output, append.           barrier
// ---------------------------------------------------------------------------
// Warps of a buffering CTA: 4 warps and ~27 KB of shared memory let 7 heads
// be in flight on an SM (the per-head critical path -- step inputs, the
// staged codes, the tensor-core GEMV, the entry stream -- is latency-bound).
constexpr int kBufWarps = 4;
constexpr int kBufThreads = kBufWarps * 32;

template <int DK, int DV>
struct BufSmem {
    float2 x2[DK];                      // (G k, G q) by key row (G: the guarded decay)
    float2 a2[DK];                      // m * x2 by INT8 slot (BF16-row layout)
    float2 red[kBufWarps][DV];             // per-warp partial column sums (BF16 rows + entries)
    float2 rc[DV];                      // codes part of (y_k, y_q)
    int8_t dig[8][DK + 16];             // base-256 digits of a_k (rows 0-3) and a_q (rows 4-7)
    int rows[DK];                       // DAMP: key row of INT8 slot j, then of BF16 row p
    float v[DV];
    float qk[DK];                       // q (BF16 buffer: k . q is formed at the end)
    int rebase;                         // decay guard: some key channel rescales its entries this step
    float amax[kBufWarps][2];
    float kqw[kBufWarps];
    uint64_t mbar;
};

template <int DK, int DV>
__host__ __device__ constexpr size_t buf_fixed_bytes() {
    return (sizeof(BufSmem<DK, DV>) + 127) / 128 * 128;
}

inline size_t buffer_smem_bytes(int dk, int dv, const Layout &L) {
    size_t fixed = 0;
    if (dk == 64 && dv == 64) fixed = buf_fixed_bytes<64, 64>();
    if (dk == 64 && dv == 128) fixed = buf_fixed_bytes<64, 128>();
    if (dk == 128 && dv == 64) fixed = buf_fixed_bytes<128, 64>();
    if (dk == 128 && dv == 128) fixed = buf_fixed_bytes<128, 128>();
    return fixed + (size_t)align_up(L.off_ent, 128);
}

// Sum V = 2 NE values (v[2e] = dot_k of entry e, v[2e+1] = dot_q) over the
// warp: a transpose-reduce butterfly leaves each value's total in one lane
// group (log2(V) halving steps, then plain steps), then every lane fetches all
// V totals -- about V + 5 shuffles instead of 5 V.
template <int NE>
__device__ __forceinline__ void warp_reduce_dots(float (&v)[2 * NE]) {
    constexpr int V = 2 * NE;
    const int lane = threadIdx.x & 31;
    float cur[V];
#pragma unroll
    for (int i = 0; i < V; ++i) cur[i] = v[i];
    int n = V;
    int mask = 16;
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        if (n > 1) {
            const bool upper = (lane & mask) != 0;
            const int h = n / 2;
#pragma unroll
            for (int i = 0; i < V / 2; ++i) {
                if (i < h) {
                    const float send = upper ? cur[i] : cur[i + h];
                    const float keep = upper ? cur[i + h] : cur[i];
                    cur[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
                }
            }
            n = h;
        } else {
            cur[0] += __shfl_xor_sync(0xffffffffu, cur[0], mask);
        }
        mask >>= 1;
    }
    // value i ended in the lanes whose top log2(V) bits (from bit 4 down) spell i
#pragma unroll
    for (int i = 0; i < V; ++i) {
        int src = 0, bit = 16;
#pragma unroll
        for (int k = V / 2; k >= 1; k >>= 1) {
            if (i & k) src |= bit;
            bit >>= 1;
        }
        v[i] = __shfl_sync(0xffffffffu, cur[0], src);
    }
}

// GDN's BF16 buffered tokens at d = 128 stream four tokens per warp step (one
// 16-byte load per lane covers a whole entry) in the registers of six CTAs per
// SM.  (KDA's per-channel decay state leaves too few registers at that
// occupancy: there the variant spills and runs 5% slower than the pairs.)
template <int DK, int DV, bool KDA, bool TB>
constexpr bool buf_quads() { return TB && !KDA && DK == 128 && DV == 128; }

template <int DK, int DV, bool KDA, bool DAMP, bool TB, int BITS>
__global__ void __launch_bounds__(kBufThreads, buf_quads<DK, DV, KDA, TB>() ? 6 : 7)
    decode_buffer_kernel(const DecodeArgs a) {
    static_assert(BITS == 8 || !DAMP, "packed codes are built without BF16 rows");
    extern __shared__ __align__(128) unsigned char smem[];
    BufSmem<DK, DV> &S = *reinterpret_cast<BufSmem<DK, DV> *>(smem);
    unsigned char *stage = smem + buf_fixed_bytes<DK, DV>();
    const Layout &L = a.L;
    const int head = blockIdx.x;
    const int b = head / a.H, h = head - b * a.H, g = (h * a.Hk) / a.H;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int P = DAMP ? L.P : 0;
    const int NI = DK - P;
    const EntryPos pos = entry_pos(a, b);
    if (pos.ends) return;   // staggered windows: this entry's flush launch takes the step
    const int n = pos.n;
    const int E = L.r + n;
    const size_t hv = (size_t)b * a.H + h;
    unsigned char *rec = a.rec + (size_t)head * L.rec_bytes;
    const float *ent_g = reinterpret_cast<const float *>(rec + L.off_ent);
    float *rec_ent = reinterpret_cast<float *>(rec + L.off_ent);
    uint16_t *rec_tok16 = reinterpret_cast<uint16_t *>(rec + L.off_tok);   // BF16 tokens
    float *rec_gam = reinterpret_cast<float *>(rec + L.off_gam);   // G
    float *rec_sig = rec_gam + (KDA ? DK : 1);                       // sigma
    constexpr bool tb = TB;   // buffered tokens in BF16
    constexpr int XPL = DK / 32;                 // key elements per lane in a dot product
    constexpr int EF = DK + DV;                  // elements per entry

    if (t == 0) {
        mbar_init(&S.mbar, 1);
        fence_mbar_init();
        S.rebase = 0;
    }
    // Decay guard scratch in shared arrays this variant leaves unused: this
    // step's factor rho per key row (DAMP: the q row array, never used with
    // DAMP's BF16 rows; else the DAMP-only activation array) and, for DAMP,
    // sigma per key row (in the digit array, which only the tensor-core GEMV
    // of the other variants uses).
    float *rho_s = DAMP ? S.qk : reinterpret_cast<float *>(S.a2);
    float *sig_s = reinterpret_cast<float *>(&S.dig[0][0]);
    __syncthreads();
    // Programmatic dependent launch: the next step's grid may start once every
    // CTA of this one has begun, and this grid may have started while the
    // previous launch on the stream finishes.  Within a window the buffering
    // steps never write the record prefix (m, s, BF16 rows, codes), so after
    // one (n > 0) the prefix is staged before waiting for the previous grid;
    // everything else -- the entries and Gamma the previous step wrote, the
    // step's inputs -- is read after the wait.
    asm volatile("griddepcontrol.launch_dependents;");
    if (t == 0 && n > 0) {
        mbar_arrive_expect_tx(&S.mbar, (uint32_t)L.off_ent);
        bulk_g2s(stage, rec, (uint32_t)L.off_ent, &S.mbar);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (t == 0 && n == 0) {
        mbar_arrive_expect_tx(&S.mbar, (uint32_t)L.off_ent);
        bulk_g2s(stage, rec, (uint32_t)L.off_ent, &S.mbar);
    }

    // Entry pairs of this warp: entries 2 warp + 16 j + {0, 1}.
    float4 kb[2], ub[2];
    float2 kb2[2];
    // (FP32 entries -- the compensators, and FP32 tokens -- form one array;
    // BF16 tokens are widened on load)
    auto load_fp32 = [&](int p, int e) {
        const float *kt = ent_g + (size_t)e * EF;
        if (XPL == 4) kb[p] = __ldcs(reinterpret_cast<const float4 *>(kt) + lane);
        else kb2[p] = __ldcs(reinterpret_cast<const float2 *>(kt) + lane);
        if (lane < DV / 4) ub[p] = __ldcs(reinterpret_cast<const float4 *>(kt + DK) + lane);
    };
    auto load_bf16 = [&](int p, int e) {
        const uint16_t *kt = rec_tok16 + (size_t)(e - L.r) * EF;
        if (XPL == 4) kb[p] = bf16x4_to_f4(__ldcs(reinterpret_cast<const uint2 *>(kt) + lane));
        else kb2[p] = bf16x2_to_f2(__ldcs(reinterpret_cast<const unsigned int *>(kt) + lane));
        if (lane < DV / 4) ub[p] = bf16x4_to_f4(__ldcs(reinterpret_cast<const uint2 *>(kt + DK) + lane));
    };
    // (with BF16 tokens the type is decided per pair: a pair of tokens loads
    // without branches between its loads)
    auto load_pair = [&](int e0) {
        if (!tb || e0 + 1 < L.r) {
#pragma unroll
            for (int p = 0; p < 2; ++p)
                if (e0 + p < E) load_fp32(p, e0 + p);
        } else if (e0 >= L.r) {
#pragma unroll
            for (int p = 0; p < 2; ++p)
                if (e0 + p < E) load_bf16(p, e0 + p);
        } else {
            if (e0 < E) load_fp32(0, e0);
            if (e0 + 1 < E) load_bf16(1, e0 + 1);
        }
    };
    constexpr bool Q4 = buf_quads<DK, DV, KDA, TB>();
    // BF16 tokens in quads (Q4): token j's [k | u] is 256 bf16 = 512 bytes; lane
    // l's 16-byte piece holds k channels 8 l .. 8 l + 7 (lanes 0-15) or u
    // columns 8 (l - 16) .. (lanes 16-31).  The compensators (FP32) keep the pairs.
    uint4 tkq[4];
    auto load_quad = [&](int j0) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (j0 + i < n) tkq[i] = __ldcs(reinterpret_cast<const uint4 *>(rec_tok16 + (size_t)(j0 + i) * EF) + lane);
    };
    if constexpr (Q4) {
#pragma unroll
        for (int p = 0; p < 2; ++p)
            if (2 * warp + p < L.r) load_fp32(p, 2 * warp + p);
        load_quad(4 * warp);
    } else {
        load_pair(2 * warp);
    }

    // (a) step inputs, the guarded decay (G_t, sigma_t, the entries' rescaling
    // rho), x = G_t (k, q), a = m * sigma_t * x.
    float kqp = 0.f, gt = 1.f, kk = 0.f, ak_t = 0.f, aq_t = 0.f, sg = 1.f, rho = 1.f;
    if (t < DK) {
        const size_t qk = ((size_t)b * a.Hk + g) * DK;
        kk = a.k[qk + t];
        const float qq = a.q[qk + t];
        const float gp = n > 0 ? (KDA ? rec_gam[t] : rec_gam[0]) : 1.0f;
        const float sp = n > 0 ? (KDA ? rec_sig[t] : rec_sig[0]) : 1.0f;
        gt = gate_chain(KDA ? a.alpha[hv * DK + t] : a.alpha[hv], gp, rho);
        sg = sp * rho;
        const float2 x = make_float2(gt * kk, gt * qq);
        S.x2[t] = x;
        rho_s[t] = rho;
        if (rho != 1.f) S.rebase = 1;
        // k . q for the output (BF16 buffer: Gamma bf16(k / Gamma) . q, formed
        // at the end, next to the reduction it feeds)
        kqp = tb ? 0.f : kk * qq;
        if (tb) S.qk[t] = qq;
        if (!DAMP) {
            const float mi = reinterpret_cast<const float *>(rec + L.off_m)[t];
            ak_t = mi * (sg * x.x);
            aq_t = mi * (sg * x.y);
        } else {
            S.rows[t] = a.slot_rows[(size_t)h * DK + t];
            sig_s[t] = sg;
        }
    }
    if (t < DV) S.v[t] = a.v[hv * DV + t];
    const float beta = a.beta[hv];
    kqp = warp_sum(kqp);
    if (!DAMP) {
        float mk = fabsf(ak_t), mq = fabsf(aq_t);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, o));
            mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o));
        }
        if (lane == 0) {
            S.amax[warp][0] = mk;
            S.amax[warp][1] = mq;
        }
    }
    if (lane == 0) S.kqw[warp] = kqp;
    __syncthreads();
    // a rescaling of the buffered keys this step (rare: the decay passed 2^-64)
    const bool rebase = S.rebase != 0;
    float kq = 0.f;
#pragma unroll
    for (int w = 0; w < kBufWarps; ++w) kq += S.kqw[w];

    // (b) the tensor-core operand: a_k, a_q as exact signed base-256 digits of
    // one fixed-point integer each, X = a * 2^(30 - e) with |a| < 2^e.
    int ek_ = 0, eq_ = 0;
    if (!DAMP) {
        float mk = 0.f, mq = 0.f;
#pragma unroll
        for (int w = 0; w < kBufWarps; ++w) {
            mk = fmaxf(mk, S.amax[w][0]);
            mq = fmaxf(mq, S.amax[w][1]);
        }
        frexpf(mk, &ek_);
        frexpf(mq, &eq_);
        ek_ = max(ek_, -96);
        eq_ = max(eq_, -96);
        if (t < DK) {
            const int xs[2] = {(int)rintf(ak_t * ldexpf(1.0f, 30 - ek_)), (int)rintf(aq_t * ldexpf(1.0f, 30 - eq_))};
            const int kpos = BITS == 8 ? t : lowbit_kslot(t);   // contraction slot of key row t
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                int X = xs[v];
#pragma unroll
                for (int dgt = 0; dgt < 3; ++dgt) {
                    const int d = ((X + 128) & 255) - 128;
                    S.dig[4 * v + dgt][kpos] = (int8_t)d;
                    X = (X - d) >> 8;
                }
                S.dig[4 * v + 3][kpos] = (int8_t)X;
            }
        }
    }
    const bool ok = mbar_wait_bounded(&S.mbar, 0, a.status);
    if (DAMP && t < NI) {
        const float *m_s = reinterpret_cast<const float *>(stage + L.off_m);
        const int row = S.rows[t];
        const float2 x = S.x2[row];
        const float ms = m_s[row] * sig_s[row];
        S.a2[t] = make_float2(ms * x.x, ms * x.y);
    }
    if (__syncthreads_or(!ok)) return;
    const float *s_s = reinterpret_cast<const float *>(stage + L.off_s);

    // (c) codes.
    float ek[4] = {0.f, 0.f, 0.f, 0.f}, eq[4] = {0.f, 0.f, 0.f, 0.f};
    float R[Q4 ? 16 : 1];   // BF16 token quads' registers (below)
    if (!DAMP) {
        for (int cb = warp; cb < DV / 16; cb += kBufWarps) {   // a warp per 16 value columns
            const int c0 = 16 * cb;
            const int gq = lane >> 2, tq = lane & 3;
            const unsigned char *codes = stage + L.off_codes;
            const int r = ((lane >> 3) & 1) * 8 + (lane & 7), blk = lane >> 4;
            const int c = c0 + r;   // the value column whose row address this lane supplies
            int d[4] = {0, 0, 0, 0};
            // one k-step: value columns c0 .. c0+15 x 32 contraction slots
            auto mma_step = [&](uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, int ks) {
                const uint32_t b0 = *reinterpret_cast<const uint32_t *>(&S.dig[gq][32 * ks + 4 * tq]);
                const uint32_t b1 = *reinterpret_cast<const uint32_t *>(&S.dig[gq][32 * ks + 16 + 4 * tq]);
                asm volatile(
                    "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                    "{%0,%1,%2,%3};"
                    : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                    : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
            };
            if (BITS == 8) {
#pragma unroll
                for (int ks = 0; ks < DK / 32; ++ks) {
                    const int chunk = 2 * ks + blk;
                    const uint32_t addr = smem_u32(codes + c * DK + ((chunk ^ code_swz(c, DK)) << 4));
                    uint32_t a0, a1, a2, a3;
                    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                                 : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                                 : "r"(addr));
                    mma_step(a0, a1, a2, a3, ks);
                }
            } else {
                // packed codes: a 16-byte nibble chunk is one 32-row k-step;
                // a lane's word holds 8 rows, even ones to a0/a1, odd ones to
                // a2/a3 (the digits sit in the matching slots, lowbit_kslot).
                // 6-bit: the pair plane's chunk kp serves k-steps 2kp, 2kp+1.
                constexpr int NB = DK / 2, PB = DK / 4;
                uint32_t pr[4] = {0u, 0u, 0u, 0u};
                if (BITS == 6) {
                    const unsigned char *pl = codes + DV * NB;
                    if (DK >= 128) {
                        const uint32_t addr = smem_u32(pl + c * PB + ((blk ^ chunk_swz(c, PB)) << 4));
                        asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                                     : "=r"(pr[0]), "=r"(pr[1]), "=r"(pr[2]), "=r"(pr[3])
                                     : "r"(addr));
                    } else {
                        const uint32_t addr = smem_u32(pl + c * PB);
                        asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
                                     : "=r"(pr[0]), "=r"(pr[1])
                                     : "r"(addr));
                    }
                }
#pragma unroll
                for (int kp = 0; kp < DK / 64; ++kp) {
                    const int chunk = 2 * kp + blk;
                    const uint32_t addr = smem_u32(codes + c * NB + ((chunk ^ chunk_swz(c, NB)) << 4));
                    uint32_t x[4];
                    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                                 : "=r"(x[0]), "=r"(x[1]), "=r"(x[2]), "=r"(x[3])
                                 : "r"(addr));
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const uint32_t pa = BITS == 6 ? spread_pairs(pr[2 * kp], hf) : 0u;
                        const uint32_t pb = BITS == 6 ? spread_pairs(pr[2 * kp + 1], hf) : 0u;
                        uint32_t l0, h0, l1, h1;
                        unpack_group<(BITS < 8 ? BITS : 4)>(x[2 * hf], pa, l0, h0);
                        unpack_group<(BITS < 8 ? BITS : 4)>(x[2 * hf + 1], pb, l1, h1);
                        mma_step(l0, l1, h0, h1, 2 * kp + hf);
                    }
                }
            }
            // lane (gq, tq) holds digit columns 2tq, 2tq+1 of value columns c0+gq, c0+gq+8
            const float w0 = (tq & 1) ? 65536.f : 1.f, w1 = (tq & 1) ? 16777216.f : 256.f;
            float p0 = fmaf((float)d[1], w1, (float)d[0] * w0);
            float p1 = fmaf((float)d[3], w1, (float)d[2] * w0);
            p0 += __shfl_xor_sync(0xffffffffu, p0, 1);
            p1 += __shfl_xor_sync(0xffffffffu, p1, 1);
            if ((tq & 1) == 0) {
                // (packed codes enter the MMA as c * 2^(8 - BITS))
                const float inv = ldexpf(1.0f, (tq == 0 ? ek_ : eq_) - 30 - (8 - BITS));
                float *rc = reinterpret_cast<float *>(S.rc);
                rc[2 * (c0 + gq) + (tq >> 1)] = s_s[c0 + gq] * (p0 * inv);
                rc[2 * (c0 + gq + 8) + (tq >> 1)] = s_s[c0 + gq + 8] * (p1 * inv);
            }
        }
    } else {
        constexpr int LPR = DV / 4, RPP = 32 / LPR;
        const int cq = lane % LPR, rsub = lane / LPR;
        const unsigned char *codes = stage + L.off_codes;
        float ak[4] = {0.f, 0.f, 0.f, 0.f}, aq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int j = warp * RPP + rsub; j < NI; j += kBufWarps * RPP) {
            const uint32_t w = *reinterpret_cast<const uint32_t *>(codes + (size_t)j * DV + 4 * cq);
            const float2 av = S.a2[j];
            float f[4];
            s8x4_to_f(w, f);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                ak[u] = fmaf(f[u], av.x, ak[u]);
                aq[u] = fmaf(f[u], av.y, aq[u]);
            }
        }
        if (RPP == 2) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                ak[u] += __shfl_xor_sync(0xffffffffu, ak[u], 16);
                aq[u] += __shfl_xor_sync(0xffffffffu, aq[u], 16);
            }
        }
        if (lane < DV / 4) {
            const float4 sc = *reinterpret_cast<const float4 *>(s_s + 4 * lane);
            const float s4[4] = {sc.x, sc.y, sc.z, sc.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                ek[u] = s4[u] * ak[u];
                eq[u] = s4[u] * aq[u];
            }
        }
        const uint16_t *hp = reinterpret_cast<const uint16_t *>(stage + L.off_hp);
        for (int p = warp; p < P; p += kBufWarps) {   // BF16 rows: unscaled x
            if (lane < DV / 4) {
                const uint2 hb = *reinterpret_cast<const uint2 *>(hp + (size_t)p * DV + 4 * lane);
                const int row = S.rows[NI + p];
                const float2 x = make_float2(S.x2[row].x * sig_s[row], S.x2[row].y * sig_s[row]);
                const float f0 = bf16_to_f((uint16_t)(hb.x & 0xffff)), f1 = bf16_to_f((uint16_t)(hb.x >> 16));
                const float f2 = bf16_to_f((uint16_t)(hb.y & 0xffff)), f3 = bf16_to_f((uint16_t)(hb.y >> 16));
                ek[0] = fmaf(f0, x.x, ek[0]); ek[1] = fmaf(f1, x.x, ek[1]);
                ek[2] = fmaf(f2, x.x, ek[2]); ek[3] = fmaf(f3, x.x, ek[3]);
                eq[0] = fmaf(f0, x.y, eq[0]); eq[1] = fmaf(f1, x.y, eq[1]);
                eq[2] = fmaf(f2, x.y, eq[2]); eq[3] = fmaf(f3, x.y, eq[3]);
            }
        }
    }

    // (d) entries: y += u_e (ktil_e . x), a pair per warp step, next pair in flight.
    {
        float xk[XPL], xq[XPL];
#pragma unroll
        for (int u = 0; u < XPL; ++u) {
            const float2 x = S.x2[XPL * lane + u];
            xk[u] = x.x;
            xq[u] = x.y;
        }
        // decay guard: the entries' key side rescaled by rho (exact) in
        // registers and written back, once for this step and the rest of the
        // window (entries E - 1 and before; this step's own is appended below)
        auto rescale = [&](int p, int e) {
            float rl[XPL];
#pragma unroll
            for (int u = 0; u < XPL; ++u) rl[u] = rho_s[XPL * lane + u];
            if (XPL == 4) {
                kb[p] = make_float4(kb[p].x * rl[0], kb[p].y * rl[1 % XPL], kb[p].z * rl[2 % XPL], kb[p].w * rl[3 % XPL]);
                if (!tb || e < L.r) {
                    reinterpret_cast<float4 *>(rec_ent + (size_t)e * EF)[lane] = kb[p];
                } else {
                    const uint32_t lo = (uint32_t)bf16_rne(kb[p].x) | ((uint32_t)bf16_rne(kb[p].y) << 16);
                    const uint32_t hi = (uint32_t)bf16_rne(kb[p].z) | ((uint32_t)bf16_rne(kb[p].w) << 16);
                    reinterpret_cast<uint2 *>(rec_tok16 + (size_t)(e - L.r) * EF)[lane] = make_uint2(lo, hi);
                }
            } else {
                kb2[p] = make_float2(kb2[p].x * rl[0], kb2[p].y * rl[1 % XPL]);
                if (!tb || e < L.r) {
                    reinterpret_cast<float2 *>(rec_ent + (size_t)e * EF)[lane] = kb2[p];
                } else {
                    reinterpret_cast<uint32_t *>(rec_tok16 + (size_t)(e - L.r) * EF)[lane] =
                        (uint32_t)bf16_rne(kb2[p].x) | ((uint32_t)bf16_rne(kb2[p].y) << 16);
                }
            }
        };
        if constexpr (!Q4) {
            for (int e0 = 2 * warp; e0 < E; e0 += 2 * kBufWarps) {
                if (rebase) {
#pragma unroll
                    for (int p = 0; p < 2; ++p)
                        if (e0 + p < E) rescale(p, e0 + p);
                }
                float d[4];
                float4 uv[2];
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    float dk_ = 0.f, dq_ = 0.f;
                    if (e0 + p < E) {
                        if (XPL == 4) {
                            const float4 kv = kb[p];
                            dk_ = fmaf(kv.x, xk[0], fmaf(kv.y, xk[1 % XPL], fmaf(kv.z, xk[2 % XPL], kv.w * xk[3 % XPL])));
                            dq_ = fmaf(kv.x, xq[0], fmaf(kv.y, xq[1 % XPL], fmaf(kv.z, xq[2 % XPL], kv.w * xq[3 % XPL])));
                        } else {
                            const float2 kv = kb2[p];
                            dk_ = fmaf(kv.x, xk[0], kv.y * xk[1 % XPL]);
                            dq_ = fmaf(kv.x, xq[0], kv.y * xq[1 % XPL]);
                        }
                    }
                    d[2 * p] = dk_;
                    d[2 * p + 1] = dq_;
                    uv[p] = ub[p];
                }
                const int ne = min(2, E - e0);
                load_pair(e0 + 2 * kBufWarps);   // refill the registers while this pair is reduced
                warp_reduce_dots<2>(d);
                if (lane < DV / 4) {
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        if (p < ne) {
                            ek[0] = fmaf(uv[p].x, d[2 * p], ek[0]); ek[1] = fmaf(uv[p].y, d[2 * p], ek[1]);
                            ek[2] = fmaf(uv[p].z, d[2 * p], ek[2]); ek[3] = fmaf(uv[p].w, d[2 * p], ek[3]);
                            eq[0] = fmaf(uv[p].x, d[2 * p + 1], eq[0]); eq[1] = fmaf(uv[p].y, d[2 * p + 1], eq[1]);
                            eq[2] = fmaf(uv[p].z, d[2 * p + 1], eq[2]); eq[3] = fmaf(uv[p].w, d[2 * p + 1], eq[3]);
                        }
                    }
                }
            }
        } else {
            // compensators: FP32 pairs
            for (int e0 = 2 * warp; e0 < L.r; e0 += 2 * kBufWarps) {
                if (rebase) {
#pragma unroll
                    for (int p = 0; p < 2; ++p)
                        if (e0 + p < L.r) rescale(p, e0 + p);
                }
                float d[4];
                float4 uv[2];
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    float dk_ = 0.f, dq_ = 0.f;
                    if (e0 + p < L.r) {
                        const float4 kv = kb[p];
                        dk_ = fmaf(kv.x, xk[0], fmaf(kv.y, xk[1], fmaf(kv.z, xk[2], kv.w * xk[3])));
                        dq_ = fmaf(kv.x, xq[0], fmaf(kv.y, xq[1], fmaf(kv.z, xq[2], kv.w * xq[3])));
                    }
                    d[2 * p] = dk_;
                    d[2 * p + 1] = dq_;
                    uv[p] = ub[p];
                }
                const int ne = min(2, L.r - e0);
#pragma unroll
                for (int p = 0; p < 2; ++p)
                    if (e0 + 2 * kBufWarps + p < L.r) load_fp32(p, e0 + 2 * kBufWarps + p);
                warp_reduce_dots<2>(d);
                if (lane < DV / 4) {
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        if (p < ne) {
                            ek[0] = fmaf(uv[p].x, d[2 * p], ek[0]); ek[1] = fmaf(uv[p].y, d[2 * p], ek[1]);
                            ek[2] = fmaf(uv[p].z, d[2 * p], ek[2]); ek[3] = fmaf(uv[p].w, d[2 * p], ek[3]);
                            eq[0] = fmaf(uv[p].x, d[2 * p + 1], eq[0]); eq[1] = fmaf(uv[p].y, d[2 * p + 1], eq[1]);
                            eq[2] = fmaf(uv[p].z, d[2 * p + 1], eq[2]); eq[3] = fmaf(uv[p].w, d[2 * p + 1], eq[3]);
                        }
                    }
                }
            }
            if (lane < DV / 4) {   // the compensators' part, before the tokens' registers
#pragma unroll
                for (int u = 0; u < 4; ++u) S.red[warp][4 * lane + u] = make_float2(ek[u], eq[u]);
            }
            // tokens: BF16 quads.  R holds (G k, G q) of key channels 8 l ..
            // 8 l + 7 on lanes l < 16, which form the dot products, and the
            // sums of value columns 8 (l - 16) .. on lanes l >= 16.
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float2 x = lane < 16 ? S.x2[8 * lane + c] : make_float2(0.f, 0.f);
                R[c] = x.x;
                R[8 + c] = x.y;
            }
            for (int j0 = 4 * warp; j0 < n; j0 += 4 * kBufWarps) {
                if (rebase && lane < 16) {   // the keys' rescaling, written back in BF16
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (j0 + i < n) {
                            uint32_t w[4] = {tkq[i].x, tkq[i].y, tkq[i].z, tkq[i].w};
#pragma unroll
                            for (int c2 = 0; c2 < 4; ++c2) {
                                const float2 f = bf16x2_to_f2(w[c2]);
                                w[c2] = (uint32_t)bf16_rne(f.x * rho_s[8 * lane + 2 * c2]) |
                                        ((uint32_t)bf16_rne(f.y * rho_s[8 * lane + 2 * c2 + 1]) << 16);
                            }
                            tkq[i] = make_uint4(w[0], w[1], w[2], w[3]);
                            reinterpret_cast<uint4 *>(rec_tok16 + (size_t)(j0 + i) * EF)[lane] = tkq[i];
                        }
                    }
                }
                float d[8];
                uint4 uk[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float dk_ = 0.f, dq_ = 0.f;
                    if (j0 + i < n && lane < 16) {
                        const uint32_t w[4] = {tkq[i].x, tkq[i].y, tkq[i].z, tkq[i].w};
#pragma unroll
                        for (int c2 = 0; c2 < 4; ++c2) {
                            const float2 f = bf16x2_to_f2(w[c2]);
                            dk_ = fmaf(f.x, R[2 * c2], fmaf(f.y, R[2 * c2 + 1], dk_));
                            dq_ = fmaf(f.x, R[8 + 2 * c2], fmaf(f.y, R[8 + 2 * c2 + 1], dq_));
                        }
                    }
                    d[2 * i] = dk_;
                    d[2 * i + 1] = dq_;
                    uk[i] = tkq[i];
                }
                const int ne = min(4, n - j0);
                load_quad(j0 + 4 * kBufWarps);   // the next quad in flight while this one is reduced
                warp_reduce_dots<4>(d);
                if (lane >= 16) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (i < ne) {
                            const uint32_t w[4] = {uk[i].x, uk[i].y, uk[i].z, uk[i].w};
#pragma unroll
                            for (int c2 = 0; c2 < 4; ++c2) {
                                const float2 f = bf16x2_to_f2(w[c2]);
                                R[2 * c2] = fmaf(f.x, d[2 * i], R[2 * c2]);
                                R[2 * c2 + 1] = fmaf(f.y, d[2 * i], R[2 * c2 + 1]);
                                R[8 + 2 * c2] = fmaf(f.x, d[2 * i + 1], R[8 + 2 * c2]);
                                R[8 + 2 * c2 + 1] = fmaf(f.y, d[2 * i + 1], R[8 + 2 * c2 + 1]);
                            }
                        }
                    }
                }
            }
        }
    }

    // (e) combine, output, append.
    if constexpr (!Q4) {
        if (lane < DV / 4) {
#pragma unroll
            for (int u = 0; u < 4; ++u) S.red[warp][4 * lane + u] = make_float2(ek[u], eq[u]);
        }
    } else {
        __syncwarp();
        if (lane >= 16) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float2 &r = S.red[warp][8 * (lane - 16) + c];
                r = make_float2(r.x + R[c], r.y + R[8 + c]);
            }
        }
    }
    uint16_t khat = 0;
    if (tb) {
        // the key of the update the state carries: Gamma bf16(k / Gamma)
        float kqh = 0.f;
        if (t < DK) {
            khat = bf16_rne(kk / gt);
            kqh = (gt * bf16_to_f(khat)) * S.qk[t];
        }
        kqh = warp_sum(kqh);
        if (lane == 0) S.kqw[warp] = kqh;
    }
    __syncthreads();
    if (tb) {
        kq = 0.f;
#pragma unroll
        for (int w = 0; w < kBufWarps; ++w) kq += S.kqw[w];
    }
    if (t < DV) {
        float yk = DAMP ? 0.f : S.rc[t].x, yq = DAMP ? 0.f : S.rc[t].y;
#pragma unroll
        for (int w = 0; w < kBufWarps; ++w) {
            const float2 p = S.red[w][t];
            yk += p.x;
            yq += p.y;
        }
        float ut = beta * (S.v[t] - yk);
        if (tb) {
            const uint16_t uh = bf16_rne(ut);
            rec_tok16[(size_t)n * EF + DK + t] = uh;
            ut = bf16_to_f(uh);
        } else {
            rec_ent[(size_t)E * EF + DK + t] = ut;
        }
        const float o = fmaf(ut, kq, yq);
        a.o[hv * DV + t] = o;
        if (!isfinite(o) || !isfinite(ut)) atomicOr(a.status, kStatusNonFinite);
    }
    if (t < DK) {
        if (tb) rec_tok16[(size_t)n * EF + t] = khat;
        else rec_ent[(size_t)E * EF + t] = kk / gt;
        if (KDA) {
            rec_gam[t] = gt;
            rec_sig[t] = sg;
        } else if (t == 0) {
            rec_gam[0] = gt;
            rec_sig[0] = sg;
        }
    }
}

// ---------------------------------------------------------------------------
// Window-end step: one CTA of 128 threads per head, three per SM (a 128-row
// tile is 128 registers a thread).  The record prefix (m, s, BF16 rows,
// codes) is staged with one bulk copy and the r+n entries stream through two
// shared-memory buffers of kFlushChunk entries, one chunk in flight while the
// previous one is applied; the tile
//   S' = Gamma_t [Deq + sum_e ktil_e u_e^T]
// is built in registers, the step's outputs come from it (y_k = S'^T k_t,
// y_q = S'^T q_t), S_t = S' + k_t u_t^T is quantized in place (new
// compensators, smoothing, codes) and Gamma restarts at 1.
// kExport instead writes the current state Gamma [Deq + buffer] (no token);
// kFlushOnly ends the window without a token (lq_window_flush).
// ---------------------------------------------------------------------------
constexpr int kFlushThreads = 128;
constexpr int kFlushWarps = kFlushThreads / 32;
constexpr int kFlushChunk = 8;   // entries per staged chunk: one TF32 MMA K-block

template <int DK, int DV>
struct FlushSmem {
    float k[DK], ke[DK], q[DK], gam[DK], sig[DK];
    float u[DV];
    float kqw[kFlushWarps];
    int map[DK];
    int wscr[kFlushWarps];
    CodecSmem<DK, DV, kFlushThreads> cs;
    uint64_t mbar_pre;
    uint64_t mbar_mma[2];
    uint32_t tmem_base;
};

template <int DK, int DV>
__host__ __device__ constexpr size_t flush_fixed_bytes() {
    return (sizeof(FlushSmem<DK, DV>) + 127) / 128 * 128;
}

// Shared memory of the flush, in this order (all 128-byte aligned):
//   FlushSmem | work area | record prefix
// d_k = 128 (tensor-core reconstruction): the work area holds two operand
// buffers, each the TF32 big / small parts of one chunk's ktil^T [dk][8] and
// u^T [dv][8] in K-major core-matrix layout; the entries come from global
// memory into registers one chunk ahead.  They come before the prefix so that
// everything a descriptor can address stays inside the allocation; afterwards
// the work area is the accumulator's transposition scratch.  d_k = 64 needs
// no work area.
__host__ __device__ inline size_t flush_ops_bytes(int dk, int dv) { return (size_t)2 * (dk + dv) * 32; }
__host__ __device__ inline size_t flush_work_bytes(int dk, int dv) { return dk == 128 ? 2 * flush_ops_bytes(dk, dv) : 0; }

inline size_t flush_smem_bytes(int dk, int dv, const Layout &L) {
    size_t fixed = 0;
    if (dk == 64 && dv == 64) fixed = flush_fixed_bytes<64, 64>();
    if (dk == 64 && dv == 128) fixed = flush_fixed_bytes<64, 128>();
    if (dk == 128 && dv == 64) fixed = flush_fixed_bytes<128, 64>();
    if (dk == 128 && dv == 128) fixed = flush_fixed_bytes<128, 128>();
    return fixed + flush_work_bytes(dk, dv) + (size_t)align_up(L.off_ent, 128);
}

enum { kFlushStep = 0, kFlushOnly = 1, kExport = 2 };

template <int DK, int DV, bool KDA, bool DAMP, int MODE, bool TB, int BITS>
__global__ void __launch_bounds__(kFlushThreads, 3) decode_flush_kernel(const DecodeArgs a) {
    static_assert(BITS == 8 || !DAMP, "packed codes are built without BF16 rows");
    constexpr int NT = kFlushThreads;
    constexpr int EF = DK + DV;   // floats per entry
    extern __shared__ __align__(128) unsigned char smem[];
    using T = Tile<DK, DV, NT>;
    FlushSmem<DK, DV> &F = *reinterpret_cast<FlushSmem<DK, DV> *>(smem);
    const Layout &L = a.L;
    unsigned char *work = smem + flush_fixed_bytes<DK, DV>();
    unsigned char *stage = work + flush_work_bytes(DK, DV);
    // (staggered windows: the grid covers the listed batch entries only)
    const int b = a.flush_list ? __ldg(a.flush_list + blockIdx.x / a.H) : (int)(blockIdx.x / a.H);
    const int h = (int)(blockIdx.x % a.H), g = (h * a.Hk) / a.H;
    const int head = b * a.H + h;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int cg = t % T::CG, row0 = (t / T::CG) * T::RPT;
    const int P = DAMP ? L.P : 0;
    const int n = entry_pos(a, b).n;
    // an explicit window end with nothing buffered leaves the state as it is
    if (MODE == kFlushOnly && n == 0) return;
    const int E = L.r + n;
    const int nch = (E + kFlushChunk - 1) / kFlushChunk;
    unsigned char *rec = a.rec + (size_t)head * L.rec_bytes;
    float *rec_ent = reinterpret_cast<float *>(rec + L.off_ent);
    const uint16_t *rec_tok16 = reinterpret_cast<const uint16_t *>(rec + L.off_tok);
    float *rec_gam = reinterpret_cast<float *>(rec + L.off_gam);   // G
    float *rec_sig = rec_gam + (KDA ? DK : 1);                       // sigma
    const size_t hv = (size_t)b * a.H + h;
    constexpr bool tb = TB;   // buffered tokens in BF16
    // element x of entry e (e < r: a compensator, else buffered token e - r)
    auto entry_at = [&](int e, int x) -> float {
        if (!tb || e < L.r) return __ldcs(rec_ent + (size_t)e * EF + x);
        return bf16_to_f(__ldcs(rec_tok16 + (size_t)(e - L.r) * EF + x));
    };

    if (t == 0) {
        mbar_init(&F.mbar_pre, 1);
        mbar_init(&F.mbar_mma[0], 1);
        mbar_init(&F.mbar_mma[1], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (t == 0) {
        mbar_arrive_expect_tx(&F.mbar_pre, (uint32_t)L.off_ent);
        bulk_g2s(stage, rec, (uint32_t)L.off_ent, &F.mbar_pre);
    }
    float kqp = 0.f;
    if (t < DK) {
        // the buffer is keyed to G and the quantized state scaled by sigma G
        // (decay guard); the tile is G [sigma Deq + entries], times this
        // step's decay for a window-end token (a product: it may underflow)
        const float gp = n > 0 ? (KDA ? rec_gam[t] : rec_gam[0]) : 1.0f;
        const float sp = n > 0 ? (KDA ? rec_sig[t] : rec_sig[0]) : 1.0f;
        float gt = gp;
        if (MODE == kFlushStep) {
            const size_t qk = ((size_t)b * a.Hk + g) * DK;
            const float kk = a.k[qk + t], qq = a.q[qk + t];
            const float at = KDA ? a.alpha[hv * DK + t] : a.alpha[hv];
            gt = at * gp;
            // the key of the update the state takes: k, or G bf16(k / G) with
            // the guarded G a buffering step would key this token to
            float rho;
            const float gc = gate_chain(at, gp, rho);
            const float ke = tb ? gc * bf16_round(kk / gc) : kk;
            F.k[t] = kk;
            F.ke[t] = ke;
            F.q[t] = qq;
            kqp = ke * qq;
        }
        F.gam[t] = gt;
        F.sig[t] = sp;
    }
    kqp = warp_sum(kqp);
    if (lane == 0) F.kqw[warp] = kqp;
    if (DAMP) build_row_map<DK, NT>(a.hp_rows + (size_t)h * P, P, F.map, F.wscr);
    const bool okw = mbar_wait_bounded(&F.mbar_pre, 0, a.status);
    if (__syncthreads_or(!okw)) return;

    // R = sum_e ktil_e u_e^T over the r + n entries, then += Deq, then * Gamma.
    float R[T::RPT][16];
    auto zero_tile = [&]() {
#pragma unroll
        for (int r = 0; r < T::RPT; ++r)
#pragma unroll
            for (int q = 0; q < 16; ++q) R[r][q] = 0.f;
    };
    if constexpr (DK == 128) {
        // On the tensor cores: per chunk of 8 entries, A = ktil^T [128][8] and
        // B = u^T [DV][8] split into TF32 big + small parts, three MMAs (big
        // big, big small, small big) accumulating D [128][DV] in tensor
        // memory.  The entries of chunk c+1 are loaded into registers while
        // chunk c is converted; operand buffer c & 1 is reused once the MMAs
        // of chunk c-2, committed to mbar_mma[c & 1], have completed.
        if (nch == 0) {
            zero_tile();
        } else {
            constexpr uint32_t TCOLS = DV;   // 64 or 128 columns: a power of two >= 32
            constexpr uint32_t IDESC = umma_idesc_tf32(DK, DV);
            constexpr int OPW = (int)((2 * (DK + DV) * 32) / 4);   // words per operand buffer
            if (warp == 0) {
                tmem_alloc(&F.tmem_base, TCOLS);
                tmem_relinquish();
            }
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            const uint32_t tmem = F.tmem_base;
            // row x of a K-major [rows][8] TF32 operand: 16 bytes (4 words) per
            // core-matrix row, core matrices of 8 rows 128 bytes (32 words)
            // apart (SBO), the second 16 bytes of K rows*16 bytes further (LBO)
            auto put_row = [&](uint32_t *big, uint32_t *small, int rows, int x, const float (&src)[8]) {
                uint32_t hb[8], hs[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) tf32_split(src[e], hb[e], hs[e]);
                uint32_t *pb = big + (x >> 3) * 32 + (x & 7) * 4;
                uint32_t *ps = small + (x >> 3) * 32 + (x & 7) * 4;
                *reinterpret_cast<uint4 *>(pb) = make_uint4(hb[0], hb[1], hb[2], hb[3]);
                *reinterpret_cast<uint4 *>(pb + rows * 4) = make_uint4(hb[4], hb[5], hb[6], hb[7]);
                *reinterpret_cast<uint4 *>(ps) = make_uint4(hs[0], hs[1], hs[2], hs[3]);
                *reinterpret_cast<uint4 *>(ps + rows * 4) = make_uint4(hs[4], hs[5], hs[6], hs[7]);
            };
            // this thread's key row (A) / value column (B) of a chunk's entries,
            // loaded one chunk ahead of its conversion
            float xa[8], xb[8];
            // (the FP32-or-BF16 choice is made per chunk, so that the common
            // all-token chunk issues its 16 loads without branches between them)
            auto load_chunk = [&](int c) {
                const int n = min(kFlushChunk, E - c * kFlushChunk);
                if (tb && c * kFlushChunk >= L.r) {
                    const uint16_t *src = rec_tok16 + (size_t)(c * kFlushChunk - L.r) * EF;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        xa[e] = e < n ? bf16_to_f(__ldcs(src + e * EF + t)) : 0.f;
                        xb[e] = (e < n && t < DV) ? bf16_to_f(__ldcs(src + e * EF + DK + t)) : 0.f;
                    }
                } else if (!tb) {
                    const float *src = rec_ent + (size_t)c * kFlushChunk * EF;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        xa[e] = e < n ? __ldcs(src + e * EF + t) : 0.f;
                        xb[e] = (e < n && t < DV) ? __ldcs(src + e * EF + DK + t) : 0.f;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        xa[e] = e < n ? entry_at(c * kFlushChunk + e, t) : 0.f;
                        xb[e] = (e < n && t < DV) ? entry_at(c * kFlushChunk + e, DK + t) : 0.f;
                    }
                }
            };
            load_chunk(0);
            int c = 0;   // chunks committed
            bool ok = true;
            for (int cc = 0; cc < nch; ++cc) {
                uint32_t *opA_big = reinterpret_cast<uint32_t *>(work) + (cc & 1) * OPW;
                uint32_t *opA_small = opA_big + DK * 8;
                uint32_t *opB_big = opA_small + DK * 8;
                uint32_t *opB_small = opB_big + DV * 8;
                const bool okc = cc < 2 || mbar_wait_bounded(&F.mbar_mma[cc & 1], ((cc >> 1) - 1) & 1, a.status);
                if (__syncthreads_or(!okc)) {
                    ok = false;
                    break;
                }
                put_row(opA_big, opA_small, DK, t, xa);
                if (t < DV) put_row(opB_big, opB_small, DV, t, xb);
                if (cc + 1 < nch) load_chunk(cc + 1);
                fence_async_smem();
                tc_fence_before();
                __syncthreads();
                if (t == 0) {
                    tc_fence_after();
                    const uint64_t ab = umma_smem_desc(opA_big, DK * 16, 128);
                    const uint64_t bb = umma_smem_desc(opB_big, DV * 16, 128);
                    umma_tf32(tmem, ab, bb, IDESC, cc > 0 ? 1u : 0u);
                    // BF16 tokens are exact in TF32 (the small parts are zero):
                    // a chunk of them needs the big x big pass only
                    if (!tb || cc * kFlushChunk < L.r) {
                        const uint64_t as = umma_smem_desc(opA_small, DK * 16, 128);
                        const uint64_t bs = umma_smem_desc(opB_small, DV * 16, 128);
                        umma_tf32(tmem, ab, bs, IDESC, 1u);
                        umma_tf32(tmem, as, bb, IDESC, 1u);
                    }
                    umma_commit(&F.mbar_mma[cc & 1]);
                }
                c = cc + 1;
            }
            // chunks 0 .. c-1 were committed; the last commit completes after
            // every earlier MMA
            bool okm = c == 0 || mbar_wait_bounded(&F.mbar_mma[(c - 1) & 1], ((c - 1) >> 1) & 1, a.status);
            okm = !__syncthreads_or(!okm) && ok;
            tc_fence_after();
            if (okm) {
                // D -> register tile in four slices of DV/4 columns through
                // the work area (both operand buffers, consumed): thread l of
                // warp w holds D row 32 w + l of the slice
                constexpr int SW = DV / 4, SP = SW + 4;   // slice width, padded row pitch
                float *scr = reinterpret_cast<float *>(work);
#pragma unroll
                for (int qs = 0; qs < 4; ++qs) {
                    uint32_t v[SW];
                    tmem_ld_32x32b<SW>(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)(qs * SW), v);
                    tmem_ld_wait();
                    float *rowp = scr + (size_t)(32 * warp + lane) * SP;
#pragma unroll
                    for (int j = 0; j < SW / 4; ++j)
                        *reinterpret_cast<float4 *>(rowp + 4 * j) =
                            make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                        __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                    __syncthreads();
#pragma unroll
                    for (int r = 0; r < T::RPT; ++r) {
                        const float4 f = *reinterpret_cast<const float4 *>(scr + (size_t)(row0 + r) * SP + 4 * cg);
                        R[r][4 * qs] = f.x;
                        R[r][4 * qs + 1] = f.y;
                        R[r][4 * qs + 2] = f.z;
                        R[r][4 * qs + 3] = f.w;
                    }
                    __syncthreads();
                }
            }
            tc_fence_before();
            __syncthreads();
            if (warp == 0) {
                tc_fence_after();
                tmem_dealloc(tmem, TCOLS);
            }
            if (!okm) return;
        }
    } else {
        // d_k = 64: the entries straight from memory (every thread of the CTA
        // reads the same rows: cached), packed FP32 FMAs on the tile
        zero_tile();
        for (int e = 0; e < E; ++e) {
            float kv[T::RPT], uv[16];
#pragma unroll
            for (int r = 0; r < T::RPT; ++r) kv[r] = entry_at(e, row0 + r);
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int u = 0; u < 4; ++u) uv[4 * q + u] = entry_at(e, DK + T::col(cg, q) + u);
#pragma unroll
            for (int r = 0; r < T::RPT; ++r)
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float2 o = ffma2(f2(kv[r], kv[r]), f2(uv[2 * q], uv[2 * q + 1]), f2(R[r][2 * q], R[r][2 * q + 1]));
                    R[r][2 * q] = o.x;
                    R[r][2 * q + 1] = o.y;
                }
        }
    }
    tile_dequant<DK, DV, NT, true, BITS>(R, reinterpret_cast<const float *>(stage + L.off_m),
                                   reinterpret_cast<const float *>(stage + L.off_s),
                                   reinterpret_cast<const uint16_t *>(stage + L.off_hp),
                                   reinterpret_cast<const int8_t *>(stage + L.off_codes), P, DAMP ? F.map : nullptr,
                                   !DAMP, F.sig);
    const bool fin = tile_gamma<DK, DV, NT>(R, F.gam);
    if (!fin) atomicOr(a.status, kStatusNonFinite);

    if (MODE == kExport) {
        tile_store_global<DK, DV, NT>(R, a.S_out + (size_t)head * DK * DV);
        return;
    }
    if (MODE == kFlushStep) {
        // y_k = S'^T k, y_q = S'^T q over the tile (one vector at a time, to
        // keep the registers beside the tile few), one barrier.
        float(*rk)[DV] = F.cs.red[0];
        float(*rq)[DV] = F.cs.red[1];
#pragma unroll 1
        for (int vsel = 0; vsel < 2; ++vsel) {
            const float *xs = vsel ? F.q : F.k;
            float zx[T::RPT];
#pragma unroll
            for (int r = 0; r < T::RPT; ++r) zx[r] = xs[row0 + r];
            float acc[16];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float2 ax = f2(0.f, 0.f);
#pragma unroll
                for (int r = 0; r < T::RPT; ++r) ax = ffma2(f2(R[r][2 * j], R[r][2 * j + 1]), f2(zx[r], zx[r]), ax);
                acc[2 * j] = ax.x;
                acc[2 * j + 1] = ax.y;
            }
            xpose_reduce<16, 16, T::CG>(acc);   // over the warp's row groups
            constexpr int NR = 16 >> xpose_bits<16, T::CG>();
            const int base = xpose_base<16, 16, T::CG>(lane);
            float *dst = (vsel ? rq[warp] : rk[warp]) + T::col(cg, base / 4) + base % 4;
            if (NR == 4) *reinterpret_cast<float4 *>(dst) = make_float4(acc[0], acc[1], acc[2 % NR], acc[3 % NR]);
            else *reinterpret_cast<float2 *>(dst) = make_float2(acc[0], acc[1 % NR]);
        }
        cbar<NT>();
        if (t < DV) {
            float yk = 0.f, yq = 0.f, kq = 0.f;
#pragma unroll
            for (int w = 0; w < kFlushWarps; ++w) {
                yk += rk[w][t];
                yq += rq[w][t];
                kq += F.kqw[w];
            }
            float ut = a.beta[hv] * (a.v[hv * DV + t] - yk);
            if (tb) ut = bf16_round(ut);   // the update the state takes: u or bf16(u)
            const float o = fmaf(ut, kq, yq);
            a.o[hv * DV + t] = o;
            F.u[t] = ut;
            if (!isfinite(o) || !isfinite(ut)) atomicOr(a.status, kStatusNonFinite);
        }
        cbar<NT>();
        float uv[16];
        load_cols16<DK, DV>(F.u, uv);
#pragma unroll
        for (int r = 0; r < T::RPT; ++r) {
            const float kk = F.ke[row0 + r];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float2 o = ffma2(f2(kk, kk), f2(uv[2 * c], uv[2 * c + 1]), f2(R[r][2 * c], R[r][2 * c + 1]));
                R[r][2 * c] = o.x;
                R[r][2 * c + 1] = o.y;
            }
        }
    }
    CodecOut out;
    out.codes = reinterpret_cast<int8_t *>(rec + L.off_codes);
    out.codes_t = DAMP ? 0 : 1;
    out.hp = reinterpret_cast<uint16_t *>(rec + L.off_hp);
    out.m = reinterpret_cast<float *>(rec + L.off_m);
    out.s = reinterpret_cast<float *>(rec + L.off_s);
    out.ck = rec_ent;
    out.ck_stride = DK + DV;
    out.cw = rec_ent + DK;
    out.cw_stride = DK + DV;
    double eacc[T::RPT];
    codec_quantize<DK, DV, false, NT, BITS>(R, L.r, a.K, a.smoothing, P, DAMP ? F.map : nullptr, F.cs, out, eacc);
    if (KDA) {
        if (t < DK) {
            rec_gam[t] = 1.0f;
            rec_sig[t] = 1.0f;
        }
    } else if (t == 0) {
        rec_gam[0] = 1.0f;
        rec_sig[0] = 1.0f;
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

// Shared-memory carveout of the buffering kernel: 85% of the SM's 228 KB,
// rounded up by the driver to the 196 KB configuration, leaves ~60 KB of L1
// for the streamed entries and step inputs and room for 7 CTAs of ~27 KB
// (measured: the 228 KB configuration that 8 CTAs would need, with 28 KB of
// L1, is ~9% slower).
constexpr int kBufCarveoutPct = 85;

template <int DK, int DV, bool KDA, bool DAMP, bool TB, int BITS>
static cudaError_t launch_buffer_t(const DecodeArgs &a, int heads, cudaStream_t s) {
    const size_t sm = buffer_smem_bytes(DK, DV, a.L);
    auto kern = decode_buffer_kernel<DK, DV, KDA, DAMP, TB, BITS>;
    static size_t done = 0;
    static bool carved = false;
    cudaError_t e = set_smem(kern, sm, done);
    if (e != cudaSuccess) return e;
    if (!carved) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, kBufCarveoutPct);
        if (e != cudaSuccess) return e;
        carved = true;
    }
    // launched as a programmatic dependent of the previous launch on the
    // stream (the kernel waits for it before reading what it wrote)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)heads);
    cfg.blockDim = dim3(kBufThreads);
    cfg.dynamicSmemBytes = sm;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int DK, int DV, bool KDA, bool DAMP, int MODE, bool TB, int BITS>
static cudaError_t launch_flush_t(const DecodeArgs &a, int heads, cudaStream_t s) {
    const size_t sm = flush_smem_bytes(DK, DV, a.L);
    auto kern = decode_flush_kernel<DK, DV, KDA, DAMP, MODE, TB, BITS>;
    static size_t done = 0;
    cudaError_t e = set_smem(kern, sm, done);
    if (e != cudaSuccess) return e;
    kern<<<heads, kFlushThreads, sm, s>>>(a);
    return cudaGetLastError();
}

#define LQ_DISPATCH_DKDV(dk, dv, FN)                   \
    (((dk) == 128 && (dv) == 128)  ? FN<128, 128>      \
     : ((dk) == 64 && (dv) == 64)  ? FN<64, 64>        \
     : ((dk) == 64 && (dv) == 128) ? FN<64, 128>       \
                                   : FN<128, 64>)

// BF16 tokens and packed codes are built without BF16 rows (the
// configuration check rejects those combinations).
template <int BITS>
struct DecodeSet {
    template <int DK, int DV, bool KDA>
    static cudaError_t buffer(const DecodeArgs &a, int heads, bool damp, cudaStream_t s) {
        if (damp) {
            if constexpr (BITS == 8) return launch_buffer_t<DK, DV, KDA, true, false, 8>(a, heads, s);
            else return cudaErrorInvalidValue;
        }
        return a.L.tok_bf16 ? launch_buffer_t<DK, DV, KDA, false, true, BITS>(a, heads, s)
                            : launch_buffer_t<DK, DV, KDA, false, false, BITS>(a, heads, s);
    }
    template <int DK, int DV, bool KDA, int MODE>
    static cudaError_t flush(const DecodeArgs &a, int heads, bool damp, cudaStream_t s) {
        if (damp) {
            if constexpr (BITS == 8) return launch_flush_t<DK, DV, KDA, true, MODE, false, 8>(a, heads, s);
            else return cudaErrorInvalidValue;
        }
        return a.L.tok_bf16 ? launch_flush_t<DK, DV, KDA, false, MODE, true, BITS>(a, heads, s)
                            : launch_flush_t<DK, DV, KDA, false, MODE, false, BITS>(a, heads, s);
    }
    template <int DK, int DV>
    static cudaError_t buffer_dkdv(const DecodeArgs &a, int heads, bool kda, bool damp, cudaStream_t s) {
        return kda ? buffer<DK, DV, true>(a, heads, damp, s) : buffer<DK, DV, false>(a, heads, damp, s);
    }
    template <int DK, int DV>
    static cudaError_t flush_dkdv(const DecodeArgs &a, int heads, bool kda, bool damp, int mode, cudaStream_t s) {
        if (mode == kFlushStep)
            return kda ? flush<DK, DV, true, kFlushStep>(a, heads, damp, s)
                       : flush<DK, DV, false, kFlushStep>(a, heads, damp, s);
        if (mode == kFlushOnly)
            return kda ? flush<DK, DV, true, kFlushOnly>(a, heads, damp, s)
                       : flush<DK, DV, false, kFlushOnly>(a, heads, damp, s);
        return kda ? flush<DK, DV, true, kExport>(a, heads, damp, s) : flush<DK, DV, false, kExport>(a, heads, damp, s);
    }
    // A decode step (buffering, or flush-step when `flush`) or a flush /
    // export launch (mode kFlushOnly / kExport) for all heads.
    static cudaError_t decode(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool flush, bool damp,
                              cudaStream_t s) {
        if (flush) return LQ_DISPATCH_DKDV(dk, dv, flush_dkdv)(a, heads, kda, damp, kFlushStep, s);
        return LQ_DISPATCH_DKDV(dk, dv, buffer_dkdv)(a, heads, kda, damp, s);
    }
    static cudaError_t flush_only(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool damp, bool exp,
                                  cudaStream_t s) {
        return LQ_DISPATCH_DKDV(dk, dv, flush_dkdv)(a, heads, kda, damp, exp ? kExport : kFlushOnly, s);
    }
};

}  // namespace lq
