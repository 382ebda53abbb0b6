// lq_decode.cu -- the FP32-state reference step and the host entry points of
// the decode kernels; the windowed INT8 / low-bit kernels themselves live in
// lq_decode.cuh and are instantiated per code width in lq_decode_b8.cu,
// lq_decode_b6.cu and lq_decode_b4.cu (compiled in parallel).
#include "lq_common.cuh"
#include "lq_kernels.h"

namespace lq {

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
    __shared__ float u_s[DV];
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

template <int DK, int DV>
static cudaError_t fp32_dispatch(const Fp32Args &a, int heads, bool kda, cudaStream_t s) {
    if (kda) fp32_step_kernel<DK, DV, true><<<heads, kThreads, 0, s>>>(a);
    else fp32_step_kernel<DK, DV, false><<<heads, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool flush, bool damp,
                          cudaStream_t s) {
    switch (a.L.bits) {
        case 8: return launch_decode_b8(a, dk, dv, heads, kda, flush, damp, s);
        case 6: return launch_decode_b6(a, dk, dv, heads, kda, flush, damp, s);
        case 4: return launch_decode_b4(a, dk, dv, heads, kda, flush, damp, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_flush(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool damp, bool exp,
                         cudaStream_t s) {
    switch (a.L.bits) {
        case 8: return launch_flush_b8(a, dk, dv, heads, kda, damp, exp, s);
        case 6: return launch_flush_b6(a, dk, dv, heads, kda, damp, exp, s);
        case 4: return launch_flush_b4(a, dk, dv, heads, kda, damp, exp, s);
        default: return cudaErrorInvalidValue;
    }
}

#define LQ_FP32_DKDV(dk, dv, FN)                       \
    (((dk) == 128 && (dv) == 128)  ? FN<128, 128>      \
     : ((dk) == 64 && (dv) == 64)  ? FN<64, 64>        \
     : ((dk) == 64 && (dv) == 128) ? FN<64, 128>       \
                                   : FN<128, 64>)

cudaError_t launch_fp32_step(const Fp32Args &a, int dk, int dv, int heads, bool kda, cudaStream_t s) {
    return LQ_FP32_DKDV(dk, dv, fp32_dispatch)(a, heads, kda, s);
}

size_t decode_smem_bytes(int dk, int dv, const Layout &L) {
    const size_t a = flush_smem_bytes_of(dk, dv, L), b = buffer_smem_bytes_of(dk, dv, L);
    return a > b ? a : b;
}

}  // namespace lq
