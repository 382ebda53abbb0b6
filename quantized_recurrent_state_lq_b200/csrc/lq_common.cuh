// lq_common.cuh -- device helpers shared by the decode, flush and codec kernels:
// the per-head record layout, bulk-copy (TMA, non-tensor) staging with a
// bounded mbarrier wait, warp/block reductions and BF16 rounding.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace lq {

constexpr int kThreads = 256;  // every kernel here runs 8 warps per CTA
constexpr int kWarps = kThreads / 32;

// Sticky device status bits (reported by lq_get_status).
constexpr int kStatusNonFinite = 1;
constexpr int kStatusTimeout = 2;

// ---------------------------------------------------------------------------
// Per-head record in the workspace (INT8 modes).  One contiguous, 128-byte
// aligned slab per (batch, head):
//   m       f32   [dk]              smoothing scale per key row (1 on BF16 rows)
//   s       f32   [dv]              quantization scale per value column
//   hp      u16   [P][dv]           BF16 rows (order of the head's row list)
//   codes   int8  [dk-P][dv]        INT8 codes (layout: code_off_t below), or
//                                   4 / 6-bit codes bit-packed (nib_off, pair_off)
//   comps   f32   [r][dk+dv]        compensator j = (c_j [dk], w_j [dv])
//   tokens  f32 or bf16 [W][dk+dv]  buffered token tau = (k_tau/G_tau, u_tau)
//   gam     f32   [2][dk] (KDA) / [4] (GDN)   the decay since the window start
//                                   as G [dk] (GDN: [0]) and sigma [dk] ([1])
// Entries e < r are the compensators, e = r + tau the buffered tokens; with
// FP32 tokens both form one array [r+W][dk+dv].  A decode step reads
// [m .. codes] with one bulk copy and the r + n entries as coalesced streams.
//
// Decay guard.  The product Gamma_t of a window's decays can leave the FP32
// range for strong decays or long windows (a KDA channel at a = 0.73 passes
// 2^-126 after ~280 tokens; a gate of 0 ends it at once), and the buffered
// keys k / Gamma would overflow.  The kernels therefore carry Gamma_t, per
// key channel, as G_t * sigma_t: G_t in [2^-64, 1] (1 at the window start)
// keys the buffer (ktil = k / G, contribution ktil_tau u_tau^T G_t), and
// sigma_t, a power of two or 0, scales the quantized state alone
// (S_t = sigma_t G_t Deq + G_t [sum_j c_j w_j^T + sum_tau ktil_tau u_tau^T]).
// When a step's product a_t G_{t-1} falls below 2^-64, G is rescaled by 2^64
// and every buffered entry's key side (compensators included) and sigma by
// 2^-64 -- all exact -- or, when one step's decay takes it below 2^-128, the
// channel restarts: G = 1, and the entries' key side and sigma become 0
// (what they multiply is below 2^-128 of its size).  gate_chain takes that
// decision.
// ---------------------------------------------------------------------------
struct Layout {
    int dk, dv, P, r, W, kda;
    int tok_bf16;   // buffered tokens stored in BF16
    int bits;       // code width: 8, 6 or 4 (6 and 4 bit-packed, no BF16 rows)
    int off_m, off_s, off_hp, off_codes, off_ent, off_tok, off_gam;
    int rec_bytes;
};

__host__ __device__ inline int align_up(int x, int a) { return (x + a - 1) / a * a; }

__host__ inline Layout make_layout(int dk, int dv, int P, int r, int W, int kda, int tok_bf16 = 0, int bits = 8) {
    Layout L;
    L.dk = dk; L.dv = dv; L.P = P; L.r = r; L.W = W; L.kda = kda; L.tok_bf16 = tok_bf16; L.bits = bits;
    L.off_m = 0;
    L.off_s = dk * 4;
    L.off_hp = (dk + dv) * 4;
    L.off_codes = L.off_hp + P * dv * 2;
    L.off_ent = align_up(L.off_codes + (dk - P) * dv * bits / 8, 16);
    L.off_tok = L.off_ent + r * (dk + dv) * 4;
    int o = L.off_tok + W * (dk + dv) * (tok_bf16 ? 2 : 4);
    L.off_gam = align_up(o, 16);
    o = L.off_gam + (kda ? 2 * dk : 4) * 4;
    L.rec_bytes = align_up(o, 128);
    return L;
}

// INT8 codes without BF16 rows are stored value-column-major (row c holds the
// dk codes of value column c) so that they are the row-major A operand of an
// int8 tensor-core MMA over the key dimension; 16-byte chunks are XOR-swizzled
// by the column so that 8 consecutive columns read with ldmatrix hit 8
// different shared-memory bank groups.  With BF16 rows the codes stay
// row-major by INT8 slot: [slot][c].
// Chunk swizzle of a column-major plane whose columns are `row_bytes` (16 ..
// 128) long: the 16-byte chunk index is XORed with bits of the column so that
// the same chunk of 8 consecutive columns covers all 8 bank groups of 128 bytes.
__host__ __device__ __forceinline__ int chunk_swz(int c, int row_bytes) {
    return row_bytes >= 128 ? (c & 7) : row_bytes == 64 ? ((c >> 1) & 3) : row_bytes == 32 ? ((c >> 2) & 1) : 0;
}

__host__ __device__ __forceinline__ int code_swz(int c, int dk) { return chunk_swz(c, dk); }

__host__ __device__ __forceinline__ int code_off_t(int c, int i, int dk) {
    return c * dk + ((((i >> 4) ^ code_swz(c, dk)) << 4) | (i & 15));
}

// 4- and 6-bit codes (no BF16 rows), value-column-major and swizzled like the
// INT8 codes, in groups of 8 key rows g = i / 8:
//   nibble plane [dv][dk/2]: the low 4 bits of each code; a group is one
//     32-bit word (row 8g+k in bits 4k .. 4k+3) at byte nib_off(c, g);
//   pair plane [dv][dk/4] (6-bit only, after the nibble plane): bits 4-5 of
//     each code; a group is one 16-bit word (row 8g+k in bits 2k, 2k+1) at
//     byte pair_off(c, g).  Groups g and g+4 of a 64-row block share a 32-bit
//     word, so that one shared-memory matrix load hands a lane the pair bits
//     of both 32-row halves it multiplies.
__host__ __device__ __forceinline__ int nib_off(int c, int g, int dk) {
    const int rb = dk / 2, b = 4 * g;
    return c * rb + ((((b >> 4) ^ chunk_swz(c, rb)) << 4) | (b & 15));
}

__host__ __device__ __forceinline__ int pair_off(int c, int g, int dk, int dv) {
    const int rb = dk / 4, b = 16 * (g >> 3) + 4 * (g & 3) + 2 * ((g >> 2) & 1);
    return dv * (dk / 2) + c * rb + ((((b >> 4) ^ chunk_swz(c, rb)) << 4) | (b & 15));
}

// Position of key row i in the contraction order of the packed tensor-core
// GEMV: a lane's nibble word of 32-row block i / 32 holds rows 8tq .. 8tq+7,
// whose even rows fill MMA k-slots 4tq .. 4tq+3 and odd rows 16+4tq .. 16+4tq+3.
__host__ __device__ __forceinline__ int lowbit_kslot(int i) {
    return (i & ~31) | ((i & 1) << 4) | (((i >> 3) & 3) << 2) | ((i >> 1) & 3);
}

// An 8-row group as signed bytes c * 2^(8 - BITS) (exact: the code sits in the
// byte's top BITS bits): lo = rows 0, 2, 4, 6, hi = rows 1, 3, 5, 7 (byte j =
// row 2j resp. 2j+1).  `pairs` is the group's 16-bit pair word spread as bytes
// [p0, p0, p1, p1] (spread_pairs).
__device__ __forceinline__ uint32_t spread_pairs(uint32_t w32, bool high_half) {
    return __byte_perm(w32, 0u, high_half ? 0x3322u : 0x1100u);
}

template <int BITS>
__device__ __forceinline__ void unpack_group(uint32_t nib, uint32_t pairs, uint32_t &lo, uint32_t &hi) {
    static_assert(BITS == 4 || BITS == 6, "packed widths");
    if (BITS == 4) {
        lo = (nib << 4) & 0xF0F0F0F0u;
        hi = nib & 0xF0F0F0F0u;
    } else {
        lo = ((nib << 2) & 0x3C3C3C3Cu) | ((pairs << 6) & 0x00C000C0u) | ((pairs << 2) & 0xC000C000u);
        hi = ((nib >> 2) & 0x3C3C3C3Cu) | ((pairs << 4) & 0x00C000C0u) | (pairs & 0xC000C000u);
    }
}

// Code of key row i, column c in a packed plane set (any width; 8 = code_off_t).
__device__ __forceinline__ int packed_code(const unsigned char *codes, int c, int i, int dk, int dv, int bits) {
    if (bits == 8) return (int)(int8_t)codes[code_off_t(c, i, dk)];
    const int g = i >> 3, k = i & 7;
    const uint32_t nib = (codes[nib_off(c, g, dk) + (k >> 1)] >> (4 * (k & 1))) & 15u;
    if (bits == 4) return ((int)(nib << 28)) >> 28;
    const uint32_t pr = (*reinterpret_cast<const uint16_t *>(codes + pair_off(c, g, dk, dv)) >> (2 * k)) & 3u;
    return ((int)((nib | (pr << 4)) << 26)) >> 26;
}

// One step of the decay guard (see the record layout): from the step's decay
// a and the carried G_{t-1} in [2^-64, 1], the new G_t and the factor rho
// applied to the buffered entries' key side and to sigma -- 1, 2^-64 (an
// exact rescaling) or 0 (a restart).  a * 2^64 and the rescaled product are
// exact scalings of a and of the in-range product.  NaN and negative decays
// take the plain product (they reach the outputs and the status word).
__host__ __device__ __forceinline__ float gate_chain(float a, float gp, float &rho) {
    float g = a * gp;
    rho = 1.0f;
    if (g >= 0.0f && g < 0x1p-64f) {
        const float g2 = (a * 0x1p64f) * gp;
        if (g2 >= 0x1p-64f) {
            g = g2;
            rho = 0x1p-64f;
        } else {
            g = 1.0f;
            rho = 0.0f;
        }
    }
    return g;
}

// Named barrier over the NT compute threads (warps 0 .. NT/32-1) of a CTA;
// with an NT-thread CTA it is a full barrier, with extra warps it leaves them
// out.
template <int NT = kThreads>
__device__ __forceinline__ void cbar() { asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory"); }

// ---------------------------------------------------------------------------
// PTX wrappers: mbarrier + cp.async.bulk (global -> shared, no multicast).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of `bar` for at most ~limit_ns.  On a timeout, raise
// the status bit, then keep waiting (again bounded) so that the copy in flight
// lands before the caller's shared memory is released, and report failure.
__device__ inline bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, int *status,
                                         uint64_t limit_ns = 1000000000ull) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > limit_ns) {
            if (status) atomicOr(status, kStatusTimeout);
            uint64_t t1 = global_ns();
            while (!mbar_try_wait(bar, parity)) {
                if (global_ns() - t1 > 4 * limit_ns) break;
            }
            return false;
        }
    }
    return true;
}

// ---------------------------------------------------------------------------
// Reductions.
// ---------------------------------------------------------------------------
template <int WIDTH>
__device__ __forceinline__ float shfl_xor_sum(float v) {
#pragma unroll
    for (int m = WIDTH / 2; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}

__device__ __forceinline__ float warp_sum(float v) { return shfl_xor_sum<32>(v); }

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}

// Transpose-reduce of V values per lane over the lanes that differ in bits
// HI, HI/2, ..., LO (powers of two, LO <= HI <= 16).  At each of the first
// log2(V) bits a lane keeps one half of its list and adds the other half,
// received from its partner -- V/2 + V/4 + ... shuffles instead of V per bit;
// any further bits are plain butterflies on the one value left.  Afterwards
// v[0 .. V >> S) (S = the number of halving bits) hold the totals of the
// entries xpose_base<V, HI, LO>(lane) + j.
template <int HI, int LO>
__host__ __device__ constexpr int xpose_bits() {
    return HI < LO ? 0 : 1 + xpose_bits<HI / 2, LO>();
}

template <int V>
__host__ __device__ constexpr int ilog2() {
    return V <= 1 ? 0 : 1 + ilog2<V / 2>();
}

template <bool MAX, typename F>
__device__ __forceinline__ F xpose_op(F a, F b) {
    if constexpr (MAX) return fmax(a, b);   // fmaxf / fmax: a NaN operand is ignored
    else return a + b;
}

template <int V, int HI, int LO, bool MAX = false, typename F>
__device__ __forceinline__ void xpose_reduce(F (&v)[V]) {
    const int lane = threadIdx.x & 31;
    constexpr int L = xpose_bits<HI, LO>();
#pragma unroll
    for (int l = 0; l < L; ++l) {
        const int m = HI >> l;
        const int n = V >> l;   // values still held before this bit
        if (n > 1) {
            const bool up = (lane & m) != 0;
#pragma unroll
            for (int i = 0; i < V / 2; ++i) {
                if (i < n / 2) {
                    const F send = up ? v[i] : v[i + n / 2];
                    const F keep = up ? v[i + n / 2] : v[i];
                    v[i] = xpose_op<MAX>(keep, __shfl_xor_sync(0xffffffffu, send, m));
                }
            }
        } else {
            v[0] = xpose_op<MAX>(v[0], __shfl_xor_sync(0xffffffffu, v[0], m));
        }
    }
}

template <int V, int HI, int LO>
__device__ __forceinline__ int xpose_base(int lane) {
    constexpr int S = ilog2<V>() < xpose_bits<HI, LO>() ? ilog2<V>() : xpose_bits<HI, LO>();
    int b = 0;
#pragma unroll
    for (int l = 0; l < S; ++l)
        if (lane & (HI >> l)) b += V >> (l + 1);
    return b;
}

// All-reduce of V values over the lanes differing in bits HI..LO, with
// V <= 2^(number of bits): a transpose-reduce, then every lane gathers the V
// totals (V shuffles).
template <int V, int HI, int LO, typename F>
__device__ __forceinline__ void xpose_allreduce(F (&v)[V]) {
    static_assert(ilog2<V>() <= xpose_bits<HI, LO>(), "more values than lanes");
    const int lane = threadIdx.x & 31;
    xpose_reduce<V, HI, LO>(v);
    const F mine = v[0];
    constexpr int ALL = 2 * HI - LO;   // bits HI..LO
#pragma unroll
    for (int i = 0; i < V; ++i) {
        int src = lane & ~ALL;
#pragma unroll
        for (int l = 0; l < ilog2<V>(); ++l)
            if (i & (V >> (l + 1))) src |= HI >> l;
        v[i] = __shfl_sync(0xffffffffu, mine, src);
    }
}

// ---------------------------------------------------------------------------
// Correctly rounded a / b from a precomputed y = RN(1/b), three operations:
//   q = RN(a y);  r = a - b q (exact, one FMA);  q' = RN(q + r y).
// Markstein's correction step (P. Markstein, IBM J. Res. Dev. 34(1), 1990;
// also Muller et al., Handbook of Floating-Point Arithmetic, section on
// FMA-based division): q' is the IEEE quotient whenever the residual r is
// exact, i.e. away from the subnormal range.  The guard keeps a, q' and y
// well inside the normal range (|a|, |q'| >= 2^-100, |q'| <= 2^126,
// b <= 2^100); everything else -- zeros included -- takes the IEEE division.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool div_fast_ok(float a, float q, float b) {
    return fabsf(a) >= 0x1p-100f && fabsf(q) >= 0x1p-100f && fabsf(q) <= 0x1p126f && b <= 0x1p100f;
}

// The three operations alone, for callers that have established the range.
__device__ __forceinline__ float div_rn_unchecked(float a, float b, float y) {
    const float q = __fmul_rn(a, y);
    const float r = __fmaf_rn(-q, b, a);
    return __fmaf_rn(r, y, q);
}

__device__ __forceinline__ float div_rn(float a, float b, float y) {
    const float q2 = div_rn_unchecked(a, b, y);
    return div_fast_ok(a, q2, b) ? q2 : __fdiv_rn(a, b);
}

// Two FP32 fused multiply-adds per instruction (sm_100 packed FP32).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// div_rn on a pair of dividends sharing the divisor.
__device__ __forceinline__ float2 div2_rn_unchecked(float2 a, float b, float y) {
    const float2 q = __fmul2_rn(a, f2(y, y));
    const float2 r = __ffma2_rn(q, f2(-b, -b), a);
    return __ffma2_rn(r, f2(y, y), q);
}

__device__ __forceinline__ float2 div2_rn(float2 a, float b, float y) {
    float2 q2 = div2_rn_unchecked(a, b, y);
    if (!div_fast_ok(a.x, q2.x, b)) q2.x = __fdiv_rn(a.x, b);
    if (!div_fast_ok(a.y, q2.y, b)) q2.y = __fdiv_rn(a.y, b);
    return q2;
}

// Sum of one double per compute thread (warps 0..7); every compute thread
// gets the result.  `scratch` holds kWarps doubles; two barriers inside.
__device__ inline double block_sum_d(double v, double *scratch) {
    v = warp_sum_d(v);
    cbar();
    if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
    cbar();
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += scratch[w];
    return s;
}

// ---------------------------------------------------------------------------
// BF16 round-to-nearest-even from float bits, and back.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint16_t bf16_rne(float x) {
    uint32_t u = __float_as_uint(x);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x0040u);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

__device__ __forceinline__ float bf16_to_f(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }
__device__ __forceinline__ float4 bf16x4_to_f4(uint2 w) {
    return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u), __uint_as_float(w.y << 16),
                       __uint_as_float(w.y & 0xffff0000u));
}
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
// x rounded to BF16 (nearest even), as an FP32 value
__device__ __forceinline__ float bf16_round(float x) { return bf16_to_f(bf16_rne(x)); }

// Signed bytes of a 32-bit word -> floats (exact).  Each byte, offset to
// unsigned, is placed in the low mantissa byte of 2^23 (bit pattern
// 0x4B0000xx) with one byte permute, and 2^23 + 128 is subtracted: the
// integer-to-float bias trick, two ALU operations per value instead of a
// conversion instruction.
__device__ __forceinline__ void s8x4_to_f(uint32_t w, float f[4]) {
    const uint32_t u = w ^ 0x80808080u;
    f[0] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540u)) - 8388736.0f;
    f[1] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541u)) - 8388736.0f;
    f[2] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542u)) - 8388736.0f;
    f[3] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543u)) - 8388736.0f;
}

// Build the key-row map of one head in shared memory: map[i] = INT8 slot of
// row i (rows in increasing order, BF16 rows skipped) or -1-p for the p-th
// BF16 row.  Run by the NT compute threads; needs DK <= NT.  Ends with a
// barrier over them.
template <int DK, int NT = kThreads>
__device__ inline void build_row_map(const int *hp_rows_h, int P, int *map, int *scratch_w) {
    static_assert(DK <= NT, "one thread per key row");
    const int i = threadIdx.x;
    int p_of = -1;
    if (i < DK) {
        for (int p = 0; p < P; ++p)
            if (hp_rows_h[p] == i) p_of = p;
    }
    const bool hp = (i < DK) && (p_of >= 0);
    const uint32_t bal = __ballot_sync(0xffffffffu, hp);
    const int lane = i & 31, warp = i >> 5;
    if (lane == 0) scratch_w[warp] = __popc(bal);
    cbar<NT>();
    int before = __popc(bal & ((1u << lane) - 1u));
    for (int w = 0; w < warp; ++w) before += scratch_w[w];
    if (i < DK) map[i] = hp ? (-1 - p_of) : (i - before);
    cbar<NT>();
}

}  // namespace lq
