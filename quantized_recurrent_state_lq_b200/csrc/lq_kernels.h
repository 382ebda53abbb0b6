// lq_kernels.h -- internal launch interface between the C ABI (lq_api.cu) and
// the kernels.  Not installed; the public interface is include/lq_state.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "lq_common.cuh"

namespace lq {

struct DecodeArgs {
    Layout L;
    unsigned char *rec;   // records of all heads
    int B, H, Hk, K, smoothing, n;
    const float *q, *k, *v, *beta, *alpha;
    float *o;
    const int *hp_rows;   // [H][P] (device)
    const int *slot_rows; // [H][dk] (device): key row of INT8 slot j, then of BF16 row p
    int *status;
    float *S_out;         // export target [heads][dk][dv]
    // Window phases (staggered windows): batch entry b ends its windows at the
    // steps where (since + phase[b]) mod W = W - 1, since counting the steps
    // from the last common window start; it then holds
    // min((since + phase[b]) mod W, since) buffered tokens.  With phases, n is
    // min(since, W) and nmod is since mod W; without (phase null) every entry
    // holds n tokens.
    const int *phase;       // [B] (device) or null
    const int *flush_list;  // flush launches: the batch entries of the grid, H CTAs each (null: all heads)
    int nmod;
};

struct Fp32Args {
    float *S;             // [heads][dk][dv]
    int B, H, Hk;
    const float *q, *k, *v, *beta, *alpha;
    float *o;
    int *status;
};

// A quantized state addressed per head: base pointers plus per-head strides in
// BYTES, and per-compensator strides in floats.  Serves both the workspace
// record layout and the plain lq_qstate_view arrays.
struct QPtrs {
    unsigned char *codes; size_t codes_hs;
    int codes_t;                                    // 1: column-major swizzled (record, no BF16 rows;
                                                    //    4 / 6-bit codes packed, CodecArgs::bits)
    unsigned char *hp;    size_t hp_hs;
    unsigned char *m;     size_t m_hs;
    unsigned char *s;     size_t s_hs;
    unsigned char *ck;    size_t ck_hs; int ck_js;
    unsigned char *cw;    size_t cw_hs; int cw_js;
    unsigned char *gam;   size_t gam_hs; int gam_n;   // decay guard (G, sigma): set to 1 after writing (may be null)
};

struct CodecArgs {
    int H, r, K, smoothing, P;
    int bits;             // code width: 8, 6 or 4 (the quantizer's qmax; packing of codes_t stores)
    const float *static_ms;   // smoothing 2: per head h, key-row then value-column scales [H][dk+dv]
    const int *hp_rows;   // [H][P] (device), may be null when P == 0
    const float *S_in;    // [heads][dk][dv]
    float *S_out;         // [heads][dk][dv]
    QPtrs q;              // destination (quantize) or source (dequantize)
    QPtrs q2;             // second target for copies (view <-> record)
    int *status;
    // DAMP selection and the static-scale fit's row weights
    int n_states, n_gate_samples, gate_per_channel;
    const float *gates;   // [n_gate_samples][H][1 or dk]
    double *energy;       // [H][dk]
    int *rows_out;        // [H][P]
};

size_t decode_smem_bytes(int dk, int dv, const Layout &L);
size_t buffer_smem_bytes_of(int dk, int dv, const Layout &L);
size_t flush_smem_bytes_of(int dk, int dv, const Layout &L);
// Per code width (L.bits): launch_decode / launch_flush dispatch to these.
cudaError_t launch_decode_b8(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool flush, bool damp,
                             cudaStream_t s);
cudaError_t launch_decode_b6(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool flush, bool damp,
                             cudaStream_t s);
cudaError_t launch_decode_b4(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool flush, bool damp,
                             cudaStream_t s);
cudaError_t launch_flush_b8(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool damp, bool exp,
                            cudaStream_t s);
cudaError_t launch_flush_b6(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool damp, bool exp,
                            cudaStream_t s);
cudaError_t launch_flush_b4(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool damp, bool exp,
                            cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool flush, bool damp,
                          cudaStream_t s);
cudaError_t launch_flush(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool damp, bool exp,
                         cudaStream_t s);
cudaError_t launch_fp32_step(const Fp32Args &a, int dk, int dv, int heads, bool kda, cudaStream_t s);

cudaError_t launch_quantize(const CodecArgs &a, int dk, int dv, int heads, cudaStream_t s);
cudaError_t launch_dequantize(const CodecArgs &a, int dk, int dv, int heads, cudaStream_t s);
cudaError_t launch_qcopy(const CodecArgs &a, int dk, int dv, int heads, cudaStream_t s);
cudaError_t launch_damp_select(const CodecArgs &a, int dk, int dv, cudaStream_t s);
cudaError_t launch_fit_static(const CodecArgs &a, int dk, int dv, int n, float *m, float *sc, cudaStream_t s);

cudaError_t launch_div_selftest(const float *a, const float *b, float *fast, float *pair, float *ieee, int n,
                                cudaStream_t s);
cudaError_t launch_wait_selftest(const unsigned char *src, int *status, unsigned long long limit_ns,
                                 cudaStream_t s);

}  // namespace lq
