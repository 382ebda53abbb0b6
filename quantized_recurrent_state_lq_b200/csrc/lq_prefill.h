// lq_prefill.h -- internal launch interface of the chunked prefill
// (lq_prefill.cu), used by the C ABI (lq_api.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace lq {

struct PrefillArgs {
    int B, H, Hk, T;
    const float *q, *k, *v, *beta, *alpha;   // token-major, as a decode step's inputs x T
    const float *S0;      // [heads][dk][dv] or null (zero state)
    float *S_out;         // [heads][dk][dv] (may be S0)
    float *o;             // [T][B][H][dv] or null
    int *status;          // sticky status word or null
};

cudaError_t launch_prefill(const PrefillArgs &a, int dk, int dv, int heads, bool kda, cudaStream_t s);
size_t prefill_smem_bytes(int dk, int dv, bool kda);

}  // namespace lq
