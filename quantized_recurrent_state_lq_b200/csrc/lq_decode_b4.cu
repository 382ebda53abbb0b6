// lq_decode_b4.cu -- the decode kernels for 4-bit window-start codes.
#include "lq_decode.cuh"

namespace lq {

cudaError_t launch_decode_b4(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool flush, bool damp,
                              cudaStream_t s) {
    return DecodeSet<4>::decode(a, dk, dv, heads, kda, flush, damp, s);
}

cudaError_t launch_flush_b4(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool damp, bool exp,
                             cudaStream_t s) {
    return DecodeSet<4>::flush_only(a, dk, dv, heads, kda, damp, exp, s);
}

}  // namespace lq
