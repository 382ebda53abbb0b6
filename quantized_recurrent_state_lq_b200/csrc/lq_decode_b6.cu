// lq_decode_b6.cu -- the decode kernels for 6-bit window-start codes.
#include "lq_decode.cuh"

namespace lq {

cudaError_t launch_decode_b6(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool flush, bool damp,
                              cudaStream_t s) {
    return DecodeSet<6>::decode(a, dk, dv, heads, kda, flush, damp, s);
}

cudaError_t launch_flush_b6(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool damp, bool exp,
                             cudaStream_t s) {
    return DecodeSet<6>::flush_only(a, dk, dv, heads, kda, damp, exp, s);
}

}  // namespace lq
