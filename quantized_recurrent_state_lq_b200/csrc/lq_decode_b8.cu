// lq_decode_b8.cu -- the decode kernels for 8-bit window-start codes.
#include "lq_decode.cuh"

namespace lq {

cudaError_t launch_decode_b8(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool flush, bool damp,
                              cudaStream_t s) {
    return DecodeSet<8>::decode(a, dk, dv, heads, kda, flush, damp, s);
}

cudaError_t launch_flush_b8(const DecodeArgs &a, int dk, int dv, int heads, bool kda, bool damp, bool exp,
                             cudaStream_t s) {
    return DecodeSet<8>::flush_only(a, dk, dv, heads, kda, damp, exp, s);
}

size_t buffer_smem_bytes_of(int dk, int dv, const Layout &L) { return buffer_smem_bytes(dk, dv, L); }
size_t flush_smem_bytes_of(int dk, int dv, const Layout &L) { return flush_smem_bytes(dk, dv, L); }

}  // namespace lq
