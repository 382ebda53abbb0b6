// Host program for tests/test_layout_cpu.py: prints the packed-code offsets of
// the library's header (nib_off, pair_off, lowbit_kslot, chunk_swz) for one
// head shape, one table per line.  Uses host-callable helpers only.
#include <cstdio>
#include <cstdlib>

#include "../quantized_recurrent_state_lq_b200/csrc/lq_common.cuh"

int main(int argc, char **argv) {
    const int dk = atoi(argv[1]), dv = atoi(argv[2]);
    printf("nib");
    for (int c = 0; c < dv; ++c)
        for (int g = 0; g < dk / 8; ++g) printf(" %d", lq::nib_off(c, g, dk));
    printf("\npair");
    for (int c = 0; c < dv; ++c)
        for (int g = 0; g < dk / 8; ++g) printf(" %d", lq::pair_off(c, g, dk, dv));
    printf("\nkslot");
    for (int i = 0; i < dk; ++i) printf(" %d", lq::lowbit_kslot(i));
    printf("\nswz");
    for (int c = 0; c < dv; ++c) printf(" %d %d", lq::chunk_swz(c, dk / 2), lq::chunk_swz(c, dk / 4));
    printf("\n");
    return 0;
}
