// Prints the tensor-core state layout (tc_layout.cuh, compiled for the host):
// one line "r i j" per state row, then one line "i j r" per pair i <= j.
#include <cstdio>

#include "tc_layout.cuh"

int main() {
    using namespace kata::tc;
    for (int r = 0; r < kStateRows; ++r) {
        const PairIJ p = row_ij(r);
        std::printf("R %d %d %d\n", r, p.i, p.j);
    }
    for (int i = 0; i < kD; ++i)
        for (int j = i; j < kD; ++j) std::printf("P %d %d %d\n", i, j, row_index(i, j));
    return 0;
}
