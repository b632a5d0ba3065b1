// Prints the tensor-core state layouts (tc_layout.cuh, compiled for the host):
// for G = 1 and G = 2 factors, one line "R<G> r i j" per state row, then one
// line "P<G> i j r" per pair i <= j that the layout holds.
#include <cstdio>

#include "tc_layout.cuh"

int main() {
    using namespace kata::tc;
    for (int G = 1; G <= 2; ++G) {
        for (int r = 0; r < state_rows(G); ++r) {
            const PairIJ p = row_ij_g(G, r);
            std::printf("R%d %d %d %d\n", G, r, p.i, p.j);
        }
        for (int i = 0; i < kD; ++i)
            for (int j = i; j < kD; ++j)
                if (same_factor(G, i, j)) std::printf("P%d %d %d %d\n", G, i, j, row_index_g(G, i, j));
    }
    return 0;
}
