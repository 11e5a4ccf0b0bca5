// Prints the read kernels' balanced tile ranges for the shapes given on the
// command line (total_tiles tiles_per_head ctas change_cost ...), one line each:
// the ctas + 1 range starts.  Host code only; built by tests/test_tile_ranges.py.
#include <cstdio>
#include <cstdlib>

#include "lut_read.cuh"

int main(int argc, char **argv)
{
    for (int i = 1; i + 3 < argc; i += 4) {
        const int total = std::atoi(argv[i]), tph = std::atoi(argv[i + 1]);
        const int ctas = std::atoi(argv[i + 2]), cc = std::atoi(argv[i + 3]);
        int starts[axr::lut::kMaxCtas + 1];
        axr::lut::balanced_ranges(total, tph, ctas, cc, starts);
        for (int c = 0; c <= ctas; ++c) std::printf("%d%c", starts[c], c == ctas ? '\n' : ' ');
    }
    return 0;
}
