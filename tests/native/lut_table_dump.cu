// Prints the read kernels' lookup table (lut_read.cuh, build_lut) for
// b = 1, 2, 3, 4, built with the thread count given on the command line from
// fixed test digits hi[i] = 7 i - 50, lo[i] = 100 + i: one line per b, the
// 65536 table bytes in hex.  Host code only; built by tests/test_lut_table.py.
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "lut_read.cuh"

template <int B>
static void dump(int nthreads)
{
    alignas(16) static uint8_t lut[axr::lut::kLutBytes];
    std::memset(lut, 0, sizeof(lut));
    int8_t hi[axr::kMaxLevels], lo[axr::kMaxLevels];
    for (int i = 0; i < axr::kMaxLevels; ++i) {
        hi[i] = static_cast<int8_t>(7 * i - 50);
        lo[i] = static_cast<int8_t>(100 + i);
    }
    for (int tid = 0; tid < nthreads; ++tid) axr::lut::build_lut<B>(hi, lo, lut, tid, nthreads);
    for (int i = 0; i < axr::lut::kLutBytes; ++i) std::printf("%02x", lut[i]);
    std::printf("\n");
}

int main(int argc, char **argv)
{
    const int nthreads = argc > 1 ? std::atoi(argv[1]) : 512;
    dump<1>(nthreads);
    dump<2>(nthreads);
    dump<3>(nthreads);
    dump<4>(nthreads);
    return 0;
}
