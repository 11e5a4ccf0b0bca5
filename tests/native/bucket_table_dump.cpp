// Prints the write kernels' bucket tables for every supported (d, b), for the
// CPU test that checks them against the codebook boundaries
// (tests/test_bucket_table.py).  Host code only: built with a C++ compiler
// against lut_attention_b200/csrc/codebook.cpp.
//
// Output, per (d, b):  "table d b nt g_scale g_off margin", then nt lines
// "tau base" (tau as a hexadecimal float; inf where the bucket holds no boundary).
#include <cstdio>

#include "axr_internal.cuh"

int main()
{
    for (int d = 8; d <= 512; d *= 2) {
        for (int b = 1; b <= 4; ++b) {
            axr::BucketTable t;
            if (!axr::get_bucket_table(d, b, &t)) {
                std::printf("missing %d %d\n", d, b);
                return 1;
            }
            std::printf("table %d %d %d %a %a %a\n", d, b, t.nt, t.g_scale, t.g_off, t.margin);
            for (int j = 0; j < t.nt; ++j) std::printf("%a %d\n", t.tau[j], t.base[j]);
        }
    }
    return 0;
}
