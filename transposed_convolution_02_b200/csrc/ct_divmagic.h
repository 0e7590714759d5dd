// Division by a run-time invariant through a multiply (Granlund and
// Montgomery, "Division by invariant integers using multiplication", 1994):
// with l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1,
// floor(t / d) = (umulhi(t, m) + t) >> l for every 0 <= t < 2^31.
#pragma once

#include <stdint.h>

namespace ct {

struct DivMagic {
    uint32_t m;
    int32_t l;
};

inline DivMagic make_magic(uint32_t d) {
    int l = 0;
    while ((1ull << l) < d) ++l;
    const uint64_t m = ((1ull << 32) * ((1ull << l) - d)) / d + 1;
    return DivMagic{(uint32_t)m, l};
}

#ifdef __CUDACC__
__device__ __forceinline__ int divq(int t, DivMagic d) {
    return (int)((__umulhi((uint32_t)t, d.m) + (uint32_t)t) >> d.l);
}
#endif

}  // namespace ct
