// Host check of the bit -> bf16x2 lane-mask expansion used by the kernels
// (masked_glu_b200/csrc/common.cuh).  For every n_m, register Q and mask I it
// compares pair_mask against the packed-format definition: bit (w*n_m + i) of
// an 8-weight chunk is mask i of weight w.  Prints "ok" and exits 0 on success.
#include <cstdint>
#include <cstdio>
#include <random>

#include "common.cuh"

template <int NM, int Q, int I>
static int check_one(uint32_t lo, uint32_t hi)
{
    const uint64_t bits = (uint64_t)lo | ((uint64_t)hi << 32);
    const uint32_t b0 = (uint32_t)(bits >> ((2 * Q) * NM + I)) & 1u;
    const uint32_t b1 = (uint32_t)(bits >> ((2 * Q + 1) * NM + I)) & 1u;
    const uint32_t want = (b0 ? 0x0000FFFFu : 0u) | (b1 ? 0xFFFF0000u : 0u);
    const uint32_t got = mglu::pair_mask<NM, Q, I>(lo, hi);
    if (got != want) {
        std::printf("mismatch NM=%d Q=%d I=%d lo=%08x hi=%08x got=%08x want=%08x\n", NM, Q, I, lo, hi, got, want);
        return 1;
    }
    return 0;
}

template <int NM, int Q, int I>
struct Loop {
    static int run(uint32_t lo, uint32_t hi)
    {
        int bad = check_one<NM, Q, I>(lo, hi);
        if constexpr (I + 1 < NM)
            bad += Loop<NM, Q, I + 1>::run(lo, hi);
        else if constexpr (Q + 1 < 4)
            bad += Loop<NM, Q + 1, 0>::run(lo, hi);
        return bad;
    }
};

template <int NM>
static int check_nm(std::mt19937_64 &rng)
{
    const int nbits = 8 * NM;
    const uint64_t keep = nbits == 64 ? ~0ull : ((1ull << nbits) - 1);
    int bad = 0;
    // every single-bit pattern, its complement, then random patterns
    for (int b = 0; b < nbits; ++b) {
        const uint64_t v = 1ull << b;
        bad += Loop<NM, 0, 0>::run((uint32_t)v, (uint32_t)(v >> 32));
        const uint64_t c = ~v & keep;
        bad += Loop<NM, 0, 0>::run((uint32_t)c, (uint32_t)(c >> 32));
    }
    for (int n = 0; n < 20000; ++n) {
        const uint64_t v = rng() & keep;
        bad += Loop<NM, 0, 0>::run((uint32_t)v, (uint32_t)(v >> 32));
    }
    return bad;
}

int main()
{
    std::mt19937_64 rng(12345);
    int bad = check_nm<1>(rng) + check_nm<2>(rng) + check_nm<4>(rng) + check_nm<8>(rng);
    if (bad) {
        std::printf("%d mismatches\n", bad);
        return 1;
    }
    std::printf("ok\n");
    return 0;
}
