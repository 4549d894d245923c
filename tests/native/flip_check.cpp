// Host check of the sign-flip operand construction used by the decode kernel
// (masked_glu_b200/csrc/common.cuh: group_bits, flip_pair).  For every n_m,
// k16 group S, weight pair p and mask I, it shifts group_bits as the kernel
// does (left by 15 - I for the pair (4S, 4S+1); right by 8, then left by
// 15 - I, for (4S+2, 4S+3)) and checks that bits 15 and 31 are mask I of the pair's two weights as the
// packed format defines them (bit w*n_m + i of an 8-weight chunk is mask i
// of weight w), and that flip_pair negates exactly the weights whose bit is
// clear.  Prints "ok" and exits 0 on success.
#include <cstdint>
#include <cstdio>
#include <random>

#include "common.cuh"

template <int NM, int S>
static int check_group(uint32_t lo, uint32_t hi, uint32_t w)
{
    const uint64_t bits = (uint64_t)lo | ((uint64_t)hi << 32);
    const uint32_t r = mglu::group_bits<NM, S>(lo, hi);
    int bad = 0;
    for (int p = 0; p < 2; ++p)
        for (int I = 0; I < NM; ++I) {
            const uint32_t m = (p == 0 ? r : r >> 8) << (15 - I);
            const int w0 = 4 * S + 2 * p, w1 = w0 + 1;
            const uint32_t b0 = (uint32_t)(bits >> (w0 * NM + I)) & 1u;
            const uint32_t b1 = (uint32_t)(bits >> (w1 * NM + I)) & 1u;
            if (((m >> 15) & 1u) != b0 || ((m >> 31) & 1u) != b1) {
                std::printf("bit mismatch NM=%d S=%d p=%d I=%d lo=%08x hi=%08x\n", NM, S, p, I, lo, hi);
                ++bad;
            }
            const uint32_t want = w ^ (b0 ? 0u : 0x00008000u) ^ (b1 ? 0u : 0x80000000u);
            if (mglu::flip_pair(w, m) != want) {
                std::printf("flip mismatch NM=%d S=%d p=%d I=%d\n", NM, S, p, I);
                ++bad;
            }
        }
    return bad;
}

template <int NM>
static int check_nm(std::mt19937_64 &rng)
{
    int bad = 0;
    for (int it = 0; it < 200000 && bad == 0; ++it) {
        const uint64_t v = rng();
        // only the chunk's 8 * NM bits exist; the rest of the words are zero
        const uint64_t chunk = NM == 8 ? v : (v & ((1ull << (8 * NM)) - 1));
        const uint32_t lo = (uint32_t)chunk, hi = (uint32_t)(chunk >> 32);
        const uint32_t w = (uint32_t)rng();
        bad += check_group<NM, 0>(lo, hi, w) + check_group<NM, 1>(lo, hi, w);
    }
    return bad;
}

int main()
{
    std::mt19937_64 rng(12345);
    const int bad = check_nm<1>(rng) + check_nm<2>(rng) + check_nm<4>(rng) + check_nm<8>(rng);
    if (bad) {
        std::printf("%d mismatches\n", bad);
        return 1;
    }
    std::printf("ok\n");
    return 0;
}
