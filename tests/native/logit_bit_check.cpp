// Host dump of the FP16 mask-logit bit rule (masked_glu_b200/csrc/common.cuh:
// logit_bit) for all 65536 binary16 bit patterns, as 65536 characters '0' /
// '1'; the test compares them with numpy's float16 comparison logit > 0.
#include <cstdio>

#include "common.cuh"

int main()
{
    for (unsigned b = 0; b < 65536u; ++b)
        std::putchar(mglu::logit_bit(b) ? '1' : '0');
    std::putchar('\n');
    return 0;
}
