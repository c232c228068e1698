// Independent Philox4x32-10 reference for the oracle's pin: PyTorch's
// header-only at::philox_engine (ATen/core/PhiloxRNGEngine.h).  Its key is the
// 64-bit seed, its counter is (offset_lo, offset_hi, subsequence_lo,
// subsequence_hi), and it returns the four words of one block in order.
// Reads lines "seed subsequence offset" (decimal) and prints the four words.
#include <ATen/core/PhiloxRNGEngine.h>
#include <cinttypes>
#include <cstdio>

int main() {
    unsigned long long seed, subseq, offset;
    while (std::scanf("%llu %llu %llu", &seed, &subseq, &offset) == 3) {
        at::philox_engine eng(seed, subseq, offset);
        uint32_t w0 = eng(), w1 = eng(), w2 = eng(), w3 = eng();
        std::printf("%u %u %u %u\n", w0, w1, w2, w3);
    }
    return 0;
}
