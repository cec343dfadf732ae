// Independent Philox4x32-10 reference for the oracle's pin: torch's header-only
// at::philox_engine.  Reads lines "key_lo key_hi c0 c1 c2 c3" (decimal) on
// stdin and prints the four output words of one 10-round block for each.
#include <ATen/core/PhiloxRNGEngine.h>
#include <cstdio>
#include <cstdint>

int main() {
    unsigned long long klo, khi, c0, c1, c2, c3;
    while (std::scanf("%llu %llu %llu %llu %llu %llu", &klo, &khi, &c0, &c1, &c2, &c3) == 6) {
        uint64_t seed = (uint64_t)klo | ((uint64_t)khi << 32);
        uint64_t subsequence = (uint64_t)c2 | ((uint64_t)c3 << 32);
        at::philox_engine e(seed, subsequence, 0);
        e.set_offset((uint64_t)c0 | ((uint64_t)c1 << 32));  // counter words 0,1
        uint32_t w0 = e(), w1 = e(), w2 = e(), w3 = e();
        std::printf("%u %u %u %u\n", w0, w1, w2, w3);
    }
    return 0;
}
