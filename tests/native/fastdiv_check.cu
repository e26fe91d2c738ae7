// Host-side check of make_fastdiv (csrc/sm100_ptx.cuh): for the magic numbers it sets, the
// kernel's quotient (umulhi(n, m) + n) >> l, taken in 32-bit arithmetic, equals n / d for every
// 31-bit dividend n. Exhaustive over all n < 2^31 for the divisors given as arguments;
// boundary and sampled dividends for every divisor 1 .. 5000 and some large ones.
// Build: nvcc -O2 -std=c++17 -o fastdiv_check fastdiv_check.cu   (runs on the CPU)
#include <cstdio>
#include <cstdlib>

#include "../../head_attention_forward_flash_b200/csrc/sm100_ptx.cuh"

static uint32_t quotient(uint32_t n, const b200::FastDiv& f)
{
    const uint32_t hi = (uint32_t)(((uint64_t)n * f.m) >> 32);  // umulhi
    return (uint32_t)(hi + n) >> f.l;                            // 32-bit add, as on the GPU
}

static int check(uint32_t d, uint32_t n, const b200::FastDiv& f)
{
    if (quotient(n, f) != n / d) {
        std::printf("FAIL d=%u n=%u got %u want %u\n", d, n, quotient(n, f), n / d);
        return 1;
    }
    return 0;
}

int main(int argc, char** argv)
{
    const uint32_t top = 0x7FFFFFFFu;
    int bad = 0;
    for (int a = 1; a < argc; ++a) {  // exhaustive
        const uint32_t d = (uint32_t)std::strtoul(argv[a], nullptr, 10);
        const b200::FastDiv f = b200::make_fastdiv(d);
        for (uint32_t n = 0;; ++n) {
            bad += check(d, n, f);
            if (bad > 10) return 1;
            if (n == top) break;
        }
    }
    uint64_t state = 88172645463325252ull;
    const uint32_t large[] = {65535u, 65536u, 65537u, 1000003u, 1u << 20, (1u << 30) + 1, top};
    for (uint32_t i = 0; i < 5000 + sizeof(large) / sizeof(large[0]); ++i) {
        const uint32_t d = i < 5000 ? i + 1 : large[i - 5000];
        const b200::FastDiv f = b200::make_fastdiv(d);
        for (uint32_t n = 0; n < 20000; ++n) bad += check(d, n, f);
        for (uint64_t k = top / d; k + 2 > top / d && k > 0; --k) {  // multiples near 2^31
            for (int e = -1; e <= 1; ++e) {
                const uint64_t n = k * d + e;
                if (n <= top) bad += check(d, (uint32_t)n, f);
            }
            if (top / d - k > 64) break;
        }
        for (int r = 0; r < 20000; ++r) {
            state ^= state << 13; state ^= state >> 7; state ^= state << 17;
            bad += check(d, (uint32_t)(state & top), f);
        }
        if (bad > 10) return 1;
    }
    std::printf(bad ? "FAILED\n" : "ok\n");
    return bad ? 1 : 0;
}
