// Host-side anchor sampler (page "GLM 5.2 DSpark speculative-training design",
// §2 "anchor sampling", with the read-time rule of appendix A that the last
// position's loss_mask is 0, and §3 padding blocks).
#include <stdint.h>

#include <vector>

#include "../../include/dspark_attn.h"

namespace {

// SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
// generators", OOPSLA 2014): a Weyl sequence followed by a 64-bit finaliser.
struct SplitMix64 {
    uint64_t s;
    uint64_t next() {
        uint64_t z = (s += 0x9E3779B97F4A7C15ull);
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        return z ^ (z >> 31);
    }
    // uniform integer in [0, m), by the high half of a 64x64 product
    uint64_t below(uint64_t m) { return (uint64_t)(((unsigned __int128)next() * m) >> 64); }
};

}  // namespace

extern "C" int64_t dspark_sample_anchors(const uint8_t *loss_mask, int32_t B, int32_t S, int32_t N, uint64_t seed,
                                         int32_t *anchors_out, uint8_t *keep_out) {
    if (B < 0 || S < 1 || N < 0) return -1;
    if ((int64_t)B * N > 0 && (!anchors_out || !keep_out)) return -1;
    if ((int64_t)B * S > 0 && !loss_mask) return -1;
    int64_t kept = 0;
    std::vector<int32_t> cand;
    for (int32_t b = 0; b < B; b++) {
        const uint8_t *lm = loss_mask + (size_t)b * S;
        cand.clear();
        for (int32_t a = 0; a <= S - 2; a++) {
            const uint8_t next = (a + 1 == S - 1) ? 0 : lm[a + 1];
            if (lm[a] && next) cand.push_back(a);
        }
        SplitMix64 rng{seed + (uint64_t)b};
        const int32_t take = (int32_t)cand.size() < N ? (int32_t)cand.size() : N;
        for (int32_t i = 0; i < take; i++) {
            const uint64_t j = i + rng.below((uint64_t)cand.size() - i);
            const int32_t t = cand[i];
            cand[i] = cand[j];
            cand[j] = t;
            anchors_out[(size_t)b * N + i] = cand[i];
            keep_out[(size_t)b * N + i] = 1;
        }
        for (int32_t i = take; i < N; i++) {
            anchors_out[(size_t)b * N + i] = 0;
            keep_out[(size_t)b * N + i] = 0;
        }
        kept += take;
    }
    return kept;
}
