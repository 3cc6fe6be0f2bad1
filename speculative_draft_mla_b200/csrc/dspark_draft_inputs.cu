// Draft inputs on the GPU: anchor sampling and the draft block's ids,
// positions, labels, Markov-head predecessors and eval_mask (page "GLM 5.2
// DSpark speculative-training design", §2 "anchor sampling" and "Draft block",
// §5 Markov head, §6 labels and eval_mask).
//
// Sampling. The page draws N anchors at random among the valid positions. Here
// every candidate A of batch row b gets the 64-bit key k_A = output A of
// SplitMix64 (Steele, Lea and Flood, OOPSLA 2014) started from state seed + b,
// i.e. mix(seed + b + (A + 1) * gamma), and the min(N, #candidates) candidates
// with the smallest (k_A, A) are kept: with independent keys every N-subset is
// equally likely. Unlike a shuffle this needs no sequential state, so one CTA
// per batch row finds the N-th smallest key by a radix select and compacts the
// chosen anchors in ascending order with a block-wide scan.

#include "dspark_steps.cuh"

namespace dspark {

namespace {

constexpr int kSampleThreads = 1024;

__device__ __forceinline__ uint64_t sm64_key(uint64_t seed_b, int a) {
    uint64_t z = seed_b + (uint64_t)(a + 1) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// Candidate rule of §2 with loss_mask[S-1] read as 0 (§6).
__device__ __forceinline__ bool is_candidate(const uint8_t *lm, int S, int a) {
    return a + 1 < S - 1 ? (lm[a] != 0 && lm[a + 1] != 0) : false;
}

// Keys are distinct within a batch row: the states seed + b + (A + 1) * gamma
// differ for distinct A (gamma is odd) and SplitMix64's output function is a
// bijection (xor-shifts and multiplications by odd constants). So the N chosen
// candidates are exactly those with key <= T, T the N-th smallest key. T is
// found by a radix select: an 11-bit histogram of the candidates' keys (8-bit
// digits after it while the digit holding T has more than kCollect keys), then
// the keys of that digit are collected in shared memory and ranked.
constexpr int kCollect = kSampleThreads;

__global__ void __launch_bounds__(kSampleThreads) k_sample_anchors(const uint8_t *__restrict__ loss_mask, int S,
                                                                    int N, uint64_t seed, int32_t *__restrict__ anchors,
                                                                    uint8_t *__restrict__ keep) {
    __shared__ unsigned hist[2048];
    __shared__ unsigned long long list[kCollect];
    __shared__ int warp_tot[32], s_total, s_sel[2];
    __shared__ unsigned long long s_prefix;
    const int b = blockIdx.x;
    const uint8_t *lm = loss_mask + (size_t)b * S;
    const uint64_t seed_b = seed + (uint64_t)b;
    int32_t *an = anchors + (size_t)b * N;
    uint8_t *kp = keep + (size_t)b * N;

    // number of candidates
    int local = 0;
    for (int a = threadIdx.x; a < S; a += blockDim.x) local += is_candidate(lm, S, a);
    for (int d = 16; d > 0; d >>= 1) local += __shfl_xor_sync(0xffffffffu, local, d);
    if ((threadIdx.x & 31) == 0) warp_tot[threadIdx.x >> 5] = local;
    __syncthreads();
    if (threadIdx.x == 0) {
        int c = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); w++) c += warp_tot[w];
        s_total = c;
    }
    __syncthreads();
    const int C = s_total;
    __syncthreads();

    uint64_t T = ~0ull;  // C <= N: every candidate
    if (C > N) {
        // radix select: the top `bits` bits of T are `prefix`; k = rank (1-based)
        // of T among the candidates whose keys share them
        uint64_t prefix = 0;
        int bits = 0, k = N, m = C;
        while (m > kCollect && bits < 64) {
            const int w = bits == 0 ? 11 : min(8, 64 - bits);
            const int nb = 1 << w, shift = 64 - bits - w;
            for (int i = threadIdx.x; i < nb; i += blockDim.x) hist[i] = 0;
            __syncthreads();
            for (int a = threadIdx.x; a < S; a += blockDim.x) {
                if (!is_candidate(lm, S, a)) continue;
                const uint64_t key = sm64_key(seed_b, a);
                if (bits > 0 && (key >> (64 - bits)) != prefix) continue;
                atomicAdd(&hist[(key >> shift) & (uint64_t)(nb - 1)], 1u);
            }
            __syncthreads();
            if (threadIdx.x < 32) {
                // the digit holding the k-th key: each lane sums nb / 32 bins,
                // a warp scan, then the first lane whose running count reaches k
                const int lane = threadIdx.x, per = nb / 32;
                int sum = 0;
                for (int i = 0; i < per; i++) sum += (int)hist[per * lane + i];
                int incl = sum;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, d);
                    if (lane >= d) incl += y;
                }
                const unsigned ball = __ballot_sync(0xffffffffu, incl >= k);
                const int owner = ball ? __ffs(ball) - 1 : 31;
                if (lane == owner) {
                    int acc = incl - sum, d = per * lane + per - 1;
                    for (int i = 0; i < per; i++) {
                        const int h = (int)hist[per * lane + i];
                        if (acc + h >= k) {
                            d = per * lane + i;
                            break;
                        }
                        acc += h;
                    }
                    s_prefix = (prefix << w) | (uint64_t)d;
                    s_sel[0] = k - acc;
                    s_sel[1] = (int)hist[d];
                }
            }
            __syncthreads();
            prefix = s_prefix;
            k = s_sel[0];
            m = s_sel[1];
            bits += w;
            __syncthreads();
        }
        // the keys sharing the prefix (m <= kCollect of them), then the k-th
        if (threadIdx.x == 0) s_total = 0;
        __syncthreads();
        for (int a = threadIdx.x; a < S; a += blockDim.x) {
            if (!is_candidate(lm, S, a)) continue;
            const uint64_t key = sm64_key(seed_b, a);
            if (bits > 0 && (key >> (64 - bits)) != prefix) continue;
            const int slot = atomicAdd(&s_total, 1);
            if (slot < kCollect) list[slot] = key;
        }
        __syncthreads();
        const int mm = min(s_total, kCollect);
        if ((int)threadIdx.x < mm) {
            const uint64_t x = list[threadIdx.x];
            int below = 0;
            for (int i = 0; i < mm; i++) below += list[i] < x;
            if (below == k - 1) s_prefix = x;
        }
        __syncthreads();
        T = s_prefix;
        __syncthreads();
    }

    // compaction in ascending A of the candidates with key <= T: warp w owns
    // the positions [w S / 32, (w + 1) S / 32); it counts its chosen ones, one
    // scan over the warps gives its first output slot, and it writes them in order
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int lo = (int)((long long)S * warp / nw), hi = (int)((long long)S * (warp + 1) / nw);
    auto chosen_at = [&](int a) {
        return a < hi && is_candidate(lm, S, a) && (C <= N || sm64_key(seed_b, a) <= T);
    };
    int mine = 0;
    for (int a0 = lo; a0 < hi; a0 += 32) mine += __popc(__ballot_sync(0xffffffffu, chosen_at(a0 + lane)));
    if (lane == 0) warp_tot[warp] = mine;
    __syncthreads();
    if (warp == 0) {
        int t = lane < nw ? warp_tot[lane] : 0;
        const int own = t;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, t, d);
            if (lane >= d) t += y;
        }
        if (lane < nw) warp_tot[lane] = t - own;  // exclusive
        if (lane == 31) s_total = t;
    }
    __syncthreads();
    int slot = warp_tot[warp];
    for (int a0 = lo; a0 < hi; a0 += 32) {
        const bool c = chosen_at(a0 + lane);
        const unsigned bal = __ballot_sync(0xffffffffu, c);
        const int at = slot + __popc(bal & ((1u << lane) - 1u));
        if (c && at < N) {
            an[at] = a0 + lane;
            kp[at] = 1;
        }
        slot += __popc(bal);
    }
    const int out = s_total;
    // padding blocks (page §3): anchor 0, keep 0
    const int filled = min(out, N);
    for (int i = filled + threadIdx.x; i < N; i += blockDim.x) {
        an[i] = 0;
        kp[i] = 0;
    }
}

// One thread per draft row (b, 5 n + j) with A = anchors[b][n]:
//   draft_ids = x_A (j = 0) or MASK; position = A + j; label = x_{A+j+1};
//   prev = x_{A+j}; eval_mask = prod over j' <= j of [A+j'+1 < S,
//   loss_mask[A+j'+1] = 1 (loss_mask[S-1] read as 0), keep = 1].
// Reads outside [0, S) give MASK (ids, prev), -1 (label) and eval_mask 0.
__global__ void __launch_bounds__(256) k_build_draft_inputs(const int32_t *__restrict__ input_ids,
                                                            const uint8_t *__restrict__ loss_mask, int B, int S,
                                                            int N, const int32_t *__restrict__ anchors,
                                                            const uint8_t *__restrict__ keep, int mask_id,
                                                            int32_t *draft_ids, int32_t *position_ids, int32_t *labels,
                                                            int32_t *prev_ids, uint8_t *eval_mask) {
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t R = (size_t)kBlock * N;
    if (idx >= (size_t)B * R) return;
    const int b = (int)(idx / R), r = (int)(idx % R);
    const int n = r / kBlock, j = r % kBlock;
    const int A = anchors[(size_t)b * N + n];
    const bool kept = keep[(size_t)b * N + n] != 0;
    const int32_t *x = input_ids + (size_t)b * S;
    const uint8_t *lm = loss_mask + (size_t)b * S;
    const long long p = (long long)A + j;
    draft_ids[idx] = j == 0 ? (p >= 0 && p < S ? x[p] : mask_id) : mask_id;
    position_ids[idx] = (int32_t)p;
    labels[idx] = p + 1 >= 0 && p + 1 < S ? x[p + 1] : -1;
    prev_ids[idx] = p >= 0 && p < S ? x[p] : mask_id;
    bool on = kept;
    for (int jj = 0; jj <= j && on; jj++) {
        const long long q = (long long)A + jj + 1;
        on = q >= 0 && q < S - 1 && lm[q] != 0;  // q = S-1 reads loss_mask[S-1] := 0
    }
    eval_mask[idx] = on ? 1 : 0;
}

}  // namespace

cudaError_t launch_sample_anchors(const uint8_t *loss_mask, int B, int S, int N, uint64_t seed, int32_t *anchors,
                                  uint8_t *keep, cudaStream_t st) {
    if (B == 0 || N == 0) return cudaSuccess;
    count_launch();
    k_sample_anchors<<<B, kSampleThreads, 0, st>>>(loss_mask, S, N, seed, anchors, keep);
    return cudaGetLastError();
}

cudaError_t launch_build_draft_inputs(const int32_t *input_ids, const uint8_t *loss_mask, int B, int S, int N,
                                      const int32_t *anchors, const uint8_t *keep, int mask_id, int32_t *draft_ids,
                                      int32_t *position_ids, int32_t *labels, int32_t *prev_ids, uint8_t *eval_mask,
                                      cudaStream_t st) {
    const size_t rows = (size_t)B * kBlock * N;
    if (rows == 0) return cudaSuccess;
    count_launch();
    k_build_draft_inputs<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(input_ids, loss_mask, B, S, N, anchors, keep,
                                                                          mask_id, draft_ids, position_ids, labels,
                                                                          prev_ids, eval_mask);
    return cudaGetLastError();
}

}  // namespace dspark
