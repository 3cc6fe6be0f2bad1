// Mask descriptor and RoPE preparation kernels.
//
// The mask of the DSpark design page (§3 "attention mask") is fixed by the
// anchors and block_keep_mask alone, and is built once before the three draft
// layers run (§3, §4). Its device form here is, per batch row, the kept blocks
// sorted by anchor: the blocks whose context windows cover a key range are then
// a contiguous run of that list. The RoPE table holds (cos, sin) of
// pos * base^(-2i/d_r) for every position a query or key can take (§4 "RoPE").
#include <algorithm>
#include <climits>

#include "dspark_internal.cuh"

namespace dspark {

// The descriptor in one launch. The first B * chunks CTAs sort: CTA (b, c)
// loads all keys (anchor << 32 | block) of batch row b into shared memory
// (~0 for blocks that are not kept), validates the kept anchors, and places
// the kept keys kSortChunk c .. + kSortChunk - 1 at their rank, the number of
// kept keys below them; the keys are unique, so the ranks are the sorted order.
// Each key's comparisons are split over kSortParts threads. CTA (b, 0) also
// writes the kept count and the sentinel entries after the kept ones, and
// CTA 0 writes the error word: the anchor bit if a kept anchor of any batch
// row is out of range, else 0 (a new error epoch; the kernels that may set
// other bits run after this one). The remaining CTAs fill the RoPE table: (cos, sin) of
// pos * base^(-2i/d_r), angle formed and evaluated in fp64, for positions
// 0 .. P-1 (page §4 "RoPE").
constexpr int kSortThreads = 1024, kSortChunk = 128, kSortParts = kSortThreads / kSortChunk;

__global__ void __launch_bounds__(kSortThreads) k_build_descriptor(
    const int32_t *__restrict__ anchors, const uint8_t *__restrict__ keep, int B, int sort_ctas, int chunks, int N,
    int S,
    uint32_t *err, int32_t *cnt, int32_t *sorted_n, int32_t *sorted_a, float2 *tab, int P, int half, int d_r,
    double base) {
    extern __shared__ unsigned long long keys[];  // N keys
    __shared__ int rank[kSortChunk];
    __shared__ double theta[kSortThreads / 8];  // base^(-2i/d_r), i < half <= 128
    pdl_wait();
    pdl_trigger();
    if ((int)blockIdx.x >= sort_ctas) {
        // table: entry e = pos * half + i of CTA c's range (c - sort_ctas) * T + t,
        // + (gridDim.x - sort_ctas) * T, ... (one per thread at the usual grid)
        if ((int)threadIdx.x < half) theta[threadIdx.x] = pow(base, -2.0 * (double)threadIdx.x / (double)d_r);
        __syncthreads();
        const size_t total = (size_t)P * half;
        for (size_t e = (size_t)((int)blockIdx.x - sort_ctas) * blockDim.x + threadIdx.x; e < total;
             e += (size_t)((int)gridDim.x - sort_ctas) * blockDim.x) {
            const int pos = (int)(e / half), i = (int)(e % half);
            double sn, cs;
            sincos((double)pos * theta[i], &sn, &cs);
            tab[e] = make_float2((float)cs, (float)sn);
        }
        return;
    }
    const int b = blockIdx.x / chunks, ch = blockIdx.x % chunks;
    const int32_t *an = anchors + (size_t)b * N;
    const uint8_t *kp = keep + (size_t)b * N;
    if (blockIdx.x == 0) {
        bool any_bad = false;
        for (int e = threadIdx.x; e < B * N; e += blockDim.x) {
            const int a = anchors[e];
            any_bad |= keep[e] && (a < 0 || a > S - 2);
        }
        any_bad = __syncthreads_or(any_bad);
        if (threadIdx.x == 0) *err = any_bad ? kErrAnchor : 0u;
    }
    int c = 0;
    for (int i0 = 0; i0 < N; i0 += blockDim.x) {  // uniform trip count: every thread meets each barrier
        const int i = i0 + threadIdx.x;
        bool kept = false;
        if (i < N) {
            unsigned long long k = ~0ull;
            if (kp[i]) {
                const int a = an[i];
                if (a >= 0 && a <= S - 2) {
                    k = ((unsigned long long)(uint32_t)a << 32) | (uint32_t)i;
                    kept = true;
                }
            }
            keys[i] = k;
        }
        c += __syncthreads_count(kept);
    }
    if (threadIdx.x < kSortChunk) rank[threadIdx.x] = 0;
    __syncthreads();
    const int kl = threadIdx.x % kSortChunk, part = threadIdx.x / kSortChunk;
    const int i = ch * kSortChunk + kl;
    const unsigned long long x = i < N ? keys[i] : ~0ull;
    if (x != ~0ull) {
        const int j0 = (int)((long long)N * part / kSortParts), j1 = (int)((long long)N * (part + 1) / kSortParts);
        int r0 = 0, r1 = 0;
        int j = j0;
        for (; j + 1 < j1; j += 2) {
            r0 += keys[j] < x;
            r1 += keys[j + 1] < x;
        }
        if (j < j1) r0 += keys[j] < x;
        atomicAdd(&rank[kl], r0 + r1);
    }
    __syncthreads();
    int32_t *on = sorted_n + (size_t)b * N, *oa = sorted_a + (size_t)b * N;
    if (part == 0 && x != ~0ull) {
        on[rank[kl]] = (int32_t)(x & 0xffffffffull);
        oa[rank[kl]] = (int32_t)(x >> 32);
    }
    if (ch == 0) {
        for (int k = c + threadIdx.x; k < N; k += blockDim.x) {
            on[k] = -1;
            oa[k] = INT_MAX;
        }
        if (threadIdx.x == 0) cnt[b] = c;
    }
}

// Rope key of every kv position rotated to its position: context c -> c,
// draft key S + 5n + i -> A_n + i. Positions of padding or invalid blocks are
// clamped into the table (those keys are never attended). Warp w of the grid
// takes positions 4w .. 4w + 3 (all their loads in flight together), lane i
// turning pairs i, i + 32, ... (adjacent elements, page §4). CTA g also takes blocks (n, b) = g, g + G, ... of pad_blocks (G
// CTAs) and zeroes the rows of the padding ones in the PadRows tensors; CTA 0
// also zeroes the word pad.clear.
template <typename T> struct Pair;
template <> struct Pair<float> { using V = float2; };
template <> struct Pair<__nv_bfloat16> { using V = __nv_bfloat162; };
__device__ __forceinline__ float2 pair_f(float2 v) { return v; }
__device__ __forceinline__ float2 pair_f(__nv_bfloat162 v) { return __bfloat1622float2(v); }
template <typename V> __device__ __forceinline__ V pair_from(float a, float b);
template <> __device__ __forceinline__ float2 pair_from<float2>(float a, float b) { return make_float2(a, b); }
template <> __device__ __forceinline__ __nv_bfloat162 pair_from<__nv_bfloat162>(float a, float b) {
    return __floats2bfloat162_rn(a, b);
}

template <typename T>
__global__ void __launch_bounds__(256) k_rotate_kr(const T *__restrict__ kr, const int32_t *__restrict__ anchors,
                                                   const uint8_t *__restrict__ keep, const float2 *__restrict__ tab,
                                                   T *__restrict__ out, int B, int S, int N, int L, int d_r, int P,
                                                   int n_h, int pad_blocks, PadRows pad) {
    pdl_wait();
    pdl_trigger();
    const int half = d_r / 2, lane = threadIdx.x & 31;
    const size_t rows = half > 0 ? (size_t)B * L : 0;
    using V = typename Pair<T>::V;
    constexpr int kRows = 4;  // positions per warp
    const size_t row0 = ((size_t)blockIdx.x * 8 + (threadIdx.x >> 5)) * kRows;
    if (row0 < rows) {
        int pos[kRows];
#pragma unroll
        for (int r = 0; r < kRows; r++) {
            const size_t row = min(row0 + r, rows - 1);
            const int key = (int)(row % (unsigned)L), b = (int)(row / (unsigned)L);
            int ps = key;
            if (key >= S) {
                const int n = (key - S) / kBlock, j = (key - S) % kBlock;
                ps = anchors[(size_t)b * N + n] + j;
            }
            pos[r] = min(max(ps, 0), P - 1);
        }
        for (int i = lane; i < half; i += 32) {
            float2 v[kRows], c[kRows];
#pragma unroll
            for (int r = 0; r < kRows; r++) {
                const size_t row = min(row0 + r, rows - 1);
                v[r] = pair_f(reinterpret_cast<const V *>(kr + row * d_r)[i]);
                c[r] = tab[(size_t)pos[r] * half + i];
            }
#pragma unroll
            for (int r = 0; r < kRows; r++)
                if (row0 + r < rows)
                    reinterpret_cast<V *>(out + (row0 + r) * d_r)[i] =
                        pair_from<V>(v[r].x * c[r].x - v[r].y * c[r].y, v[r].x * c[r].y + v[r].y * c[r].x);
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0 && pad.clear) *pad.clear = 0;
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int id = blockIdx.x; id < pad_blocks; id += gridDim.x) {
        const int n = id % N, b = id / N;
        const int a = anchors[(size_t)b * N + n];
        if (keep[(size_t)b * N + n] && a >= 0 && a <= S - 2) continue;
        for (int h = 0; h < n_h; h++) {
            const size_t bh = (size_t)b * n_h + h;
#pragma unroll
            for (int k = 0; k < 3; k++) {
                if (!pad.t[k]) continue;
                const int w8 = pad.width[k] / 8;
                uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(pad.t[k]) +
                                                       (bh * pad.rows[k] + pad.first[k] + (size_t)kBlock * n) *
                                                           pad.width[k]);
                for (int e = threadIdx.x; e < kBlock * w8; e += blockDim.x) dst[e] = z;
            }
            if (pad.lse && threadIdx.x < kBlock) pad.lse[bh * kBlock * N + (size_t)kBlock * n + threadIdx.x] = -INFINITY;
        }
    }
}

cudaError_t launch_build_descriptor(const Prob &p, const int32_t *anchors, const uint8_t *keep, const Ws &ws,
                                    cudaStream_t st) {
    // a new descriptor starts a new error epoch (a fresh workspace holds
    // garbage): the kernel's CTA 0 writes the error word when it sorts, else a memset clears it
    cudaError_t e;
    const int half = p.d_r / 2;
    const int sort_ctas = p.N > 0 ? p.B : 0;
    // one table entry per thread, up to 2 CTAs per SM
    const int table_ctas = half > 0 ? (int)std::min<size_t>(((size_t)p.P * half + kSortThreads - 1) / kSortThreads, 296) : 0;
    if (sort_ctas == 0) {
        if ((e = cudaMemsetAsync(ws.err, 0, sizeof(uint32_t), st)) != cudaSuccess) return e;
        if (p.B > 0 && (e = cudaMemsetAsync(ws.cnt, 0, sizeof(int32_t) * p.B, st)) != cudaSuccess) return e;
    }
    if (sort_ctas + table_ctas == 0) return cudaSuccess;
    const int chunks = (p.N + kSortChunk - 1) / kSortChunk;
    const size_t smem = sizeof(unsigned long long) * (size_t)p.N;
    e = cudaFuncSetAttribute(k_build_descriptor, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    return launch_pdl(k_build_descriptor, dim3(sort_ctas * chunks + table_ctas), dim3(kSortThreads), smem, st, anchors,
                      keep, p.B, sort_ctas * chunks, chunks, p.N, p.S, ws.err, ws.cnt, ws.sorted_n, ws.sorted_a,
                      ws.rope, p.P, half > 0 ? half : 1, p.d_r, p.base);
}

cudaError_t launch_rotate_kr(const Prob &p, const void *kr, const int32_t *anchors, const uint8_t *keep,
                             const PadRows *pad, const Ws &ws, cudaStream_t st) {
    const size_t rows = p.d_r > 0 ? (size_t)p.B * p.L : 0;
    const int pad_blocks = pad ? p.N * p.B : 0;
    // four positions per warp; the padding blocks over at least 4 CTAs per SM
    const size_t want = std::max<size_t>(std::max<size_t>((rows + 31) / 32, (size_t)std::min(pad_blocks, 148 * 4)),
                                         pad && pad->clear ? 1 : 0);
    if (want == 0) return cudaSuccess;
    const unsigned grid = (unsigned)want;
    PadRows pr{};
    if (pad) pr = *pad;
    count_launch();
    if (p.dtype == DSPARK_BF16)
        return launch_pdl(k_rotate_kr<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, (const __nv_bfloat16 *)kr,
                          anchors, keep, (const float2 *)ws.rope, (__nv_bfloat16 *)ws.kr_rot, p.B, p.S, p.N, p.L,
                          p.d_r, p.P, p.n_h, pad_blocks, pr);
    return launch_pdl(k_rotate_kr<float>, dim3(grid), dim3(256), 0, st, (const float *)kr, anchors, keep,
                      (const float2 *)ws.rope, (float *)ws.kr_rot, p.B, p.S, p.N, p.L, p.d_r, p.P, p.n_h, pad_blocks,
                      pr);
}

}  // namespace dspark
