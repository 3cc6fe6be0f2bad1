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

// The descriptor in one launch. CTAs 0 .. B-1, one per batch row: validate the
// kept anchors, sort the keys (anchor << 32 | block) ascending, write the
// sorted run and the kept count. The keys are unique, so for N <= 1024 the
// position of a key is its rank, the number of kept keys below it (each key's
// comparisons split over the CTA's threads); larger N take a bitonic sort in
// shared memory (NP = N rounded up to a power of two). CTAs from B on fill the
// RoPE table: (cos, sin) of pos * base^(-2i/d_r), angle formed and evaluated in
// fp64, for positions 0 .. P-1 (page §4 "RoPE").
constexpr int kRankSortMax = 1024;

__global__ void __launch_bounds__(1024) k_build_descriptor(const int32_t *__restrict__ anchors,
                                                           const uint8_t *__restrict__ keep, int B, int N, int S,
                                                           int NP, uint32_t *err, int32_t *cnt, int32_t *sorted_n,
                                                           int32_t *sorted_a, float2 *tab, int P, int half, int d_r,
                                                           double base) {
    extern __shared__ unsigned long long keys[];  // NP keys; rank sort: then N ranks
    if ((int)blockIdx.x >= B) {
        // table: thread t of CTA c covers frequency t % half at positions
        // (c - B) * (T / half) + t / half, + (gridDim.x - B) * (T / half), ...
        const int per = blockDim.x / half;  // positions per CTA round (half <= 128 <= blockDim.x)
        const int i = threadIdx.x % half, r = threadIdx.x / half;
        if (r >= per) return;
        const double theta = pow(base, -2.0 * (double)i / (double)d_r);
        for (int pos = ((int)blockIdx.x - B) * per + r; pos < P; pos += ((int)gridDim.x - B) * per) {
            double sn, cs;
            sincos((double)pos * theta, &sn, &cs);
            tab[(size_t)pos * half + i] = make_float2((float)cs, (float)sn);
        }
        return;
    }
    const int b = blockIdx.x;
    const int32_t *an = anchors + (size_t)b * N;
    const uint8_t *kp = keep + (size_t)b * N;
    int c = 0;
    bool bad = false;
    // keys (~0 for blocks that are not kept, which sort last), counting kept ones
    for (int i0 = 0; i0 < NP; i0 += blockDim.x) {
        const int i = i0 + threadIdx.x;
        bool kept = false;
        if (i < NP) {
            unsigned long long k = ~0ull;
            if (i < N && kp[i]) {
                const int a = an[i];
                if (a >= 0 && a <= S - 2) {
                    k = ((unsigned long long)(uint32_t)a << 32) | (uint32_t)i;
                    kept = true;
                } else {
                    bad = true;
                }
            }
            keys[i] = k;
        }
        c += __syncthreads_count(kept);
    }
    if (bad) atomicOr(err, kErrAnchor);
    int32_t *on = sorted_n + (size_t)b * N, *oa = sorted_a + (size_t)b * N;
    if (N <= kRankSortMax) {
        int *rank = reinterpret_cast<int *>(keys + NP);
        const int parts = max(1, (int)blockDim.x / max(N, 1));
        for (int i = threadIdx.x; i < N; i += blockDim.x) rank[i] = 0;
        __syncthreads();
        if ((int)threadIdx.x < parts * N) {
            const int i = threadIdx.x % N, part = threadIdx.x / N;
            const unsigned long long x = keys[i];
            if (x != ~0ull) {
                const int j0 = (int)((long long)N * part / parts), j1 = (int)((long long)N * (part + 1) / parts);
                int r0 = 0, r1 = 0;
                int j = j0;
                for (; j + 1 < j1; j += 2) {
                    r0 += keys[j] < x;
                    r1 += keys[j + 1] < x;
                }
                if (j < j1) r0 += keys[j] < x;
                atomicAdd(&rank[i], r0 + r1);
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < N; i += blockDim.x) {
            const unsigned long long x = keys[i];
            if (x != ~0ull) {
                on[rank[i]] = (int32_t)(x & 0xffffffffull);
                oa[rank[i]] = (int32_t)(x >> 32);
            }
        }
    } else {
        for (int k = 2; k <= NP; k <<= 1) {
            for (int j = k >> 1; j > 0; j >>= 1) {
                for (int i = threadIdx.x; i < NP; i += blockDim.x) {
                    const int ixj = i ^ j;
                    if (ixj > i) {
                        const unsigned long long x = keys[i], y = keys[ixj];
                        const bool up = (i & k) == 0;
                        if ((x > y) == up) {
                            keys[i] = y;
                            keys[ixj] = x;
                        }
                    }
                }
                __syncthreads();
            }
        }
        for (int i = threadIdx.x; i < c; i += blockDim.x) {
            on[i] = (int32_t)(keys[i] & 0xffffffffull);
            oa[i] = (int32_t)(keys[i] >> 32);
        }
    }
    for (int i = c + threadIdx.x; i < N; i += blockDim.x) {
        on[i] = -1;
        oa[i] = INT_MAX;
    }
    if (threadIdx.x == 0) cnt[b] = c;
}

// Rope key of every kv position rotated to its position: context c -> c,
// draft key S + 5n + i -> A_n + i. Positions of padding or invalid blocks are
// clamped into the table (those keys are never attended). One warp per kv
// position, lane i turning pairs i, i + 32, ... (adjacent elements, page §4).
// CTAs from rot_ctas on take one block (n, b) each and zero its rows in the
// PadRows tensors if it is a padding block.
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
                                                   int n_h, unsigned rot_ctas, PadRows pad) {
    if (blockIdx.x < rot_ctas) {
        const int half = d_r / 2, lane = threadIdx.x & 31;
        const size_t row = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
        if (row >= (size_t)B * L) return;
        const int key = (int)(row % (unsigned)L), b = (int)(row / (unsigned)L);
        int pos = key;
        if (key >= S) {
            const int n = (key - S) / kBlock, j = (key - S) % kBlock;
            pos = anchors[(size_t)b * N + n] + j;
        }
        pos = min(max(pos, 0), P - 1);
        using V = typename Pair<T>::V;
        const V *x = reinterpret_cast<const V *>(kr + row * d_r);
        V *y = reinterpret_cast<V *>(out + row * d_r);
        const float2 *cs = tab + (size_t)pos * half;
        for (int i = lane; i < half; i += 32) {
            const float2 v = pair_f(x[i]);
            const float2 c = cs[i];
            y[i] = pair_from<V>(v.x * c.x - v.y * c.y, v.x * c.y + v.y * c.x);
        }
        return;
    }
    const unsigned id = blockIdx.x - rot_ctas;
    const int n = (int)(id % (unsigned)N), b = (int)(id / (unsigned)N);
    const int a = anchors[(size_t)b * N + n];
    if (keep[(size_t)b * N + n] && a >= 0 && a <= S - 2) return;
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int h = 0; h < n_h; h++) {
        const size_t bh = (size_t)b * n_h + h;
#pragma unroll
        for (int k = 0; k < 3; k++) {
            if (!pad.t[k]) continue;
            const int w8 = pad.width[k] / 8;
            uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(pad.t[k]) +
                                                   (bh * pad.rows[k] + pad.first[k] + (size_t)kBlock * n) * pad.width[k]);
            for (int e = threadIdx.x; e < kBlock * w8; e += blockDim.x) dst[e] = z;
        }
        if (pad.lse && threadIdx.x < kBlock) pad.lse[bh * kBlock * N + (size_t)kBlock * n + threadIdx.x] = -INFINITY;
    }
}

cudaError_t launch_build_descriptor(const Prob &p, const int32_t *anchors, const uint8_t *keep, const Ws &ws,
                                    cudaStream_t st) {
    // a new descriptor starts a new error epoch (a fresh workspace holds garbage)
    cudaError_t e = cudaMemsetAsync(ws.err, 0, sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
    const int half = p.d_r / 2;
    const int sort_ctas = p.N > 0 ? p.B : 0;
    const int table_ctas = half > 0 ? 64 : 0;
    if (p.N == 0 && p.B > 0) {
        if ((e = cudaMemsetAsync(ws.cnt, 0, sizeof(int32_t) * p.B, st)) != cudaSuccess) return e;
    }
    if (sort_ctas + table_ctas == 0) return cudaSuccess;
    int NP = 1;
    while (NP < p.N) NP <<= 1;
    const size_t smem = sizeof(unsigned long long) * (size_t)NP + (p.N <= kRankSortMax ? sizeof(int) * (size_t)p.N : 0);
    e = cudaFuncSetAttribute(k_build_descriptor, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    k_build_descriptor<<<sort_ctas + table_ctas, 1024, smem, st>>>(anchors, keep, sort_ctas, p.N, p.S, NP, ws.err,
                                                                    ws.cnt, ws.sorted_n, ws.sorted_a, ws.rope, p.P,
                                                                    half > 0 ? half : 1, p.d_r, p.base);
    return cudaGetLastError();
}

cudaError_t launch_rotate_kr(const Prob &p, const void *kr, const int32_t *anchors, const uint8_t *keep,
                             const PadRows *pad, const Ws &ws, cudaStream_t st) {
    const size_t rows = p.d_r > 0 ? (size_t)p.B * p.L : 0;
    const unsigned rot_ctas = (unsigned)((rows + 7) / 8);
    const unsigned pad_ctas = pad ? (unsigned)((size_t)p.N * p.B) : 0u;
    if (rot_ctas + pad_ctas == 0) return cudaSuccess;
    PadRows pr{};
    if (pad) pr = *pad;
    count_launch();
    if (p.dtype == DSPARK_BF16)
        k_rotate_kr<__nv_bfloat16><<<rot_ctas + pad_ctas, 256, 0, st>>>(
            (const __nv_bfloat16 *)kr, anchors, keep, ws.rope, (__nv_bfloat16 *)ws.kr_rot, p.B, p.S, p.N, p.L, p.d_r,
            p.P, p.n_h, rot_ctas, pr);
    else
        k_rotate_kr<float><<<rot_ctas + pad_ctas, 256, 0, st>>>((const float *)kr, anchors, keep, ws.rope,
                                                                (float *)ws.kr_rot, p.B, p.S, p.N, p.L, p.d_r, p.P,
                                                                p.n_h, rot_ctas, pr);
    return cudaGetLastError();
}

}  // namespace dspark
