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

// One CTA per batch row: validate kept anchors, bitonic-sort the keys
// (anchor << 32 | block) ascending in shared memory, write the sorted run.
__global__ void __launch_bounds__(1024) k_sort_blocks(const int32_t *__restrict__ anchors,
                                                      const uint8_t *__restrict__ keep, int N, int S, int NP,
                                                      uint32_t *err, int32_t *cnt, int32_t *sorted_n,
                                                      int32_t *sorted_a) {
    extern __shared__ unsigned long long keys[];
    __shared__ int s_cnt;
    const int b = blockIdx.x;
    if (threadIdx.x == 0) s_cnt = 0;
    __syncthreads();
    int local = 0;
    bool bad = false;
    for (int i = threadIdx.x; i < NP; i += blockDim.x) {
        unsigned long long k = ~0ull;
        if (i < N && keep[(size_t)b * N + i]) {
            int a = anchors[(size_t)b * N + i];
            if (a >= 0 && a <= S - 2) {
                k = ((unsigned long long)(uint32_t)a << 32) | (uint32_t)i;
                local++;
            } else {
                bad = true;
            }
        }
        keys[i] = k;
    }
    if (bad) atomicOr(err, kErrAnchor);
    atomicAdd(&s_cnt, local);
    __syncthreads();
    for (int k = 2; k <= NP; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < NP; i += blockDim.x) {
                int ixj = i ^ j;
                if (ixj > i) {
                    unsigned long long x = keys[i], y = keys[ixj];
                    bool up = (i & k) == 0;
                    if ((x > y) == up) {
                        keys[i] = y;
                        keys[ixj] = x;
                    }
                }
            }
            __syncthreads();
        }
    }
    const int c = s_cnt;
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
        if (i < c) {
            sorted_n[(size_t)b * N + i] = (int32_t)(keys[i] & 0xffffffffull);
            sorted_a[(size_t)b * N + i] = (int32_t)(keys[i] >> 32);
        } else {
            sorted_n[(size_t)b * N + i] = -1;
            sorted_a[(size_t)b * N + i] = INT_MAX;
        }
    }
    if (threadIdx.x == 0) cnt[b] = c;
}

// (cos, sin) of pos * base^(-2i/d_r), angle formed and evaluated in fp64.
__global__ void k_rope_table(float2 *tab, int P, int half, int d_r, double base) {
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (size_t)P * half) return;
    const int pos = (int)(idx / half), i = (int)(idx % half);
    const double theta = pow(base, -2.0 * (double)i / (double)d_r);
    double s, c;
    sincos((double)pos * theta, &s, &c);
    tab[idx] = make_float2((float)c, (float)s);
}

// Rope key of every kv position rotated to its position: context c -> c,
// draft key S + 5n + i -> A_n + i. Positions of padding or invalid blocks are
// clamped into the table (those keys are never attended).
template <typename T>
__global__ void k_rotate_kr(const T *__restrict__ kr, const int32_t *__restrict__ anchors,
                            const float2 *__restrict__ tab, T *__restrict__ out, int B, int S, int N, int L, int d_r,
                            int P) {
    const int half = d_r / 2;
    const size_t total = (size_t)B * L * half;
    for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int i = (int)(idx % half);
        const size_t bk = idx / half;
        const int key = (int)(bk % L), b = (int)(bk / L);
        int pos = key;
        if (key >= S) {
            const int n = (key - S) / kBlock, j = (key - S) % kBlock;
            pos = anchors[(size_t)b * N + n] + j;
        }
        pos = min(max(pos, 0), P - 1);
        const float2 cs = tab[(size_t)pos * half + i];
        const T *x = kr + bk * d_r + 2 * i;
        const float x0 = to_f(x[0]), x1 = to_f(x[1]);
        T *y = out + bk * d_r + 2 * i;
        y[0] = from_f<T>(x0 * cs.x - x1 * cs.y);
        y[1] = from_f<T>(x0 * cs.y + x1 * cs.x);
    }
}

cudaError_t launch_build_descriptor(const Prob &p, const int32_t *anchors, const uint8_t *keep, const Ws &ws,
                                    cudaStream_t st) {
    // a new descriptor starts a new error epoch (a fresh workspace holds garbage)
    cudaError_t e0 = cudaMemsetAsync(ws.err, 0, sizeof(uint32_t), st);
    if (e0 != cudaSuccess) return e0;
    if (p.B > 0 && p.N > 0) {
        int NP = 1;
        while (NP < p.N) NP <<= 1;
        const size_t smem = sizeof(unsigned long long) * NP;
        cudaError_t e = cudaFuncSetAttribute(k_sort_blocks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        count_launch();
        k_sort_blocks<<<p.B, 1024, smem, st>>>(anchors, keep, p.N, p.S, NP, ws.err, ws.cnt, ws.sorted_n,
                                               ws.sorted_a);
    } else if (p.B > 0) {
        cudaError_t e = cudaMemsetAsync(ws.cnt, 0, sizeof(int32_t) * p.B, st);
        if (e != cudaSuccess) return e;
    }
    const int half = p.d_r / 2;
    if (half > 0) {
        const size_t total = (size_t)p.P * half;
        count_launch();
        k_rope_table<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(ws.rope, p.P, half, p.d_r, p.base);
    }
    return cudaGetLastError();
}

cudaError_t launch_rotate_kr(const Prob &p, const void *kr, const int32_t *anchors, const Ws &ws, cudaStream_t st) {
    const int half = p.d_r / 2;
    const size_t total = (size_t)p.B * p.L * half;
    if (total == 0) return cudaSuccess;
    const unsigned grid = (unsigned)std::min<size_t>((total + 255) / 256, 148 * 16);
    count_launch();
    if (p.dtype == DSPARK_BF16)
        k_rotate_kr<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)kr, anchors, ws.rope,
                                                         (__nv_bfloat16 *)ws.kr_rot, p.B, p.S, p.N, p.L, p.d_r, p.P);
    else
        k_rotate_kr<float><<<grid, 256, 0, st>>>((const float *)kr, anchors, ws.rope, (float *)ws.kr_rot, p.B, p.S,
                                                 p.N, p.L, p.d_r, p.P);
    return cudaGetLastError();
}

}  // namespace dspark
