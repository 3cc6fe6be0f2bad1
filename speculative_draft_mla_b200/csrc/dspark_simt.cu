// CUDA-core (SIMT) forward and backward of the DSpark draft attention.
//
// This family computes in fp32 for any head widths the library accepts and is
// the fp32 path. Each CTA owns one (batch, block) or one key tile, so that every
// output element has exactly one writer and no atomics are needed.
//
// Definitions (page "GLM 5.2 DSpark speculative-training design"): key set of
// block n = context window [max(0, A-W+1), A) plus the block's own 5 draft
// positions (§3); scores use [q^C; rot(q^R, A+j)] . [k^C; rot(k^R, pos)] scaled
// by (d_c + d_r)^(-1/2) (§4); rows of padding blocks are zero (§3).
#include <algorithm>

#include "dspark_internal.cuh"

namespace dspark {

namespace {

constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float warp_max(float x) {
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ bool block_live(const Prob &p, const int32_t *anchors, const uint8_t *keep, int b, int n,
                                           int *a_out) {
    const int a = anchors[(size_t)b * p.N + n];
    *a_out = a;
    return keep[(size_t)b * p.N + n] && a >= 0 && a <= p.S - 2;
}

// Query rows 5n..5n+4 of head h, rope slice rotated to positions A+j, as fp32.
template <typename T>
__device__ __forceinline__ void load_q_rot(const Prob &p, const T *q, size_t row0, int a, const float2 *tab,
                                           float *qs) {
    const int half = p.d_r / 2;
    for (int e = threadIdx.x; e < kBlock * p.dqk; e += blockDim.x) {
        const int j = e / p.dqk, d = e % p.dqk;
        const T *qrow = q + (row0 + j) * p.dqk;
        float val;
        if (d < p.d_c) {
            val = to_f(qrow[d]);
        } else {
            const int r = d - p.d_c, i = r >> 1;
            const float2 cs = tab[(size_t)(a + j) * half + i];
            const float x0 = to_f(qrow[p.d_c + 2 * i]), x1 = to_f(qrow[p.d_c + 2 * i + 1]);
            val = (r & 1) ? (x0 * cs.y + x1 * cs.x) : (x0 * cs.x - x1 * cs.y);
        }
        qs[e] = val;
    }
}

// ---------------------------------------------------------------------------
// Forward: one CTA per (block n, head h, batch b); 5 rows x |key set|.
template <typename T>
__global__ void __launch_bounds__(128) k_fwd_simt(Prob p, const T *__restrict__ q, const T *__restrict__ kc,
                                                  const T *__restrict__ krr, const T *__restrict__ v,
                                                  const int32_t *__restrict__ anchors,
                                                  const uint8_t *__restrict__ keep, const float2 *__restrict__ tab,
                                                  T *__restrict__ o, float *__restrict__ lse) {
    extern __shared__ float sm[];
    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int kmax = p.W - 1 + kBlock;
    float *qs = sm;                  // [5][dqk]
    float *sc = sm + kBlock * p.dqk;  // [5][kmax]
    const size_t row0 = (size_t)(b * p.n_h + h) * p.R + kBlock * n;
    int a;
    if (!block_live(p, anchors, keep, b, n, &a)) {
        for (int e = threadIdx.x; e < kBlock * p.d_v; e += blockDim.x) o[row0 * p.d_v + e] = from_f<T>(0.f);
        if (threadIdx.x < kBlock) lse[row0 + threadIdx.x] = -INFINITY;
        return;
    }
    const int lo = max(0, a - p.W + 1);
    const int nctx = a - lo, nk = nctx + kBlock;
    load_q_rot(p, q, row0, a, tab, qs);
    __syncthreads();
    const size_t kvbase = (size_t)(b * p.n_h + h) * p.L;
    for (int t = threadIdx.x; t < nk; t += blockDim.x) {
        const int key = t < nctx ? lo + t : p.S + kBlock * n + (t - nctx);
        const T *kcr = kc + (kvbase + key) * p.d_c;
        const T *krow = krr + ((size_t)b * p.L + key) * p.d_r;
        float acc[kBlock] = {0.f, 0.f, 0.f, 0.f, 0.f};
        for (int d = 0; d < p.d_c; d++) {
            const float kd = to_f(kcr[d]);
#pragma unroll
            for (int j = 0; j < kBlock; j++) acc[j] = fmaf(qs[j * p.dqk + d], kd, acc[j]);
        }
        for (int d = 0; d < p.d_r; d++) {
            const float kd = to_f(krow[d]);
#pragma unroll
            for (int j = 0; j < kBlock; j++) acc[j] = fmaf(qs[j * p.dqk + p.d_c + d], kd, acc[j]);
        }
#pragma unroll
        for (int j = 0; j < kBlock; j++) sc[j * kmax + t] = acc[j] * p.scale_log2;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int j = warp; j < kBlock; j += blockDim.x >> 5) {
        float *s = sc + j * kmax;
        float m = -INFINITY;
        for (int t = lane; t < nk; t += 32) m = fmaxf(m, s[t]);
        m = warp_max(m);
        float l = 0.f;
        for (int t = lane; t < nk; t += 32) {
            const float e = exp2f(s[t] - m);
            s[t] = e;
            l += e;
        }
        l = warp_sum(l);
        const float inv = 1.f / l;
        for (int t = lane; t < nk; t += 32) s[t] *= inv;
        if (lane == 0) lse[row0 + j] = (m + log2f(l)) * kLn2;
    }
    __syncthreads();
    for (int d = threadIdx.x; d < p.d_v; d += blockDim.x) {
        float acc[kBlock] = {0.f, 0.f, 0.f, 0.f, 0.f};
        for (int t = 0; t < nk; t++) {
            const int key = t < nctx ? lo + t : p.S + kBlock * n + (t - nctx);
            const float vd = to_f(v[(kvbase + key) * p.d_v + d]);
#pragma unroll
            for (int j = 0; j < kBlock; j++) acc[j] = fmaf(sc[j * kmax + t], vd, acc[j]);
        }
#pragma unroll
        for (int j = 0; j < kBlock; j++) o[(row0 + j) * p.d_v + d] = from_f<T>(acc[j]);
    }
}

// ---------------------------------------------------------------------------
// Backward preprocess: D = rowsum(dO * O), one warp per row.
template <typename T>
__global__ void __launch_bounds__(256) k_bwd_dvec(const T *__restrict__ o, const T *__restrict__ dout, size_t rows,
                                                  int d_v, float *__restrict__ dvec) {
    const size_t row = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float acc = 0.f;
    for (int d = lane; d < d_v; d += 32) acc = fmaf(to_f(o[row * d_v + d]), to_f(dout[row * d_v + d]), acc);
    acc = warp_sum(acc);
    if (lane == 0) dvec[row] = acc;
}

// ---------------------------------------------------------------------------
// Backward, query side: one CTA per (block n, batch b), looping over heads.
// Writes dq for the block's 5 rows (all heads) and dkc / dv / dkr of the
// block's own 5 draft keys, which no other block attends to. dkr is the sum
// over heads of the un-rotated rope-key gradient.
template <typename T>
__global__ void __launch_bounds__(256) k_bwd_query_simt(Prob p, const T *__restrict__ q, const T *__restrict__ kc,
                                                        const T *__restrict__ krr, const T *__restrict__ v,
                                                        const int32_t *__restrict__ anchors,
                                                        const uint8_t *__restrict__ keep,
                                                        const float2 *__restrict__ tab,
                                                        const float *__restrict__ lse, const T *__restrict__ dout,
                                                        const float *__restrict__ dvec, T *__restrict__ dq,
                                                        T *__restrict__ dkc, T *__restrict__ dkr,
                                                        T *__restrict__ dv) {
    extern __shared__ float sm[];
    const int n = blockIdx.x, b = blockIdx.y;
    const int kmax = p.W - 1 + kBlock;
    const int half = p.d_r / 2;
    float *qs = sm;                               // [5][dqk]
    float *dos = qs + kBlock * p.dqk;             // [5][d_v]
    float *pb = dos + kBlock * p.d_v;             // [5][kmax]
    float *dsb = pb + kBlock * kmax;              // [5][kmax]
    float *dqs = dsb + kBlock * kmax;             // [5][dqk]
    float *dkra = dqs + kBlock * p.dqk;           // [5][d_r]
    float *rowv = dkra + kBlock * p.d_r;          // [2][5]: lse*log2e, D
    int a;
    const bool live = block_live(p, anchors, keep, b, n, &a);
    const int draft0 = p.S + kBlock * n;
    if (!live) {
        for (int h = 0; h < p.n_h; h++) {
            const size_t row0 = (size_t)(b * p.n_h + h) * p.R + kBlock * n;
            const size_t kv0 = (size_t)(b * p.n_h + h) * p.L + draft0;
            for (int e = threadIdx.x; e < kBlock * p.dqk; e += blockDim.x) dq[row0 * p.dqk + e] = from_f<T>(0.f);
            for (int e = threadIdx.x; e < kBlock * p.d_c; e += blockDim.x) dkc[kv0 * p.d_c + e] = from_f<T>(0.f);
            for (int e = threadIdx.x; e < kBlock * p.d_v; e += blockDim.x) dv[kv0 * p.d_v + e] = from_f<T>(0.f);
        }
        for (int e = threadIdx.x; e < kBlock * p.d_r; e += blockDim.x)
            dkr[((size_t)b * p.L + draft0) * p.d_r + e] = from_f<T>(0.f);
        return;
    }
    const int lo = max(0, a - p.W + 1);
    const int nctx = a - lo, nk = nctx + kBlock;
    for (int e = threadIdx.x; e < kBlock * p.d_r; e += blockDim.x) dkra[e] = 0.f;
    for (int h = 0; h < p.n_h; h++) {
        const size_t row0 = (size_t)(b * p.n_h + h) * p.R + kBlock * n;
        const size_t kvbase = (size_t)(b * p.n_h + h) * p.L;
        load_q_rot(p, q, row0, a, tab, qs);
        for (int e = threadIdx.x; e < kBlock * p.d_v; e += blockDim.x) dos[e] = to_f(dout[row0 * p.d_v + e]);
        if (threadIdx.x < kBlock) {
            rowv[threadIdx.x] = lse[row0 + threadIdx.x] * kLog2e;
            rowv[kBlock + threadIdx.x] = dvec[row0 + threadIdx.x];
        }
        __syncthreads();
        for (int t = threadIdx.x; t < nk; t += blockDim.x) {
            const int key = t < nctx ? lo + t : draft0 + (t - nctx);
            const T *kcr = kc + (kvbase + key) * p.d_c;
            const T *krow = krr + ((size_t)b * p.L + key) * p.d_r;
            const T *vr = v + (kvbase + key) * p.d_v;
            float s[kBlock] = {0.f, 0.f, 0.f, 0.f, 0.f}, dp[kBlock] = {0.f, 0.f, 0.f, 0.f, 0.f};
            for (int d = 0; d < p.d_c; d++) {
                const float kd = to_f(kcr[d]);
#pragma unroll
                for (int j = 0; j < kBlock; j++) s[j] = fmaf(qs[j * p.dqk + d], kd, s[j]);
            }
            for (int d = 0; d < p.d_r; d++) {
                const float kd = to_f(krow[d]);
#pragma unroll
                for (int j = 0; j < kBlock; j++) s[j] = fmaf(qs[j * p.dqk + p.d_c + d], kd, s[j]);
            }
            for (int d = 0; d < p.d_v; d++) {
                const float vd = to_f(vr[d]);
#pragma unroll
                for (int j = 0; j < kBlock; j++) dp[j] = fmaf(dos[j * p.d_v + d], vd, dp[j]);
            }
#pragma unroll
            for (int j = 0; j < kBlock; j++) {
                const float pj = exp2f(s[j] * p.scale_log2 - rowv[j]);
                pb[j * kmax + t] = pj;
                dsb[j * kmax + t] = pj * (dp[j] - rowv[kBlock + j]) * p.scale;
            }
        }
        __syncthreads();
        // dq in the rotated frame
        for (int e = threadIdx.x; e < kBlock * p.dqk; e += blockDim.x) {
            const int j = e / p.dqk, d = e % p.dqk;
            float acc = 0.f;
            for (int t = 0; t < nk; t++) {
                const int key = t < nctx ? lo + t : draft0 + (t - nctx);
                const float kd = d < p.d_c ? to_f(kc[(kvbase + key) * p.d_c + d])
                                           : to_f(krr[((size_t)b * p.L + key) * p.d_r + (d - p.d_c)]);
                acc = fmaf(dsb[j * kmax + t], kd, acc);
            }
            dqs[e] = acc;
        }
        // the block's own draft keys
        const int wk = p.dqk + p.d_v;
        for (int e = threadIdx.x; e < kBlock * wk; e += blockDim.x) {
            const int i = e / wk, d = e % wk, t = nctx + i;
            float acc = 0.f;
            if (d < p.dqk) {
#pragma unroll
                for (int j = 0; j < kBlock; j++) acc = fmaf(dsb[j * kmax + t], qs[j * p.dqk + d], acc);
                if (d < p.d_c)
                    dkc[(kvbase + draft0 + i) * p.d_c + d] = from_f<T>(acc);
                else
                    dkra[i * p.d_r + (d - p.d_c)] += acc;
            } else {
                const int dd = d - p.dqk;
#pragma unroll
                for (int j = 0; j < kBlock; j++) acc = fmaf(pb[j * kmax + t], dos[j * p.d_v + dd], acc);
                dv[(kvbase + draft0 + i) * p.d_v + dd] = from_f<T>(acc);
            }
        }
        __syncthreads();
        // un-rotate the rope slice of dq (transpose of the rotation at A+j)
        for (int e = threadIdx.x; e < kBlock * p.dqk; e += blockDim.x) {
            const int j = e / p.dqk, d = e % p.dqk;
            float val;
            if (d < p.d_c) {
                val = dqs[e];
            } else {
                const int r = d - p.d_c, i = r >> 1;
                const float2 cs = tab[(size_t)(a + j) * half + i];
                const float x0 = dqs[j * p.dqk + p.d_c + 2 * i], x1 = dqs[j * p.dqk + p.d_c + 2 * i + 1];
                val = (r & 1) ? (x1 * cs.x - x0 * cs.y) : (x0 * cs.x + x1 * cs.y);
            }
            dq[(row0 + j) * p.dqk + d] = from_f<T>(val);
        }
        __syncthreads();
    }
    for (int e = threadIdx.x; e < kBlock * p.d_r; e += blockDim.x) {
        const int i = e / p.d_r, r = e % p.d_r, pi = r >> 1;
        const float2 cs = tab[(size_t)(a + i) * half + pi];
        const float x0 = dkra[i * p.d_r + 2 * pi], x1 = dkra[i * p.d_r + 2 * pi + 1];
        const float val = (r & 1) ? (x1 * cs.x - x0 * cs.y) : (x0 * cs.x + x1 * cs.y);
        dkr[((size_t)b * p.L + draft0 + i) * p.d_r + r] = from_f<T>(val);
    }
}

// ---------------------------------------------------------------------------
// Backward, context-key side: one CTA per (tile of kTK context positions,
// batch b), looping over heads. The blocks whose window covers a position of
// the tile are a contiguous run of the anchor-sorted list: t0 < A <= t0+kTK-1+W-1.
constexpr int kTK = 32;
constexpr int kTKP = kTK + 1;  // padded stride of the transposed accumulators

template <typename T>
__global__ void __launch_bounds__(256) k_bwd_ctx_simt(Prob p, const T *__restrict__ q, const T *__restrict__ kc,
                                                      const T *__restrict__ krr, const T *__restrict__ v,
                                                      const int32_t *__restrict__ cnt,
                                                      const int32_t *__restrict__ sorted_n,
                                                      const int32_t *__restrict__ sorted_a,
                                                      const float2 *__restrict__ tab,
                                                      const float *__restrict__ lse, const T *__restrict__ dout,
                                                      const float *__restrict__ dvec, T *__restrict__ dkc,
                                                      T *__restrict__ dkr, T *__restrict__ dv) {
    extern __shared__ float sm[];
    const int t0 = blockIdx.x * kTK, b = blockIdx.y;
    const int half = p.d_r / 2;
    float *ks = sm;                            // [kTK][dqk] rotated keys
    float *vs = ks + kTK * p.dqk;              // [kTK][d_v]
    float *qs = vs + kTK * p.d_v;              // [5][dqk]
    float *dos = qs + kBlock * p.dqk;          // [5][d_v]
    float *pb = dos + kBlock * p.d_v;          // [5][kTK]
    float *dsb = pb + kBlock * kTK;            // [5][kTK]
    float *dka = dsb + kBlock * kTK;           // [dqk][kTKP]
    float *dva = dka + p.dqk * kTKP;           // [d_v][kTKP]
    float *dkra = dva + p.d_v * kTKP;          // [d_r][kTKP]
    float *rowv = dkra + p.d_r * kTKP;         // [2][5]
    __shared__ int s_lo, s_hi;
    if (threadIdx.x == 0) {
        const int c = cnt[b];
        const int32_t *sa = sorted_a + (size_t)b * p.N;
        // first i with A > t0
        int lo = 0, hi = c;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (sa[mid] > t0) hi = mid; else lo = mid + 1;
        }
        s_lo = lo;
        // first i with A > t0 + kTK - 1 + W - 1
        const long long lim = (long long)t0 + kTK - 1 + p.W - 1;
        int lo2 = lo, hi2 = c;
        while (lo2 < hi2) {
            const int mid = (lo2 + hi2) >> 1;
            if ((long long)sa[mid] > lim) hi2 = mid; else lo2 = mid + 1;
        }
        s_hi = lo2;
    }
    for (int e = threadIdx.x; e < p.d_r * kTKP; e += blockDim.x) dkra[e] = 0.f;
    __syncthreads();
    const int i_lo = s_lo, i_hi = s_hi;
    for (int h = 0; h < p.n_h; h++) {
        const size_t kvbase = (size_t)(b * p.n_h + h) * p.L;
        for (int e = threadIdx.x; e < kTK * p.dqk; e += blockDim.x) {
            const int kk = e / p.dqk, d = e % p.dqk, c = t0 + kk;
            float val = 0.f;
            if (c < p.S)
                val = d < p.d_c ? to_f(kc[(kvbase + c) * p.d_c + d])
                                : to_f(krr[((size_t)b * p.L + c) * p.d_r + (d - p.d_c)]);
            ks[e] = val;
        }
        for (int e = threadIdx.x; e < kTK * p.d_v; e += blockDim.x) {
            const int kk = e / p.d_v, d = e % p.d_v, c = t0 + kk;
            vs[e] = c < p.S ? to_f(v[(kvbase + c) * p.d_v + d]) : 0.f;
        }
        for (int e = threadIdx.x; e < (p.dqk + p.d_v) * kTKP; e += blockDim.x) dka[e] = 0.f;
        __syncthreads();
        for (int i = i_lo; i < i_hi; i++) {
            const int n = sorted_n[(size_t)b * p.N + i], a = sorted_a[(size_t)b * p.N + i];
            const size_t row0 = (size_t)(b * p.n_h + h) * p.R + kBlock * n;
            load_q_rot(p, q, row0, a, tab, qs);
            for (int e = threadIdx.x; e < kBlock * p.d_v; e += blockDim.x) dos[e] = to_f(dout[row0 * p.d_v + e]);
            if (threadIdx.x < kBlock) {
                rowv[threadIdx.x] = lse[row0 + threadIdx.x] * kLog2e;
                rowv[kBlock + threadIdx.x] = dvec[row0 + threadIdx.x];
            }
            __syncthreads();
            if (threadIdx.x < kBlock * kTK) {
                const int j = threadIdx.x / kTK, kk = threadIdx.x % kTK, c = t0 + kk;
                float pj = 0.f, ds = 0.f;
                if (c < p.S && c < a && c >= a - p.W + 1) {
                    float s = 0.f, dp = 0.f;
                    for (int d = 0; d < p.dqk; d++) s = fmaf(qs[j * p.dqk + d], ks[kk * p.dqk + d], s);
                    for (int d = 0; d < p.d_v; d++) dp = fmaf(dos[j * p.d_v + d], vs[kk * p.d_v + d], dp);
                    pj = exp2f(s * p.scale_log2 - rowv[j]);
                    ds = pj * (dp - rowv[kBlock + j]) * p.scale;
                }
                pb[j * kTK + kk] = pj;
                dsb[j * kTK + kk] = ds;
            }
            __syncthreads();
            for (int e = threadIdx.x; e < kTK * (p.dqk + p.d_v); e += blockDim.x) {
                const int kk = e % kTK, d = e / kTK;
                float acc = 0.f;
                if (d < p.dqk) {
#pragma unroll
                    for (int j = 0; j < kBlock; j++) acc = fmaf(dsb[j * kTK + kk], qs[j * p.dqk + d], acc);
                } else {
#pragma unroll
                    for (int j = 0; j < kBlock; j++) acc = fmaf(pb[j * kTK + kk], dos[j * p.d_v + d - p.dqk], acc);
                }
                dka[d * kTKP + kk] += acc;  // dka and dva are contiguous: row d >= dqk is dva
            }
            __syncthreads();
        }
        for (int e = threadIdx.x; e < kTK * p.d_c; e += blockDim.x) {
            const int kk = e / p.d_c, d = e % p.d_c, c = t0 + kk;
            if (c < p.S) dkc[(kvbase + c) * p.d_c + d] = from_f<T>(dka[d * kTKP + kk]);
        }
        for (int e = threadIdx.x; e < kTK * p.d_v; e += blockDim.x) {
            const int kk = e / p.d_v, d = e % p.d_v, c = t0 + kk;
            if (c < p.S) dv[(kvbase + c) * p.d_v + d] = from_f<T>(dva[d * kTKP + kk]);
        }
        for (int e = threadIdx.x; e < kTK * p.d_r; e += blockDim.x) {
            const int kk = e % kTK, d = e / kTK;
            dkra[d * kTKP + kk] += dka[(p.d_c + d) * kTKP + kk];
        }
        __syncthreads();
    }
    for (int e = threadIdx.x; e < kTK * p.d_r; e += blockDim.x) {
        const int kk = e / p.d_r, r = e % p.d_r, c = t0 + kk, pi = r >> 1;
        if (c >= p.S) continue;
        const float2 cs = tab[(size_t)c * half + pi];
        const float x0 = dkra[(2 * pi) * kTKP + kk], x1 = dkra[(2 * pi + 1) * kTKP + kk];
        const float val = (r & 1) ? (x1 * cs.x - x0 * cs.y) : (x0 * cs.x + x1 * cs.y);
        dkr[((size_t)b * p.L + c) * p.d_r + r] = from_f<T>(val);
    }
}

template <typename T>
cudaError_t fwd_impl(const Prob &p, const void *q, const void *kc, const void *v, const int32_t *anchors,
                     const uint8_t *keep, void *o, float *lse, const Ws &ws, cudaStream_t st) {
    const size_t smem = sizeof(float) * kBlock * (p.dqk + p.W - 1 + kBlock);
    cudaError_t e = cudaFuncSetAttribute(k_fwd_simt<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.N, p.n_h, p.B);
    count_launch();
    k_fwd_simt<T><<<grid, 128, smem, st>>>(p, (const T *)q, (const T *)kc, (const T *)ws.kr_rot, (const T *)v,
                                           anchors, keep, ws.rope, (T *)o, lse);
    return cudaGetLastError();
}

template <typename T>
cudaError_t bwd_impl(const Prob &p, const void *q, const void *kc, const void *v, const int32_t *anchors,
                     const uint8_t *keep, const void *o, const float *lse, const void *dout, void *dq, void *dkc,
                     void *dkr, void *dv, const Ws &ws, cudaStream_t st) {
    const size_t rows = (size_t)p.B * p.n_h * p.R;
    if (rows > 0) count_launch();
    if (rows > 0)
        k_bwd_dvec<T><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>((const T *)o, (const T *)dout, rows, p.d_v,
                                                                  ws.dvec);
    const int kmax = p.W - 1 + kBlock;
    if (p.N > 0) {
        const size_t smem = sizeof(float) * (kBlock * (2 * p.dqk + p.d_v + 2 * kmax + p.d_r) + 2 * kBlock);
        cudaError_t e =
            cudaFuncSetAttribute(k_bwd_query_simt<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        count_launch();
        k_bwd_query_simt<T><<<dim3(p.N, p.B), 256, smem, st>>>(
            p, (const T *)q, (const T *)kc, (const T *)ws.kr_rot, (const T *)v, anchors, keep, ws.rope, lse,
            (const T *)dout, ws.dvec, (T *)dq, (T *)dkc, (T *)dkr, (T *)dv);
    }
    {
        const size_t smem = sizeof(float) * (kTK * (p.dqk + p.d_v) + kBlock * (p.dqk + p.d_v) + 2 * kBlock * kTK +
                                             (p.dqk + p.d_v + p.d_r) * kTKP + 2 * kBlock);
        cudaError_t e =
            cudaFuncSetAttribute(k_bwd_ctx_simt<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        dim3 grid((p.S + kTK - 1) / kTK, p.B);
        count_launch();
        k_bwd_ctx_simt<T><<<grid, 256, smem, st>>>(p, (const T *)q, (const T *)kc, (const T *)ws.kr_rot,
                                                   (const T *)v, ws.cnt, ws.sorted_n, ws.sorted_a, ws.rope, lse,
                                                   (const T *)dout, ws.dvec, (T *)dkc, (T *)dkr, (T *)dv);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_simt(const Prob &p, const void *q, const void *kc, const void *v, const int32_t *anchors,
                            const uint8_t *keep, void *o, float *lse, const Ws &ws, cudaStream_t st) {
    if (p.B == 0 || p.N == 0) return cudaSuccess;
    if (p.dtype == DSPARK_BF16) return fwd_impl<__nv_bfloat16>(p, q, kc, v, anchors, keep, o, lse, ws, st);
    return fwd_impl<float>(p, q, kc, v, anchors, keep, o, lse, ws, st);
}

cudaError_t launch_bwd_simt(const Prob &p, const void *q, const void *kc, const void *v, const int32_t *anchors,
                            const uint8_t *keep, const void *o, const float *lse, const void *dout, void *dq,
                            void *dkc, void *dkr, void *dv, const Ws &ws, cudaStream_t st) {
    if (p.B == 0) return cudaSuccess;
    if (p.dtype == DSPARK_BF16)
        return bwd_impl<__nv_bfloat16>(p, q, kc, v, anchors, keep, o, lse, dout, dq, dkc, dkr, dv, ws, st);
    return bwd_impl<float>(p, q, kc, v, anchors, keep, o, lse, dout, dq, dkc, dkr, dv, ws, st);
}

}  // namespace dspark
