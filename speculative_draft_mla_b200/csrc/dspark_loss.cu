// The DSpark training loss over the draft steps and its gradient (page "GLM
// 5.2 DSpark speculative-training design", §6): per step r (student logits L,
// teacher logits T over the vocabulary, label y, confidence logit c, eval_mask
// m) CE = logsumexp(L) - L[y], L1 = ||softmax(L) - softmax(T)||_1, the
// confidence target a = clip(1 - L1 / 2, 0, 1) (gradient stopped) and
// BCE-with-logits(c, a); each term summed over the counted steps and divided by
// their number M; the gradients with respect to L and c.
//
// A vocabulary row (V = 154880: 620 KB of bf16 L and T) does not fit in one
// SM, and the L1 term needs the row's two normalisers before any |p - q|, so a
// single CTA would read the row three times. Here a cluster of kCl CTAs holds
// one row at a time, each CTA 1/kCl of L and T in shared memory, loaded by 1-D
// bulk copies; the CTAs exchange their partial (max, sum) pairs and then their
// (L1, sum s p) partials through distributed shared memory, so every logit is
// read from HBM once and every gradient written once. Two CTAs share an SM
// (one row slice each, of two different rows), so one's copies and barrier
// waits overlap the other's passes.
// Per element: exp of L and T for the normalisers, p and q for L1 (sign(p - q)
// taken in the log domain); that pass leaves p (bf16) and the sign in place of
// the logits, from which the gradient pass works without an exponential.
#include <cooperative_groups.h>

#include <algorithm>

#include "dspark_steps.cuh"
#include "dspark_tc_common.cuh"

namespace cg = cooperative_groups;

namespace dspark {

namespace {

constexpr int kCl = 8;         // CTAs per row (cluster size)
constexpr int kThr = 448;      // threads per CTA (14 warps at <= 73 registers: two CTAs per SM)
constexpr int kBufs = 1;       // row buffers per CTA (two CTAs per SM overlap each other's waits)
constexpr int kWarps = kThr / 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct LossArgs {
    int R, V, seg;  // rows, vocabulary, elements per CTA (a multiple of 8)
    const __nv_bfloat16 *L, *T;
    const int32_t *labels;
    const float *conf;
    const uint8_t *mask;
    const int *M;  // number of counted steps
    float ce_alpha, l1_alpha, conf_alpha;
    __nv_bfloat16 *grad;  // [R, V] or null
    float *grad_conf;     // [R] or null
    float *stats;         // [R, 4]: CE, L1, BCE, a
    uint32_t *err;
    uint64_t wait_ns;
};

__device__ __forceinline__ void unpack8(const uint4 &v, float (&x)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// Block-wide reduction of kN values per thread (op: 0 = sum, 1 = max):
// warp partials in red, warp 0 combines them and leaves the results in
// res[0..kN), which every thread then reads.
template <int kN>
__device__ __forceinline__ void block_reduce(float (&v)[kN], int op, float (*red)[4], float *res) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < kN; i++)
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) {
            const float o = __shfl_xor_sync(0xffffffffu, v[i], d);
            v[i] = op ? fmaxf(v[i], o) : v[i] + o;
        }
    if (lane == 0)
#pragma unroll
        for (int i = 0; i < kN; i++) red[warp][i] = v[i];
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int i = 0; i < kN; i++) {
            float a = lane < kWarps ? red[lane][i] : (op ? -INFINITY : 0.f);
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) {
                const float o = __shfl_xor_sync(0xffffffffu, a, d);
                a = op ? fmaxf(a, o) : a + o;
            }
            if (lane == 0) res[i] = a;
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kN; i++) v[i] = res[i];
}

// Bounded wait for a row's copies (once per row, so the clock is read at every
// poll): gives up when the CTA's abort flag is raised or after limit_ns (then
// raises it). Returns false when it gave up. try_wait may suspend the thread
// for a while before it reports "not yet", which is what the waiting warps
// should do while the SM's other CTA computes; a limit below 1 ms is honoured
// by polling without suspending instead.
__device__ __forceinline__ bool wait_row(uint64_t *bar, uint32_t parity, volatile int *abort_flag, uint64_t limit_ns) {
    const bool fine = limit_ns < 1000000ull;
    const uint64_t t0 = tc::globaltimer();
    for (;;) {
        if (fine ? tc::mbar_test(bar, parity) : tc::mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (tc::globaltimer() - t0 > limit_ns) {
            *abort_flag = 1;
            return false;
        }
    }
}

// Merge of per-thread (max m, sum z of exp(x - m)) pairs for two quantities
// over the CTA: each warp takes its maximum and rescales its sums to it, then
// warp 0 merges the warps' pairs; res[0..3] = (m0, z0, m1, z1) for every thread.
__device__ __forceinline__ void block_merge_mz(float (&m)[2], float (&z)[2], float (*red)[4], float *res) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int k = 0; k < 2; k++) {
        float M = m[k];
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, d));
        float zz = m[k] > -INFINITY ? z[k] * tc::ex2((m[k] - M) * kLog2e) : 0.f;
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) zz += __shfl_xor_sync(0xffffffffu, zz, d);
        m[k] = M;
        z[k] = zz;
    }
    if (lane == 0) {
        red[warp][0] = m[0];
        red[warp][1] = z[0];
        red[warp][2] = m[1];
        red[warp][3] = z[1];
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int k = 0; k < 2; k++) {
            const float wm = lane < kWarps ? red[lane][2 * k] : -INFINITY;
            const float wz = lane < kWarps ? red[lane][2 * k + 1] : 0.f;
            float M = wm;
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, d));
            float zz = wm > -INFINITY ? wz * tc::ex2((wm - M) * kLog2e) : 0.f;
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) zz += __shfl_xor_sync(0xffffffffu, zz, d);
            if (lane == 0) {
                res[2 * k] = M;
                res[2 * k + 1] = zz;
            }
        }
    }
    __syncthreads();
    m[0] = res[0];
    z[0] = res[1];
    m[1] = res[2];
    z[1] = res[3];
}

__global__ void __launch_bounds__(kThr, 2) k_dspark_loss(const LossArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((128u - (tc::smem_u32(smem_raw) & 127u)) & 127u);
    __nv_bfloat16 *buf = reinterpret_cast<__nv_bfloat16 *>(sm);  // [kBufs][L | T][seg]
    __shared__ float red[kWarps][4];
    __shared__ float res[4];  // block results, then the row's exchanged values
    __shared__ float x1[6];  // this CTA's max L, sum L, max T, sum T, L[y], has y
    __shared__ float x2[2];  // this CTA's L1 and sum s p
    __shared__ __align__(8) uint64_t full[2];
    __shared__ int abort_s;

    cg::cluster_group cluster = cg::this_cluster();
    const int j = (int)cluster.block_rank();
    const int cid = (int)blockIdx.x / kCl, ncl = (int)gridDim.x / kCl;
    const int e0 = j * p.seg, len = max(0, min(p.V, e0 + p.seg) - e0);  // this CTA's elements
    const int nv = len / 8;                                             // 16-byte vectors
    if (threadIdx.x == 0) {
        tc::mbar_init(&full[0], 1);
        tc::mbar_init(&full[1], 1);
        abort_s = 0;
        tc::fence_barrier_init();
    }
    __syncthreads();
    volatile int *abort_flag = &abort_s;
    const int M = *p.M;
    auto issue = [&](int row, int b) {  // thread 0: the row's two slices into buffer b
        uint64_t *bar = &full[b];
        tc::mbar_arrive_expect_tx(bar, (uint32_t)(4 * len));
        if (len > 0) {
            const size_t off = (size_t)row * p.V + e0;
            tc::bulk_load(buf + (size_t)(2 * b) * p.seg, p.L + off, (uint32_t)(2 * len), bar);
            tc::bulk_load(buf + (size_t)(2 * b + 1) * p.seg, p.T + off, (uint32_t)(2 * len), bar);
        }
    };
    int issued = 0, waited = 0;  // row loads issued / completed (thread 0's count)
    if (kBufs == 2 && threadIdx.x == 0 && cid < p.R) {
        issue(cid, 0);
        issued = 1;
    }
    int it = 0;
    for (int r = cid; r < p.R; r += ncl, ++it) {
        const int b = kBufs == 2 ? (it & 1) : 0;
        // every thread is done with the buffer the next copy fills (the
        // previous row's), then the copies of the row after (two buffers) or
        // of this row (one buffer)
        __syncthreads();
        if (threadIdx.x == 0 && !*abort_flag) {
            if (kBufs == 2 && r + ncl < p.R) {
                tc::fence_proxy_async_smem();
                issue(r + ncl, b ^ 1);
                issued = it + 2;
            } else if (kBufs == 1) {
                tc::fence_proxy_async_smem();
                issue(r, 0);
                issued = it + 1;
            }
        }
        const uint32_t ph = kBufs == 2 ? (uint32_t)((it >> 1) & 1) : (uint32_t)(it & 1);
        bool ok = !*abort_flag && tc::warp_all(wait_row(&full[b], ph, abort_flag, p.wait_ns));
        if (threadIdx.x == 0 && ok) waited = it + 1;
        const uint4 *Lv = reinterpret_cast<const uint4 *>(buf + (size_t)(2 * b) * p.seg);
        const uint4 *Tv = reinterpret_cast<const uint4 *>(buf + (size_t)(2 * b + 1) * p.seg);
        const int y = p.labels[r];
        const bool yvalid = y >= 0 && y < p.V;
        // this CTA's maxima and sums of exp(x - max) in one pass (each thread
        // keeps a running maximum and rescales its sum when it grows), and
        // L[y] if it holds y
        float tm[2] = {-INFINITY, -INFINITY}, tz[2] = {0.f, 0.f};
        for (int v = threadIdx.x; v < nv; v += kThr) {
            float a[8], c[8];
            unpack8(Lv[v], a);
            unpack8(Tv[v], c);
            float va = a[0], vc = c[0];
#pragma unroll
            for (int i = 1; i < 8; i++) {
                va = fmaxf(va, a[i]);
                vc = fmaxf(vc, c[i]);
            }
            if (va > tm[0]) {
                tz[0] *= tc::ex2((tm[0] - va) * kLog2e);
                tm[0] = va;
            }
            if (vc > tm[1]) {
                tz[1] *= tc::ex2((tm[1] - vc) * kLog2e);
                tm[1] = vc;
            }
            const float ma = tm[0] * kLog2e, mc = tm[1] * kLog2e;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                tz[0] += tc::ex2(fmaf(a[i], kLog2e, -ma));
                tz[1] += tc::ex2(fmaf(c[i], kLog2e, -mc));
            }
        }
        float mx[2] = {tm[0], tm[1]}, zs[2] = {tz[0], tz[1]};
        block_merge_mz(mx, zs, red, res);
        if (threadIdx.x == 0) {
            const bool mine = yvalid && y >= e0 && y < e0 + len;
            x1[0] = mx[0];
            x1[1] = zs[0];
            x1[2] = mx[1];
            x1[3] = zs[1];
            x1[4] = mine ? __bfloat162float(buf[(size_t)(2 * b) * p.seg + (y - e0)]) : 0.f;
            x1[5] = mine ? 1.f : 0.f;
        }
        cluster.sync();  // #A: every CTA's x1 is visible
        // the row's normalisers (log2 domain) and L[y]: lane k of warp 0 reads
        // CTA k's values, the warp combines them
        if (threadIdx.x < 32) {
            const int k = threadIdx.x;
            float q[6] = {-INFINITY, 0.f, -INFINITY, 0.f, 0.f, 0.f};
            if (k < kCl) {
                const float *px = cluster.map_shared_rank(x1, k);
#pragma unroll
                for (int i = 0; i < 6; i++) q[i] = px[i];
            }
            float mLg = q[0], mTg = q[2];
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) {
                mLg = fmaxf(mLg, __shfl_xor_sync(0xffffffffu, mLg, d));
                mTg = fmaxf(mTg, __shfl_xor_sync(0xffffffffu, mTg, d));
            }
            float zl = q[1] > 0.f ? q[1] * tc::ex2((q[0] - mLg) * kLog2e) : 0.f;
            float zt = q[3] > 0.f ? q[3] * tc::ex2((q[2] - mTg) * kLog2e) : 0.f;
            float ly = q[5] != 0.f ? q[4] : 0.f;
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) {
                zl += __shfl_xor_sync(0xffffffffu, zl, d);
                zt += __shfl_xor_sync(0xffffffffu, zt, d);
                ly += __shfl_xor_sync(0xffffffffu, ly, d);
            }
            if (k == 0) {
                res[0] = mLg * kLog2e + log2f(zl);  // log2 of the row's sums
                res[1] = mTg * kLog2e + log2f(zt);
                res[2] = ly;
            }
        }
        __syncthreads();
        const float lseL2 = res[0], lseT2 = res[1], Ly = res[2];
        // L1 and sum_i s_i p_i over this CTA's elements; p (bf16) and s = sign(p - q)
        // replace the slices' logits for the gradient pass (L[y] was taken above)
        float acc[2] = {0.f, 0.f};
        uint4 *Lw = reinterpret_cast<uint4 *>(buf + (size_t)(2 * b) * p.seg);
        uint4 *Tw = reinterpret_cast<uint4 *>(buf + (size_t)(2 * b + 1) * p.seg);
        for (int v = threadIdx.x; v < nv; v += kThr) {
            float a[8], c[8], pv[8], sv[8];
            unpack8(Lv[v], a);
            unpack8(Tv[v], c);
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const float la = fmaf(a[i], kLog2e, -lseL2), lc = fmaf(c[i], kLog2e, -lseT2);
                const float pi = tc::ex2(la), qi = tc::ex2(lc);
                const float si = la > lc ? 1.f : (la < lc ? -1.f : 0.f);
                acc[0] += fabsf(pi - qi);
                acc[1] += si * pi;
                pv[i] = pi;
                sv[i] = si;
            }
            Lw[v] = make_uint4(tc::pack_bf16x2(pv[0], pv[1]), tc::pack_bf16x2(pv[2], pv[3]),
                               tc::pack_bf16x2(pv[4], pv[5]), tc::pack_bf16x2(pv[6], pv[7]));
            Tw[v] = make_uint4(tc::pack_bf16x2(sv[0], sv[1]), tc::pack_bf16x2(sv[2], sv[3]),
                               tc::pack_bf16x2(sv[4], sv[5]), tc::pack_bf16x2(sv[6], sv[7]));
        }
        tc::fence_proxy_async_smem();  // these writes precede the copy that refills the buffer
        block_reduce<2>(acc, 0, red, res);
        if (threadIdx.x == 0) {
            x2[0] = acc[0];
            x2[1] = acc[1];
        }
        cluster.sync();  // #B: every CTA's x2 is visible
        if (threadIdx.x < 32) {
            const int k = threadIdx.x;
            float l1 = 0.f, sb = 0.f;
            if (k < kCl) {
                const float *px = cluster.map_shared_rank(x2, k);
                l1 = px[0];
                sb = px[1];
            }
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) {
                l1 += __shfl_xor_sync(0xffffffffu, l1, d);
                sb += __shfl_xor_sync(0xffffffffu, sb, d);
            }
            if (k == 0) {
                res[0] = l1;
                res[1] = sb;
            }
        }
        __syncthreads();
        const float L1 = res[0], Sb = res[1];
        const float a_t = fminf(fmaxf(1.f - 0.5f * L1, 0.f), 1.f);
        const float w = (p.mask[r] && M > 0) ? 1.f / (float)M : 0.f;
        if (p.grad) {
            // d/dL_i = w (ce_alpha (p_i - [i = y]) + l1_alpha p_i (s_i - Sb))
            // (a label outside [0, V) adds no CE term, so no CE gradient either)
            const float cw = yvalid ? w * p.ce_alpha : 0.f, lw = w * p.l1_alpha;
            uint4 *G = reinterpret_cast<uint4 *>(p.grad + (size_t)r * p.V + e0);
            for (int v = threadIdx.x; v < nv; v += kThr) {
                float pv[8], sv[8];
                unpack8(Lv[v], pv);  // p and s stored by the L1 pass
                unpack8(Tv[v], sv);
                float g[8];
#pragma unroll
                for (int i = 0; i < 8; i++) g[i] = pv[i] * (cw + lw * (sv[i] - Sb));
                const int ky = y - e0 - 8 * v;  // y's place in this vector, if there
                if (yvalid && ky >= 0 && ky < 8) {
#pragma unroll
                    for (int i = 0; i < 8; i++)
                        if (i == ky) g[i] -= cw;
                }
                G[v] = make_uint4(tc::pack_bf16x2(g[0], g[1]), tc::pack_bf16x2(g[2], g[3]),
                                  tc::pack_bf16x2(g[4], g[5]), tc::pack_bf16x2(g[6], g[7]));
            }
        }
        if (j == 0 && threadIdx.x == 0) {
            const float c = p.conf[r];
            const float ce = yvalid ? (lseL2 * kLn2 - Ly) : 0.f;
            const float bce = fmaxf(c, 0.f) - c * a_t + log1pf(expf(-fabsf(c)));
            float4 st = make_float4(ce, L1, bce, a_t);
            reinterpret_cast<float4 *>(p.stats)[r] = st;
            if (p.grad_conf) p.grad_conf[r] = w * p.conf_alpha * (1.f / (1.f + expf(-c)) - a_t);
        }
        (void)ok;
    }
    // copies still in flight after a wait gave up, then no CTA leaves while a
    // peer may still read its shared memory
    if (threadIdx.x == 0 && *abort_flag) {
        volatile int never = 0;
        for (int t = waited; t < issued; ++t)
            tc::mbar_wait(&full[kBufs == 2 ? (t & 1) : 0], kBufs == 2 ? (t >> 1) & 1 : t & 1, &never);
        atomicOr(p.err, kErrTimeout);
    }
    cluster.sync();
}

__global__ void k_loss_count(const uint8_t *mask, int R, int *M) {
    int c = 0;
    for (int i = threadIdx.x; i < R; i += blockDim.x) c += mask[i] != 0;
    for (int d = 16; d > 0; d >>= 1) c += __shfl_xor_sync(0xffffffffu, c, d);
    __shared__ int part[32];
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = c;
    __syncthreads();
    if (threadIdx.x == 0) {
        int t = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); w++) t += part[w];
        *M = t;
    }
}

// Means over the counted steps in a fixed order (deterministic): out = total,
// CE mean, L1 mean, BCE mean.
__global__ void k_loss_finish(const float *stats, const uint8_t *mask, int R, const int *M, float ce_alpha,
                              float l1_alpha, float conf_alpha, float *out) {
    __shared__ double part[3][256];
    double s[3] = {0, 0, 0};
    for (int i = threadIdx.x; i < R; i += blockDim.x)
        if (mask[i])
            for (int k = 0; k < 3; k++) s[k] += stats[4 * (size_t)i + k];
    for (int k = 0; k < 3; k++) part[k][threadIdx.x] = s[k];
    __syncthreads();
    if (threadIdx.x == 0) {
        double t[3] = {0, 0, 0};
        for (int i = 0; i < (int)blockDim.x; i++)
            for (int k = 0; k < 3; k++) t[k] += part[k][i];
        const int m = *M;
        const double ce = m ? t[0] / m : 0.0, l1 = m ? t[1] / m : 0.0, cf = m ? t[2] / m : 0.0;
        out[0] = (float)(ce_alpha * ce + l1_alpha * l1 + conf_alpha * cf);
        out[1] = (float)ce;
        out[2] = (float)l1;
        out[3] = (float)cf;
    }
}

}  // namespace

size_t loss_workspace_size(int R) { return 256 + align256(sizeof(float) * 4 * (size_t)(R > 0 ? R : 0)); }

int loss_seg(int V) { return ((V + kCl - 1) / kCl + 7) / 8 * 8; }

cudaError_t launch_loss(int R, int V, const void *L, const void *T, const int32_t *labels, const float *conf,
                        const uint8_t *mask, float ce_alpha, float l1_alpha, float conf_alpha, float *out,
                        void *grad, float *grad_conf, void *ws, uint64_t wait_ns, cudaStream_t st) {
    // the error word at offset 0, as in every workspace of this library
    uint32_t *err = reinterpret_cast<uint32_t *>(ws);
    int *M = reinterpret_cast<int *>(reinterpret_cast<char *>(ws) + 128);
    float *stats = reinterpret_cast<float *>(reinterpret_cast<char *>(ws) + 256);
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
    count_launch();
    k_loss_count<<<1, 1024, 0, st>>>(mask, R, M);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (R > 0) {
        LossArgs a;
        a.R = R;
        a.V = V;
        a.seg = loss_seg(V);
        a.L = (const __nv_bfloat16 *)L;
        a.T = (const __nv_bfloat16 *)T;
        a.labels = labels;
        a.conf = conf;
        a.mask = mask;
        a.M = M;
        a.ce_alpha = ce_alpha;
        a.l1_alpha = l1_alpha;
        a.conf_alpha = conf_alpha;
        a.grad = (__nv_bfloat16 *)grad;
        a.grad_conf = grad_conf;
        a.stats = stats;
        a.err = err;
        a.wait_ns = wait_ns;
        const size_t smem = (size_t)4 * kBufs * a.seg + 128;
        if ((e = cudaFuncSetAttribute(k_dspark_loss, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
            cudaSuccess)
            return e;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kCl;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cfg.blockDim = dim3(kThr);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cfg.gridDim = dim3(kCl);
        int ncl = 0;
        if ((e = cudaOccupancyMaxActiveClusters(&ncl, k_dspark_loss, &cfg)) != cudaSuccess) return e;
        if (ncl < 1) return cudaErrorInvalidConfiguration;
        ncl = std::min(ncl, R);
        cfg.gridDim = dim3(ncl * kCl);
        count_launch();
        if ((e = cudaLaunchKernelEx(&cfg, k_dspark_loss, a)) != cudaSuccess) return e;
    }
    count_launch();
    k_loss_finish<<<1, 256, 0, st>>>(stats, mask, R, M, ce_alpha, l1_alpha, conf_alpha, out);
    return cudaGetLastError();
}

}  // namespace dspark
