// Tensor-core (tcgen05 / TMEM / TMA) backward of the DSpark draft attention for
// the page's head widths (d_c = 192, d_r = 64, d_v = 256), bf16.
//
// The gradient of softmax(Q K^T s + Lambda(M)) V (appendix "Attention
// implementation" of the "GLM 5.2 DSpark speculative-training design" page,
// with the §3 mask) for the loss with dL/dO = dO:
//   P = exp(S - LSE), dP = dO V^T, D = rowsum(dO * O), dS = P * (dP - D) * s,
//   dQ = dS K, dK = dS^T Q, dV = P^T dO,
// on rotated q and k rope slices; the rope parts of dQ and dK are rotated back,
// and dK^R, shared by every head (§4), is the sum over heads.
//
// Launch sequence (one stream; the padding blocks' dq rows and draft-key
// dK^C / dV are zeroed earlier, by the rope-key rotation launch):
//   1. k_bwd_prep       per kept block and head group: rotated Q and
//                       dO copied into anchor-sorted row order, D, LSE*log2(e),
//                       and the whole backward of the block's own 5 draft keys
//                       (5 x 5 per head, on the CUDA cores): their dK^C, dV and
//                       the group's partial dK^R, and the rows' draft-key dQ
//                       contribution, stored as the first value of the fp32 dQ
//                       accumulator (anchor-sorted rows).
//   2. k_bwd_tc         key-major over the context, one CTA per (b, 64-key
//                       tile, head group), one pass over K and V: rows of the
//                       blocks whose windows meet the tile, in chunks of 64.
//                       S^T = K Q^T and dP^T = V dO^T in TMEM, P^T and dS^T
//                       through shared memory, dV += P^T dO and dK += dS^T Q
//                       accumulated in TMEM over the rows (M = 64 accumulators:
//                       dK and dV share TMEM columns, one in each half of the
//                       lanes), and the chunk's dQ contribution dS K in TMEM,
//                       added into the dQ accumulator with vector reductions.
//                       dK and dV are written once, by the CTA that owns the
//                       keys (no atomics).
//   3. k_bwd_dq_out     rotates the rope part of the accumulated dQ back,
//                       rounds to bf16 and writes dq in the caller's row order.
//   4. k_bwd_dkr_reduce sums the per-head-group rope-key partials, rotates
//                       them back and writes dK^R.
// The blocks whose windows meet a context tile [t0, t0 + 64) are a contiguous
// run of the anchor-sorted list (t0 < A <= t0 + 63 + W - 1).
#include <algorithm>

#include "dspark_tc_common.cuh"

namespace dspark {

namespace {

using namespace tc;

constexpr int kDC = 192, kDR = 64, kDQK = 256, kDV = 256;
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ prep
// The row-wise preparation and the draft-key part of the backward, one CTA
// per kept block (anchor-sorted index i), group of up to kHeads heads and
// batch row. A producer warp stages each head's inputs into shared memory with
// bulk copies (ring of kStages heads): the block's 5 rows of q, O and dO and
// its 5 draft keys' K^C and V (the rotated rope keys of the draft keys are the
// same for all heads and are staged once). Compute warp w takes the heads
// w, w + kWarps, ... of the group, one whole block per head, lane l owning
// dims 8 l .. 8 l + 7 of every row (rows 5 n + r, r = 0..4) and key:
//   - rotated q -> qs (and back into the stage), dO -> dos (anchor-sorted rows);
//   - the 55 partial sums of S = q_rot k_rot^T, dP = dO V^T over the block's
//     own 5 draft keys (which no other row sees, page §3) and D = rowsum(dO * O),
//     reduced across the warp in one butterfly that leaves sums 2 l, 2 l + 1 in
//     lane l; then P = exp(S s - LSE), dS = P (dP - D) s for the 25 pairs;
//   - the rows' draft-key dQ contribution dS K_rot, stored as the first value
//     of the fp32 dQ accumulator (the context tiles add theirs later, in
//     stream order), D and LSE * log2(e);
//   - the draft keys' gradients, complete here: dK^C = dS^T q_rot and
//     dV = P^T dO written, the rope part of dK summed over the group's heads
//     in shared memory and written, after the last head, as the group's partial
//     rope-key gradient (rotated frame; k_bwd_dkr_reduce sums the groups).
// q_rot is rounded to bf16 as the tensor-core kernels see it (the forward's
// LSE was formed from the same rounded operands). Rows past the kept blocks
// are zeroed so that tiles overhanging them multiply finite values. Every
// wait is bounded; on time-out the CTA stops issuing, waits (bounded) for its
// copies in flight and sets the timeout bit of the error word; the compute
// warps meet at one barrier only, after their loops.
namespace pr {
// Barrier 1 of the compute warps with an OR over their predicates: every warp
// gets the same answer from one barrier instance.
__device__ __forceinline__ bool compute_warps_or(bool x, int nthreads) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)x), "r"(nthreads)
        : "memory");
    return r != 0;
}
constexpr int kWarps = 4;                  // compute warps
constexpr int kHeads = 16;                 // heads per CTA at most
constexpr int kStages = 4;                 // staged heads
constexpr int kRowsB = kBlock * kDQK * 2;  // 5 rows of 256 bf16 (q, O, dO, V)
constexpr int kKcB = kBlock * kDC * 2;     // 5 rows of K^C
constexpr int oQ = 0, oO = kRowsB, oDO = 2 * kRowsB, oV = 3 * kRowsB, oKc = 4 * kRowsB;
constexpr int kStageB = 4 * kRowsB + kKcB;  // 12160
constexpr int kThreads = (kWarps + 1) * 32;
constexpr int kSmem = kStages * kStageB + 128;  // dynamic: the stages (+ alignment)
}  // namespace pr

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__global__ void __launch_bounds__(pr::kThreads, 4) k_bwd_prep(int n_h, int S, int N, int L, float scale, float scale_log2,
                                                  const __nv_bfloat16 *__restrict__ q,
                                                  const __nv_bfloat16 *__restrict__ kc,
                                                  const __nv_bfloat16 *__restrict__ krr,
                                                  const __nv_bfloat16 *__restrict__ v,
                                                  const __nv_bfloat16 *__restrict__ o,
                                                  const __nv_bfloat16 *__restrict__ dout,
                                                  const float *__restrict__ lse, const int32_t *__restrict__ cnt,
                                                  const int32_t *__restrict__ sorted_n,
                                                  const int32_t *__restrict__ sorted_a,
                                                  const float2 *__restrict__ tab, __nv_bfloat16 *__restrict__ qs,
                                                  __nv_bfloat16 *__restrict__ dos, float *__restrict__ ds_,
                                                  float *__restrict__ lses, float *__restrict__ dqacc,
                                                  __nv_bfloat16 *__restrict__ dkc, float *__restrict__ dkr_part,
                                                  __nv_bfloat16 *__restrict__ dv, uint32_t *err,
                                                  uint64_t wlim) {
    using namespace pr;
    extern __shared__ uint8_t prep_smem[];
    uint8_t *st0 = prep_smem + ((128u - (tc::smem_u32(prep_smem) & 127u)) & 127u);
    __shared__ __align__(16) uint4 s_kr[kBlock][8];         // rotated rope keys of the draft keys
    __shared__ __align__(16) float s_tot[kWarps][64];        // the warp's reduced sums
    __shared__ float s_p[kWarps][kBlock * kBlock], s_ds[kWarps][kBlock * kBlock];  // [row * 5 + key]
    __shared__ __align__(16) float s_dkr[kWarps][kBlock][kDR];  // rope part of dK, summed over the warp's heads
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages], krbar;
    __shared__ int abort_s;
    const int i = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = kBlock * N;
    const int h0 = hg * kHeads, nhh = min(kHeads, n_h - h0);  // the group's heads
    pdl_wait();
    if (i >= cnt[b]) {
        for (int hh = w; hh < nhh; hh += kWarps + 1)
            for (int r = 0; r < kBlock; r++) {
                const size_t srow = ((size_t)b * n_h + h0 + hh) * R + kBlock * i + r;
                reinterpret_cast<uint4 *>(qs + srow * kDQK)[lane] = make_uint4(0, 0, 0, 0);
                reinterpret_cast<uint4 *>(dos + srow * kDV)[lane] = make_uint4(0, 0, 0, 0);
                if (lane == 0) {
                    ds_[srow] = 0.f;
                    lses[srow] = 0.f;
                }
            }
        return;
    }
    const int n = sorted_n[(size_t)b * N + i], a = sorted_a[(size_t)b * N + i];
    const size_t key0 = (size_t)S + kBlock * n;  // the block's first draft key
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; s++) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        tc::mbar_init(&krbar, 1);
        abort_s = 0;
        tc::fence_barrier_init();
    }
    for (int e = threadIdx.x; e < kWarps * kBlock * kDR; e += blockDim.x) (&s_dkr[0][0][0])[e] = 0.f;
    __syncthreads();
    volatile int *abort_flag = &abort_s;
    if (w == kWarps) {
        // ---------------------------------------------------- producer
        int issued = 0;
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(&krbar, kBlock * kDR * 2);
            tc::bulk_load(&s_kr[0][0], krr + ((size_t)b * L + key0) * kDR, kBlock * kDR * 2, &krbar);
            for (int hh = 0; hh < nhh; hh++) {
                const int s = hh % kStages;
                if (hh >= kStages && !tc::mbar_wait(&empty[s], ((hh / kStages) - 1) & 1, abort_flag, wlim)) break;
                const size_t bh = (size_t)b * n_h + h0 + hh;
                const size_t orow = (bh * R + kBlock * n) * kDQK, krow = bh * L + key0;
                uint8_t *d = st0 + s * kStageB;
                tc::mbar_arrive_expect_tx(&full[s], kStageB);
                tc::bulk_load(d + oQ, q + orow, kRowsB, &full[s]);
                tc::bulk_load(d + oO, o + orow, kRowsB, &full[s]);
                tc::bulk_load(d + oDO, dout + orow, kRowsB, &full[s]);
                tc::bulk_load(d + oV, v + krow * kDV, kRowsB, &full[s]);
                tc::bulk_load(d + oKc, kc + krow * kDC, kKcB, &full[s]);
                issued = hh + 1;
            }
        }
        // every copy issued has landed before the CTA may end (each wait bounded)
        __syncwarp();
        if (lane == 0) {
            volatile int never = 0;
            tc::mbar_wait(&krbar, 0, &never);
            for (int hh = max(0, issued - kStages); hh < issued; hh++)
                tc::mbar_wait(&full[hh % kStages], (hh / kStages) & 1, &never);
        }
        __syncthreads();
        if (threadIdx.x == kWarps * 32 && abort_s) atomicOr(err, kErrTimeout);
        return;
    }
    // ---------------------------------------------------- compute warps
    // RoPE (cos, sin) of this lane's 4 frequencies (lanes 24-31) at position a + r
    const float2 *cs0 = tab + (size_t)a * (kDR / 2) + (lane >= 24 ? (lane - 24) * 4 : 0);
    bool ok = tc::warp_all(tc::mbar_wait(&krbar, 0, abort_flag, wlim));
    // LSE of the warp's next head (lanes 0-4: rows 0-4), read a head ahead
    float lse_n = (ok && w < nhh && lane < kBlock) ? lse[((size_t)b * n_h + h0 + w) * R + kBlock * n + lane] : 0.f;
    for (int hh = w; hh < nhh && ok; hh += kWarps) {
        const int s = hh % kStages;
        const size_t bh = (size_t)b * n_h + h0 + hh;
        const float lse_r = lse_n;
        if (hh + kWarps < nhh && lane < kBlock) lse_n = lse[(bh + kWarps) * R + kBlock * n + lane];
        ok = tc::warp_all(tc::mbar_wait(&full[s], (hh / kStages) & 1, abort_flag, wlim));
        if (!ok) break;
        uint8_t *d = st0 + s * kStageB;
        // the 55 partial sums: S[r][k] at 5 r + k, dP[r][k] at 25 + 5 r + k, D[r] at 50 + r
        float acc[64];
#pragma unroll
        for (int e = 0; e < 64; e++) acc[e] = 0.f;
#pragma unroll
        for (int r = 0; r < kBlock; r++) {
            uint4 qv = reinterpret_cast<const uint4 *>(d + oQ + r * kDQK * 2)[lane];
            if (lane >= 24) {
                uint32_t wq[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
                for (int f = 0; f < 4; f++) {
                    const float2 c = __ldg(cs0 + r * (kDR / 2) + f);
                    const float x0 = bf_lo(wq[f]), x1 = bf_hi(wq[f]);
                    wq[f] = pack_bf16x2(x0 * c.x - x1 * c.y, x0 * c.y + x1 * c.x);
                }
                qv = make_uint4(wq[0], wq[1], wq[2], wq[3]);
                reinterpret_cast<uint4 *>(d + oQ + r * kDQK * 2)[lane] = qv;  // rotated, for dK below
            }
            const uint4 dv4 = reinterpret_cast<const uint4 *>(d + oDO + r * kDV * 2)[lane];
            const uint4 ov4 = reinterpret_cast<const uint4 *>(d + oO + r * kDV * 2)[lane];
            const size_t srow = bh * R + kBlock * i + r;
            reinterpret_cast<uint4 *>(qs + srow * kDQK)[lane] = qv;
            reinterpret_cast<uint4 *>(dos + srow * kDV)[lane] = dv4;
            const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w}, dw[4] = {dv4.x, dv4.y, dv4.z, dv4.w};
            const uint32_t ow[4] = {ov4.x, ov4.y, ov4.z, ov4.w};
#pragma unroll
            for (int f = 0; f < 4; f++) {
                acc[50 + r] = fmaf(bf_lo(dw[f]), bf_lo(ow[f]), acc[50 + r]);
                acc[50 + r] = fmaf(bf_hi(dw[f]), bf_hi(ow[f]), acc[50 + r]);
            }
#pragma unroll
            for (int k = 0; k < kBlock; k++) {
                const uint4 kq = lane < 24 ? reinterpret_cast<const uint4 *>(d + oKc + k * kDC * 2)[lane] : s_kr[k][lane - 24];
                const uint4 vv = reinterpret_cast<const uint4 *>(d + oV + k * kDV * 2)[lane];
                const uint32_t kw[4] = {kq.x, kq.y, kq.z, kq.w}, vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
                for (int f = 0; f < 4; f++) {
                    acc[5 * r + k] = fmaf(bf_lo(qw[f]), bf_lo(kw[f]), acc[5 * r + k]);
                    acc[5 * r + k] = fmaf(bf_hi(qw[f]), bf_hi(kw[f]), acc[5 * r + k]);
                    acc[25 + 5 * r + k] = fmaf(bf_lo(dw[f]), bf_lo(vw[f]), acc[25 + 5 * r + k]);
                    acc[25 + 5 * r + k] = fmaf(bf_hi(dw[f]), bf_hi(vw[f]), acc[25 + 5 * r + k]);
                }
            }
        }
        // butterfly reduce-scatter over the warp: at each step keep one half of
        // the values (the upper one if this lane's bit is set) and add the
        // partner's; lane l ends with the sums of values 2 l and 2 l + 1
#pragma unroll
        for (int step = 0; step < 5; step++) {
            const int bit = 16 >> step, half = 32 >> step;
            const bool up = lane & bit;
#pragma unroll
            for (int e = 0; e < half; e++) {
                const float send = up ? acc[e] : acc[e + half];
                const float keep = up ? acc[e + half] : acc[e];
                acc[e] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
            }
        }
        s_tot[w][2 * lane] = acc[0];
        s_tot[w][2 * lane + 1] = acc[1];
        __syncwarp();
        if (lane < kBlock * kBlock) {
            const int r = lane / kBlock;
            const float lse2 = __shfl_sync(0x1ffffffu, lse_r, r) * kLog2e;
            const float pr = exp2f(fmaf(s_tot[w][lane], scale_log2, -lse2));
            s_p[w][lane] = pr;
            s_ds[w][lane] = pr * (s_tot[w][25 + lane] - s_tot[w][50 + r]) * scale;
        }
        if (lane < kBlock) {
            const size_t srow = bh * R + kBlock * i + lane;
            ds_[srow] = s_tot[w][50 + lane];
            lses[srow] = lse_r * kLog2e;
        }
        __syncwarp();
        // the rows' draft-key dQ contribution: dq[r] = sum_k dS[r][k] k_rot[k]
        {
            float kf[kBlock][8];
#pragma unroll
            for (int k = 0; k < kBlock; k++) {
                const uint4 kq = lane < 24 ? reinterpret_cast<const uint4 *>(d + oKc + k * kDC * 2)[lane] : s_kr[k][lane - 24];
                const uint32_t kw[4] = {kq.x, kq.y, kq.z, kq.w};
#pragma unroll
                for (int f = 0; f < 4; f++) {
                    kf[k][2 * f] = bf_lo(kw[f]);
                    kf[k][2 * f + 1] = bf_hi(kw[f]);
                }
            }
#pragma unroll
            for (int r = 0; r < kBlock; r++) {
                float dq8[8] = {};
#pragma unroll
                for (int k = 0; k < kBlock; k++) {
                    const float dsk = s_ds[w][kBlock * r + k];
#pragma unroll
                    for (int e = 0; e < 8; e++) dq8[e] = fmaf(dsk, kf[k][e], dq8[e]);
                }
                float4 *acc4 = reinterpret_cast<float4 *>(dqacc + (bh * R + kBlock * i + r) * kDQK) + 2 * lane;
                acc4[0] = make_float4(dq8[0], dq8[1], dq8[2], dq8[3]);
                acc4[1] = make_float4(dq8[4], dq8[5], dq8[6], dq8[7]);
            }
        }
        // the draft keys' gradients, one pass each: dK[k] = sum_r dS[r][k] q_rot[r],
        // then dV[k] = sum_r P[r][k] dO[r]
#pragma unroll
        for (int pass = 0; pass < 2; pass++) {
            const int off = pass == 0 ? oQ : oDO;
            const float *wgt = pass == 0 ? s_ds[w] : s_p[w];
            float g[kBlock][8] = {};
#pragma unroll
            for (int r = 0; r < kBlock; r++) {
                const uint4 x4 = reinterpret_cast<const uint4 *>(d + off + r * kDQK * 2)[lane];
                const uint32_t xw[4] = {x4.x, x4.y, x4.z, x4.w};
                float xf[8];
#pragma unroll
                for (int f = 0; f < 4; f++) {
                    xf[2 * f] = bf_lo(xw[f]);
                    xf[2 * f + 1] = bf_hi(xw[f]);
                }
#pragma unroll
                for (int k = 0; k < kBlock; k++) {
                    const float wk = wgt[kBlock * r + k];
#pragma unroll
                    for (int e = 0; e < 8; e++) g[k][e] = fmaf(wk, xf[e], g[k][e]);
                }
            }
            if (pass == 1) {
                // the stage is no longer read (and its rotated q, written here,
                // precedes the bulk copy that will refill it)
                tc::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&empty[s]);
            }
#pragma unroll
            for (int k = 0; k < kBlock; k++) {
                const size_t krow = bh * L + key0 + k;
                const uint4 pk = make_uint4(pack_bf16x2(g[k][0], g[k][1]), pack_bf16x2(g[k][2], g[k][3]),
                                            pack_bf16x2(g[k][4], g[k][5]), pack_bf16x2(g[k][6], g[k][7]));
                if (pass == 1) {
                    reinterpret_cast<uint4 *>(dv + krow * kDV)[lane] = pk;
                } else if (lane < 24) {
                    reinterpret_cast<uint4 *>(dkc + krow * kDC)[lane] = pk;
                } else {
                    float4 *acc4 = reinterpret_cast<float4 *>(&s_dkr[w][k][8 * (lane - 24)]);
                    const float4 x = acc4[0], y = acc4[1];
                    acc4[0] = make_float4(x.x + g[k][0], x.y + g[k][1], x.z + g[k][2], x.w + g[k][3]);
                    acc4[1] = make_float4(y.x + g[k][4], y.y + g[k][5], y.z + g[k][6], y.w + g[k][7]);
                }
            }
        }
    }
    // the compute warps meet once; unless one gave up, the draft keys' rope
    // gradient summed over the group's heads is this group's partial
    const bool give_up = compute_warps_or(!ok || *abort_flag, kWarps * 32);
    if (!give_up)
        for (int e = threadIdx.x; e < kBlock * kDR; e += kWarps * 32) {
            const int k = e / kDR, c = e % kDR;
            float x = 0.f;
#pragma unroll
            for (int ww = 0; ww < kWarps; ww++) x += s_dkr[ww][k][c];
            dkr_part[(((size_t)hg * gridDim.z + b) * L + key0 + k) * kDR + c] = x;
        }
    __syncthreads();
    if (threadIdx.x == 0 && abort_s) atomicOr(err, kErrTimeout);
}

struct BwdArgs {
    int B, n_h, S, N, W, L, R;
    float scale_log2, scale;
    const float *ds_, *lses;
    const int32_t *cnt, *sorted_n, *sorted_a;
    const float2 *tab;
    __nv_bfloat16 *dq, *dkc, *dv;
    float *dkr_part, *dqacc;
    int HG, hpg;  // head groups, heads per group
    int n_ctx;    // context tiles per batch row
    uint32_t *err;
    uint64_t wait_ns;  // limit of the pipeline waits (ns)
};

__device__ __forceinline__ void red_add_v4(float *addr, const uint4 &v) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(__uint_as_float(v.x)),
                 "f"(__uint_as_float(v.y)), "f"(__uint_as_float(v.z)), "f"(__uint_as_float(v.w))
                 : "memory");
}

// ============================================================= one pass
// Key tile = 64 keys (MMA M = 64); dK, dV and the dQ contributions of the
// tile in one CTA, so K, V and every row of Q and dO that sees the tile cross
// into shared memory once per head. With M = 64 an accumulator occupies lanes
// 0-15 of each 32-lane TMEM sub-partition, and a second one addressed at lane
// offset 16 the lanes 16-31 of the same columns:
//   columns   0..255  dK (offset 0; 192..255 the rope slice, summed over the
//                     group's heads, never reset between heads) and dV (16);
//   columns 256..383  S^T (0) and dP^T (16), two buffers of 64 columns;
//   columns 384..511  the chunk's dQ contribution: M = 64 rows, dims 0..127 at
//                     offset 0, dims 128..255 at offset 16.
// Per head: the K^C and V tiles (KVS stages; the rope-key tile is the same
// for all heads and is loaded once), then the rows that see the tile in chunks
// of 64 (Q and dO, RS stages): S^T = K Q^T and dP^T = V dO^T, P^T and dS^T
// (bf16) through one shared-memory buffer, dV += P^T dO, dK += dS^T Q, and
// dQ_c = dS K with dS read as an MN-major A operand from the dS^T tile.
// Key warps: warp w covers keys 16 (w & 3) .. + 15 (TMEM sub-partition w & 3)
// and rows 32 (w >> 2) .. + 31 of a chunk. Lane l < 16 loads S^T of its key,
// lane l + 16 dP^T of the same key; the two swap halves, so each lane holds
// both for 16 rows. At a head's end they read the accumulators, round them to
// bf16 and store dK^C and dV through a staging area in the P^T / dS^T buffer.
// dQ warps (one per TMEM sub-partition) read each chunk's dQ contribution and
// add it into the fp32 accumulator (four 128-byte row segments per vector
// reduction instruction).
namespace bw {
constexpr int kMK = 64;                    // keys per tile (MMA M)
constexpr int kRC = 64;                    // rows per chunk (MMA N of S^T / dP^T, K of the accumulations)
constexpr int kSlice = 64 * 128;           // 8 KB: 64 keys or rows x 64 columns, 128-byte swizzled
constexpr int kRowStage = 8 * kSlice;      // Q chunk (4 slices), then dO chunk (4 slices)
constexpr int kPT = 2 * kSlice;            // P^T, then dS^T: [64 keys][64 rows] bf16 each
constexpr int kDqStage = 32 * 64;          // per dQ warp: 32 lanes x 16 fp32
constexpr int kKeyWarps = 8;
constexpr int kWarpKV = kKeyWarps, kWarpRow = kKeyWarps + 1, kWarpMma = kKeyWarps + 2;
constexpr int kWarpDq = kKeyWarps + 3;     // four dQ warps, one per TMEM sub-partition
constexpr int kThreads = (kKeyWarps + 7) * 32;
constexpr uint32_t kColAcc = 0, kColS = 256, kColDQ = 384;  // S^T / dP^T buffer s at kColS + 64 s
constexpr uint32_t kHi = 16u << 16;        // lane offset of the second M = 64 accumulator

// Shared memory: the rope-key tile, one K^C and one V stage (V is free as
// soon as a head's last dP^T completed, K^C after its last dQ contribution,
// so the next head's tiles load while the current one finishes), RS row
// stages, the P^T / dS^T buffer (also the staging area of the head-end
// dK / dV readout), the dQ warps' staging, the per-row data.
template <int RS>
struct Smem {
    static constexpr int oKr = 0;                          // rope-key tile (8 KB)
    static constexpr int oKc = oKr + kSlice;               // K^C (3 slices)
    static constexpr int oV = oKc + 3 * kSlice;            // V (4 slices)
    static constexpr int oRow = oV + 4 * kSlice;           // row stage s at oRow + s * kRowStage
    static constexpr int oPT = oRow + RS * kRowStage;      // P^T, then dS^T
    static constexpr int oStage = oPT + kPT;               // dQ warps' staging
    static constexpr int oMeta = oStage + 4 * kDqStage;    // per row stage: (LSE * log2 e, D) of each row
    static constexpr int oBar = oMeta + RS * kRC * 8;
    static constexpr int kBytes = oBar + 256 + 1024;       // barriers, counters, alignment slack
    static_assert(kBytes <= 232448, "dynamic shared memory above the sm_100 per-block limit");
};
}  // namespace bw

// One CTA per (64-key tile, head group, batch row).
template <int RS>
__global__ void __launch_bounds__(bw::kThreads, 1)
    k_bwd_tc(const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_kr,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_qs,
             const __grid_constant__ CUtensorMap tm_dos, const BwdArgs p) {
    using namespace bw;
    using L = Smem<RS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::oBar);
    uint64_t *kfull = bars + 0, *kfree = bars + 1, *vfull = bars + 2, *vfree = bars + 3, *rowfull = bars + 4,
             *rowfree = bars + 6, *sfull = bars + 8, *ptfree = bars + 10, *dsready = bars + 11, *dqfull = bars + 12,
             *dqfree = bars + 13, *kdrain = bars + 14, *accdone = bars + 15, *drain = bars + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 17);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint64_t wlim = p.wait_ns;
    // K heads issued, V heads issued, row chunks issued, heads consumed, row chunks consumed
    int *counters = reinterpret_cast<int *>(tmem_slot + 2);
    int *band = counters + 5;  // first sorted row, row count

    // item = (region = (b, head group), context tile)
    const int region = (int)blockIdx.x / p.n_ctx, item = (int)blockIdx.x % p.n_ctx;
    const int b = region / p.HG, hg = region % p.HG;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    const int cnt = p.cnt[b];
    const int t0 = item * kMK;
    const int32_t *sa = p.sorted_a + (size_t)b * p.N;
    if (threadIdx.x == 0) {
        // blocks with t0 < A <= t0 + kMK - 1 + W - 1
        int lo = 0, hi = cnt;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (sa[mid] > t0) hi = mid; else lo = mid + 1;
        }
        const long long lim = (long long)t0 + kMK - 1 + p.W - 1;
        int lo2 = lo, hi2 = cnt;
        while (lo2 < hi2) {
            const int mid = (lo2 + hi2) >> 1;
            if ((long long)sa[mid] > lim) hi2 = mid; else lo2 = mid + 1;
        }
        band[0] = kBlock * lo;
        band[1] = kBlock * (lo2 - lo);
    }
    __syncthreads();
    const int row0 = band[0], nrows = band[1];
    const int nchunks = (nrows + kRC - 1) / kRC;
    const int h0 = hg * p.hpg;
    const int H = p.hpg;
    // the key this thread stands for (key warps): TMEM lane (l & 15) of its
    // sub-partition's two halves
    const int kk = 16 * (warp & 3) + (lane & 15);
    const int hr = (warp >> 2) & 1;  // row half of a chunk / column half of the accumulators
    const bool dlane = lane >= 16;   // lane of the dP^T / dV half
    const bool key_valid = warp < kKeyWarps && t0 + kk < p.S;
    const size_t key_pos = key_valid ? (size_t)t0 + kk : 0;
    float *dkr_part_row = p.dkr_part + (((size_t)hg * p.B + b) * p.L + key_pos) * kDR;

    if (nrows == 0) {
        // no row sees these keys: zero gradients for every head of the group
        // (four threads per key)
        if (warp < kKeyWarps && key_valid) {
            const int part = 2 * hr + (dlane ? 1 : 0);
            const uint4 z = make_uint4(0, 0, 0, 0);
            for (int hh = 0; hh < H; hh++) {
                const size_t bh = (size_t)b * p.n_h + h0 + hh;
                uint4 *dk = reinterpret_cast<uint4 *>(p.dkc + (bh * p.L + key_pos) * kDC);
                for (int e = part; e < kDC / 8; e += 4) dk[e] = z;
                uint4 *dvv = reinterpret_cast<uint4 *>(p.dv + (bh * p.L + key_pos) * kDV);
                for (int e = part; e < kDV / 8; e += 4) dvv[e] = z;
            }
            for (int e = part; e < kDR / 4; e += 4)
                reinterpret_cast<float4 *>(dkr_part_row)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        return;
    }

    // K/V tiles start zeroed (key slots no load reaches must hold finite values)
    for (int e = threadIdx.x; e < (L::oRow - L::oKr) / 16; e += blockDim.x)
        reinterpret_cast<uint4 *>(sm + L::oKr)[e] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        mbar_init(kfull, 1);
        mbar_init(kfree, 1);
        mbar_init(vfull, 1);
        mbar_init(vfree, 1);
        for (int s = 0; s < RS; s++) {
            mbar_init(&rowfull[s], 1);
            mbar_init(&rowfree[s], 1);
        }
        for (int s = 0; s < 2; s++) mbar_init(&sfull[s], 1);
        mbar_init(ptfree, 1);
        mbar_init(dsready, kKeyWarps);
        mbar_init(accdone, 1);
        mbar_init(dqfull, 1);
        mbar_init(dqfree, 4);
        mbar_init(kdrain, kKeyWarps);
        mbar_init(drain, 1);
        *abort_flag = 0;
        for (int c = 0; c < 5; c++) counters[c] = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int QT = H * nchunks;  // chunks over all heads of the group

    if (warp == kWarpKV) {
        // ------------------------------------------- producer of K/V tiles
        // Per head: V once the previous head's last dP^T completed, then K^C
        // (and, for the first head, the rope-key tile) once the previous head's
        // last dQ contribution completed; then the next head's tiles into L2, so
        // that those loads wait on L2 rather than on DRAM.
        for (int hh = 0; hh < H; ++hh) {
            const size_t bh = (size_t)b * p.n_h + h0 + hh;
            if (hh >= 1 && !warp_all(mbar_wait(vfree, (hh - 1) & 1, abort_flag, wlim))) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(vfull, 4 * kSlice);
                tma_load_3d(sm + L::oV, &tm_v, vfull, 0, (int)(bh * p.L + t0), 0);
                counters[1] = hh + 1;
            }
            if (hh >= 1 && !warp_all(mbar_wait(kfree, (hh - 1) & 1, abort_flag, wlim))) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(kfull, (hh == 0 ? 4 : 3) * kSlice);
                if (hh == 0) tma_load_2d(sm + L::oKr, &tm_kr, kfull, 0, (int)((size_t)b * p.L + t0));
                tma_load_3d(sm + L::oKc, &tm_kc, kfull, 0, (int)(bh * p.L + t0), 0);
                counters[0] = hh + 1;
                if (hh + 1 < H) {
                    tma_prefetch_l2_3d(&tm_kc, 0, (int)((bh + 1) * p.L + t0), 0);
                    tma_prefetch_l2_3d(&tm_v, 0, (int)((bh + 1) * p.L + t0), 0);
                }
            }
        }
    } else if (warp == kWarpRow) {
        // ---------------------------- producer of Q / dO chunks and row data
        // The row data of chunk q + 1 (LSE * log2 e and D, one value per lane
        // and 32 rows) is read into registers, and its Q / dO rows prefetched
        // into L2, while chunk q is in use, so that once the stage is free only
        // the shared-memory copy remains.
        auto meta_of = [&](int q, float2 (&m)[kRC / 32]) {
            const int hh = q / nchunks, c = q % nchunks;
            const size_t bh = (size_t)b * p.n_h + h0 + hh;
            const int r0 = row0 + c * kRC;
#pragma unroll
            for (int jj = 0; jj < kRC / 32; jj++) {
                const int rowi = r0 + 32 * jj + lane;
                m[jj] = rowi < row0 + nrows ? make_float2(p.lses[bh * p.R + rowi], p.ds_[bh * p.R + rowi])
                                            : make_float2(0.f, 0.f);
            }
        };
        float2 mnext[kRC / 32];
        meta_of(0, mnext);
        for (int q = 0; q < QT; ++q) {
            const int hh = q / nchunks, c = q % nchunks, s = q % RS;
            const size_t bh = (size_t)b * p.n_h + h0 + hh;
            const int r0 = row0 + c * kRC;
            float2 mcur[kRC / 32];
#pragma unroll
            for (int jj = 0; jj < kRC / 32; jj++) mcur[jj] = mnext[jj];
            if (q + 1 < QT) {
                meta_of(q + 1, mnext);
                if (lane == 0) {
                    const int hn = (q + 1) / nchunks, cn = (q + 1) % nchunks;
                    const int rn = (int)(((size_t)b * p.n_h + h0 + hn) * p.R + row0 + cn * kRC);
                    tma_prefetch_l2_3d(&tm_qs, 0, rn, 0);
                    tma_prefetch_l2_3d(&tm_dos, 0, rn, 0);
                }
            }
            if (q >= RS && !warp_all(mbar_wait(&rowfree[s], ((q / RS) - 1) & 1, abort_flag, wlim))) break;
            float2 *mLD = reinterpret_cast<float2 *>(sm + L::oMeta + s * kRC * 8);
#pragma unroll
            for (int jj = 0; jj < kRC / 32; jj++) mLD[32 * jj + lane] = mcur[jj];
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_expect_tx(&rowfull[s], kRowStage);
                tma_load_3d(sm + L::oRow + s * kRowStage, &tm_qs, &rowfull[s], 0, (int)(bh * p.R + r0), 0);
                tma_load_3d(sm + L::oRow + s * kRowStage + 4 * kSlice, &tm_dos, &rowfull[s], 0, (int)(bh * p.R + r0),
                            0);
                counters[2] = q + 1;
            }
        }
    } else if (warp == kWarpMma) {
        // ----------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idS = idesc_bf16(kMK, kRC, 0);   // S^T, dP^T: B = Q / dO chunk, K-major
            const uint32_t idV = idesc_bf16(kMK, kDV, 1);   // dV: B = dO chunk, MN-major
            const uint32_t idKc = idesc_bf16(kMK, kDC, 1);  // dK^C: B = Q^C columns
            const uint32_t idKr = idesc_bf16(kMK, kDR, 1);  // dK^R: B = Q^R columns
            // dQ_c = dS K: A = dS (M = 64 rows, K = keys) read MN-major from the
            // dS^T tile, B = the key tile (N = dims, K = keys), MN-major
            const uint32_t idQ128 = idesc_bf16_ab(kRC, 128, 1, 1);
            const uint32_t idQ64 = idesc_bf16_ab(kRC, 64, 1, 1);
            // A operands of S^T / dP^T: K^C / V slices kcStep bytes apart
            // (context tile: 8 KB slices of 64 keys; draft tile: block-major)
            // A operands of S^T / dP^T: K^C / V slices of 64 keys, 8 KB apart
            const SDesc krd = sdesc_split(sdesc_sw128(smem_u32(sm + L::oKr), 16, 1024));
            const SDesc ptd = sdesc_split(sdesc_sw128(smem_u32(sm + L::oPT), 16, 1024));
            const SDesc dsd = sdesc_split(sdesc_sw128(smem_u32(sm + L::oPT + kSlice), 16, 1024));
            const SDesc dsq = sdesc_split(sdesc_sw128(smem_u32(sm + L::oPT + kSlice), kSlice, 1024));
            // B operands of dQ_c, MN-major: dims 0..127 of K^C (two slices),
            // dims 128..191 (third slice), the rope key (dims 192..255); 16 keys
            // are 16 rows of 128 B (2 KB)
            const SDesc krq = sdesc_split(sdesc_sw128(smem_u32(sm + L::oKr), kSlice, 1024));
            const SDesc kq0 = sdesc_split(sdesc_sw128(smem_u32(sm + L::oKc), kSlice, 1024));
            const SDesc kq1 = sdesc_split(sdesc_sw128(smem_u32(sm + L::oKc + 2 * kSlice), kSlice, 1024));
            bool ok = true;
            const SDesc kad = sdesc_split(sdesc_sw128(smem_u32(sm + L::oKc), 16, 1024));
            const SDesc vad = sdesc_split(sdesc_sw128(smem_u32(sm + L::oV), 16, 1024));
            auto issue_s = [&](int q) {
                const int c = q % nchunks, s = q % RS, bsel = q & 1;
                tc_fence_after();
                const uint32_t rs = smem_u32(sm + L::oRow + s * kRowStage);
                const SDesc qd = sdesc_split(sdesc_sw128(rs, 16, 1024));
                const SDesc dod = sdesc_split(sdesc_sw128(rs + 4 * kSlice, 16, 1024));
                const uint32_t dS = tmem + kColS + 64 * bsel, dP = dS + kHi;
                // S^T = K Q^T and dP^T = V dO^T interleaved: two independent chains
#pragma unroll
                for (int k16 = 0; k16 < kDQK / 16; ++k16) {
                    const int cc = k16 >> 2;
                    const uint32_t sub = (k16 & 3) * 2;  // 32 bytes, in 16-byte units
                    const uint64_t ka = cc < 3 ? kad.at(((cc * kSlice) >> 4) + sub) : krd.at(sub);
                    const uint32_t ro = (cc * kSlice + (k16 & 3) * 32) >> 4;
                    mma_bf16_ss(dS, ka, qd.at(ro), idS, k16 > 0 ? 1u : 0u);
                    mma_bf16_ss(dP, vad.at(((cc * kSlice) >> 4) + sub), dod.at(ro), idS, k16 > 0 ? 1u : 0u);
                }
                mma_commit(&sfull[bsel]);
                if (c == nchunks - 1) mma_commit(vfree);  // the head's V tile is no longer read
            };
            auto issue_acc = [&](int q) {
                const int c = q % nchunks, s = q % RS;
                tc_fence_after();
                const uint32_t rs = smem_u32(sm + L::oRow + s * kRowStage);
                const SDesc qb = sdesc_split(sdesc_sw128(rs, kSlice, 1024));  // MN-major
                const SDesc dob = sdesc_split(sdesc_sw128(rs + 4 * kSlice, kSlice, 1024));
                // 16 rows per MMA: 32 bytes along the K-major P^T / dS^T rows,
                // 2 KB (16 rows of 128 bytes) in the row chunk
#pragma unroll
                for (int k16 = 0; k16 < kRC / 16; ++k16)
                    mma_bf16_ss(tmem + kColAcc + kHi, ptd.at(2 * k16), dob.at(128 * k16), idV,
                                (c > 0 || k16 > 0) ? 1u : 0u);
#pragma unroll
                for (int k16 = 0; k16 < kRC / 16; ++k16)
                    mma_bf16_ss(tmem + kColAcc, dsd.at(2 * k16), qb.at(128 * k16), idKc, (c > 0 || k16 > 0) ? 1u : 0u);
#pragma unroll
                for (int k16 = 0; k16 < kRC / 16; ++k16)
                    mma_bf16_ss(tmem + kColAcc + kDC, dsd.at(2 * k16), qb.at(((3 * kSlice) >> 4) + 128 * k16), idKr,
                                (q > 0 || k16 > 0) ? 1u : 0u);
                mma_commit(&rowfree[s]);
                mma_commit(ptfree);  // after the chunk's dQ contribution, issued before
                if (c == nchunks - 1) mma_commit(accdone);  // the head's accumulators are final
            };
            auto issue_dq = [&](int q) {
                const int c = q % nchunks;
                tc_fence_after();
#pragma unroll
                for (int k16 = 0; k16 < kMK / 16; ++k16) {
                    const uint64_t a = dsq.at(128 * k16);  // 16 keys = 16 rows of the dS^T tile
                    mma_bf16_ss(tmem + kColDQ, a, kq0.at(128 * k16), idQ128, k16 > 0 ? 1u : 0u);
                    mma_bf16_ss(tmem + kColDQ + kHi, a, kq1.at(128 * k16), idQ64, k16 > 0 ? 1u : 0u);
                    mma_bf16_ss(tmem + kColDQ + kHi + 64, a, krq.at(128 * k16), idQ64, k16 > 0 ? 1u : 0u);
                }
                mma_commit(dqfull);
                if (c == nchunks - 1) mma_commit(kfree);  // the head's K^C / K^R tiles are no longer read
            };
            // Issue whichever is ready: the S^T / dP^T stage of chunk ns (its K,
            // V and row operands landed; at most one chunk ahead of the dQ
            // contributions, so its S^T / dP^T buffer was read by the key warps
            // before they signalled chunk ns - 2), the dQ contribution of chunk
            // nd (P^T / dS^T written, the dQ warps have read chunk nd - 1's; it
            // goes first so that the head's K^C tile is freed early), or the
            // accumulation of chunk na (after its dQ contribution; at a head's
            // first chunk the key warps have also read out the previous head's
            // accumulators, which precedes their dS^T signal).
            int ns = 0, na = 0, nd = 0;
            uint64_t t_idle = 0;
            while (ok && na < QT) {
                bool issued = false;
                if (ns < QT && ns <= nd + 1) {
                    const int hh = ns / nchunks, c = ns % nchunks;
                    if ((c != 0 || (mbar_test(kfull, hh & 1) && mbar_test(vfull, hh & 1))) &&
                        mbar_test(&rowfull[ns % RS], (ns / RS) & 1)) {
                        if (c == 0) counters[3] = hh + 1;
                        counters[4] = ns + 1;
                        issue_s(ns);
                        ++ns;
                        issued = true;
                    }
                }
                if (!issued && nd < ns && mbar_test(dsready, nd & 1) && (nd == 0 || mbar_test(dqfree, (nd - 1) & 1))) {
                    issue_dq(nd);
                    ++nd;
                    issued = true;
                }
                if (!issued && na < nd) {
                    issue_acc(na);
                    ++na;
                    issued = true;
                }
                if (issued) {
                    t_idle = 0;
                } else {
                    const uint64_t now = globaltimer();
                    if (t_idle == 0) t_idle = now;
                    if (*abort_flag) ok = false;
                    else if (now - t_idle > wlim) {
                        *abort_flag = 1;
                        ok = false;
                    }
                }
            }
        }
    } else if (warp >= kWarpDq) {
        // --------------------------------------------------- dQ warps
        // Sub-partition sp: lanes 0-15 hold dims 0..127 of chunk rows
        // 16 sp .. + 15, lanes 16-31 dims 128..255 of the same rows. Per chunk:
        // four loads of 32 columns, each staged in two halves (each thread its
        // 64 bytes, 16-byte unit u at u ^ (lane & 3)); the warp writes eight
        // rows' 64-byte segments per instruction into the accumulator (sorted
        // rows) with vector reductions.
        const int sp = warp & 3;  // a warp reaches the TMEM lanes of sub-partition warp % 4 only
        const uint32_t trow = tmem + ((uint32_t)(sp * 32) << 16);
        uint8_t *stage = sm + L::oStage + sp * kDqStage;
        bool ok = true;
        for (int q = 0; q < QT && ok; ++q) {
            const int hh = q / nchunks, c = q % nchunks;
            ok = warp_all(mbar_wait(dqfull, q & 1, abort_flag, wlim));
            if (!ok) break;
            tc_fence_after();
            const size_t bh = (size_t)b * p.n_h + h0 + hh;
            const int cr0 = c * kRC + 16 * sp;  // chunk-relative band row of lane 0
            float *acc_rows = p.dqacc + (bh * p.R + row0) * kDQK;
#pragma unroll 1
            for (int rd = 0; rd < 4; rd++) {
                float v[32];
                tmem_ld32(trow + kColDQ + 32 * rd, v);
                tmem_wait_ld();
                if (rd == 3) {  // the dQ columns are free for the next chunk
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(dqfree);
                }
#pragma unroll
                for (int hf = 0; hf < 2; hf++) {
#pragma unroll
                    for (int u = 0; u < 4; u++)
                        *reinterpret_cast<uint4 *>(stage + lane * 64 + ((u ^ (lane & 3)) << 4)) =
                            make_uint4(__float_as_uint(v[16 * hf + 4 * u]), __float_as_uint(v[16 * hf + 4 * u + 1]),
                                       __float_as_uint(v[16 * hf + 4 * u + 2]), __float_as_uint(v[16 * hf + 4 * u + 3]));
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        const int sl = 8 * i + (lane >> 2), u = lane & 3;  // source lane, unit
                        const int br = cr0 + (sl & 15);                    // band row
                        if (br < nrows) {
                            const uint4 val = *reinterpret_cast<const uint4 *>(stage + sl * 64 + ((u ^ (sl & 3)) << 4));
                            red_add_v4(acc_rows + (size_t)br * kDQK + (sl >> 4) * 128 + 32 * rd + 16 * hf + 4 * u, val);
                        }
                    }
                    __syncwarp();
                }
            }
        }
    } else {
        // ------------------------------------------ key warps (0..7)
        const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const int rb = 32 * hr + 16 * (lane >> 4);  // first chunk row of this lane after the swap
        const int kpos = t0 + kk;                   // context position of this key (context tiles)
        // The rows that see this key, in sorted-row order relative to the band:
        // one range [rlo, rhi), the same for every head. Context key: blocks
        // with kpos < A <= kpos + W - 1; draft key slot: its own block.
        int rlo = 0, rhi = 0;
        if (key_valid) {
            int lo = row0 / kBlock, hi = (row0 + nrows) / kBlock;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (sa[mid] > kpos) hi = mid; else lo = mid + 1;
            }
            rlo = kBlock * lo - row0;
            const long long lim = (long long)kpos + p.W - 1;
            hi = (row0 + nrows) / kBlock;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if ((long long)sa[mid] > lim) hi = mid; else lo = mid + 1;
            }
            rhi = kBlock * lo - row0;
        }
        // this key's row of the P^T / dS^T tiles (128-byte swizzle) and the
        // two 16-byte units that hold rows rb .. rb + 15
        const uint32_t prow = (uint32_t)((kk >> 3) * 1024 + (kk & 7) * 128);
        const uint32_t pu0 = prow + ((((uint32_t)rb >> 3) ^ (kk & 7)) << 4);
        const uint32_t pu1 = prow + (((((uint32_t)rb >> 3) + 1) ^ (kk & 7)) << 4);
        bool ok = true;
        for (int q = 0; q < QT && ok; ++q) {
            const int hh = q / nchunks, c = q % nchunks, s = q % RS, bsel = q & 1;
            ok = warp_all(mbar_wait(&rowfull[s], (q / RS) & 1, abort_flag, wlim));  // row data
            if (ok) ok = warp_all(mbar_wait(&sfull[bsel], (q >> 1) & 1, abort_flag, wlim));
            if (!ok) break;
            tc_fence_after();
            float v[32];
            tmem_ld32(trow + kColS + 64 * bsel + 32 * hr, v);
            tmem_wait_ld();
            float sv[16], pv[16];
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const float send = dlane ? v[i] : v[16 + i];
                const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
                sv[i] = dlane ? recv : v[i];
                pv[i] = dlane ? v[16 + i] : recv;
            }
            const float2 *mLD = reinterpret_cast<const float2 *>(sm + L::oMeta + s * kRC * 8) + rb;
            const int jlo = rlo - c * kRC - rb, jhi = rhi - c * kRC - rb;  // visible rows, relative to rb
            uint32_t pw[8], dw[8];
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                float ep[2], ed[2];
#pragma unroll
                for (int d = 0; d < 2; d++) {
                    const int j = i + d;
                    const float2 ldv = mLD[j];
                    const float pp = (j >= jlo && j < jhi) ? ex2(fmaf(sv[j], p.scale_log2, -ldv.x)) : 0.f;
                    ep[d] = pp;
                    ed[d] = pp * (pv[j] - ldv.y) * p.scale;
                }
                pw[i / 2] = pack_bf16x2(ep[0], ep[1]);
                dw[i / 2] = pack_bf16x2(ed[0], ed[1]);
            }
            // the P^T / dS^T buffer is free once the dQ contribution and the
            // accumulation of chunk q - 1 completed; at a head's first chunk,
            // every key warp has also read its staged rows of the previous
            // head's accumulators (staged in this same buffer)
            uint8_t *pt = sm + L::oPT;
            if (q >= 1) ok = warp_all(mbar_wait(ptfree, (q - 1) & 1, abort_flag, wlim));
            if (ok && c == 0 && hh >= 1) ok = warp_all(mbar_wait(kdrain, (hh - 1) & 1, abort_flag, wlim));
            if (!ok) break;
            *reinterpret_cast<uint4 *>(pt + pu0) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
            *reinterpret_cast<uint4 *>(pt + pu1) = make_uint4(pw[4], pw[5], pw[6], pw[7]);
            *reinterpret_cast<uint4 *>(pt + kSlice + pu0) = make_uint4(dw[0], dw[1], dw[2], dw[3]);
            *reinterpret_cast<uint4 *>(pt + kSlice + pu1) = make_uint4(dw[4], dw[5], dw[6], dw[7]);
            fence_proxy_async_smem();  // visible to the MMAs that read them
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dsready);
            if (c != nchunks - 1) continue;
            // head end, once its accumulations (and, issued before them, its dQ
            // contributions) completed: accumulator columns [128 hr, 128 hr + 128)
            // (lanes 0-15 dK, 16-31 dV) -> bf16 -> dK^C / dV rows, staged 32
            // columns at a time in the P^T / dS^T buffer (2 KB per warp, each
            // thread its 64 bytes, 16-byte unit u at u ^ (lane & 3)), the warp
            // writing 8 rows' 64-byte segments per instruction. dK columns
            // 192..255 (the rope slice) stay in TMEM, summed over heads. The
            // accumulator is then free for the next head.
            ok = warp_all(mbar_wait(accdone, hh & 1, abort_flag, wlim));
            if (!ok) break;
            tc_fence_after();
            uint8_t *stage = sm + L::oPT + warp * 2048;
            const size_t bh = (size_t)b * p.n_h + h0 + hh;
#pragma unroll 1
            for (int rd = 0; rd < 4; rd++) {
                tmem_ld32(trow + kColAcc + hr * 128 + rd * 32, v);
                tmem_wait_ld();
                const int col = hr * 128 + rd * 32;
                const bool rope = col >= kDC;
#pragma unroll
                for (int u = 0; u < 4; u++)
                    *reinterpret_cast<uint4 *>(stage + lane * 64 + ((u ^ (lane & 3)) << 4)) =
                        make_uint4(pack_bf16x2(v[8 * u], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                                   pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int kl = 8 * i + (lane >> 2), u = lane & 3;  // source lane, unit
                    const int kvl = __shfl_sync(0xffffffffu, (int)key_valid, kl);
                    const long long kposl = __shfl_sync(0xffffffffu, (long long)key_pos, kl);
                    const bool is_v = kl >= 16;
                    if (kvl && (is_v || !rope)) {
                        const uint4 val = *reinterpret_cast<const uint4 *>(stage + kl * 64 + ((u ^ (kl & 3)) << 4));
                        __nv_bfloat16 *dst = is_v ? p.dv + (bh * p.L + (size_t)kposl) * kDV + col + 8 * u
                                                  : p.dkc + (bh * p.L + (size_t)kposl) * kDC + col + 8 * u;
                        *reinterpret_cast<uint4 *>(dst) = val;
                    }
                }
                __syncwarp();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(kdrain);
        }
        if (ok && hr == 1) {
            // rope slice of dK (columns 192..255 of the lanes 0-15), summed over
            // the group's heads by the MMAs
            float *d = dkr_part_row;
            const bool w_ = key_valid && !dlane;
#pragma unroll
            for (int half2 = 0; half2 < 2; half2++) {
                float v[32];
                tmem_ld32(trow + kColAcc + kDC + 32 * half2, v);
                tmem_wait_ld();
                if (w_)
#pragma unroll
                    for (int i = 0; i < 8; i++)
                        reinterpret_cast<float4 *>(d + 32 * half2)[i] =
                            make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
        }
    }

    __syncthreads();
    if (*abort_flag) {
        volatile int never = 0;
        if (warp == kWarpKV && lane == 0) {
            for (int t = counters[3]; t < counters[0]; ++t) mbar_wait(kfull, t & 1, (volatile int *)&never);
            for (int t = counters[3]; t < counters[1]; ++t) mbar_wait(vfull, t & 1, (volatile int *)&never);
        }
        if (warp == kWarpRow && lane == 0) {
            for (int t = counters[4]; t < counters[2]; ++t)
                mbar_wait(&rowfull[t % RS], (t / RS) & 1, (volatile int *)&never);
        }
        if (warp == kWarpMma && lane == 0) {
            mma_commit(drain);
            mbar_wait(drain, 0, (volatile int *)&never);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x == 0 && *abort_flag) atomicOr(p.err, kErrTimeout);
}

// ------------------------------------------------------------- dQ output
// One warp per row of a kept block (5 warps): the accumulated dQ row (sorted
// order; lane l holds dims 8 l .. 8 l + 7), its rope slice (lanes 24-31)
// rotated back by the query position A + j, rounded to bf16 and written to the
// caller's row 5 n + j.
__global__ void __launch_bounds__(160) k_bwd_dq_out(int n_h, int N, const int32_t *__restrict__ cnt,
                                                    const int32_t *__restrict__ sorted_n,
                                                    const int32_t *__restrict__ sorted_a,
                                                    const float2 *__restrict__ tab, const float *__restrict__ dqacc,
                                                    __nv_bfloat16 *__restrict__ dq) {
    const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    pdl_wait();
    if (i >= cnt[b]) return;
    const int j = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = kBlock * N;
    const size_t bh = (size_t)b * n_h + h;
    const int n = sorted_n[(size_t)b * N + i], a = sorted_a[(size_t)b * N + i];
    const float4 *src = reinterpret_cast<const float4 *>(dqacc + (bh * R + kBlock * i + j) * kDQK) + 2 * lane;
    const float4 x = src[0], y = src[1];
    float v[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
    if (lane >= 24) {  // rope slice: rotate back by the query position A + j
        const float2 *cs = tab + (size_t)(a + j) * (kDR / 2) + (lane - 24) * 4;
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const float2 t2 = __ldg(cs + k);
            const float x0 = v[2 * k], x1 = v[2 * k + 1];
            v[2 * k] = x0 * t2.x + x1 * t2.y;
            v[2 * k + 1] = x1 * t2.x - x0 * t2.y;
        }
    }
    *(reinterpret_cast<uint4 *>(dq + (bh * R + kBlock * n + j) * kDQK) + lane) =
        make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

// ------------------------------------------------------------ dK^R reduce
// One warp per (b, key): sum the head-group partials of the rope-key gradient
// (rotated frame; context keys from k_bwd_tc's HG groups, draft keys from
// k_bwd_prep's HGd groups),
// rotate back by the key's position, write dkr. Draft keys of padding blocks:
// 0.
__global__ void __launch_bounds__(256) k_bwd_dkr_reduce(int B, int S, int N, int L, int HG, int HGd,
                                                        const int32_t *anchors, const uint8_t *keep,
                                                        const float2 *tab, const float *part,
                                                        __nv_bfloat16 *dkr) {
    const int lane = threadIdx.x & 31;
    pdl_wait();
    for (size_t wid = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); wid < (size_t)B * L;
         wid += (size_t)gridDim.x * (blockDim.x >> 5)) {
        const int b = (int)(wid / L), key = (int)(wid % L);
        int pos = key;
        bool live = true;
        if (key >= S) {
            const int n = (key - S) / kBlock, i = (key - S) % kBlock;
            const int a = anchors[(size_t)b * N + n];
            live = keep[(size_t)b * N + n] && a >= 0 && a <= S - 2;
            pos = a + i;
        }
        float x0 = 0.f, x1 = 0.f;
        if (live) {
            const int groups = key < S ? HG : HGd;  // context keys: the tensor-core kernel's groups
            const float *src = part + ((size_t)b * L + key) * kDR + 2 * lane;
            const size_t gstride = (size_t)B * L * kDR;
#pragma unroll 4
            for (int g = 0; g < groups; g++) {
                const float2 v = *reinterpret_cast<const float2 *>(src + g * gstride);
                x0 += v.x;
                x1 += v.y;
            }
            const float2 cs = tab[(size_t)pos * (kDR / 2) + lane];
            const float y0 = x0 * cs.x + x1 * cs.y, y1 = x1 * cs.x - x0 * cs.y;
            x0 = y0;
            x1 = y1;
        }
        *reinterpret_cast<__nv_bfloat162 *>(dkr + ((size_t)b * L + key) * kDR + 2 * lane) = __floats2bfloat162_rn(x0, x1);
    }
}

// Row stages of the one-pass kernel.
constexpr int kRS = 2;

}  // namespace

bool bwd_tc_supported(const Prob &p) {
    return p.dtype == DSPARK_BF16 && p.d_c == kDC && p.d_r == kDR && p.d_v == kDV &&
           (long long)p.B * p.n_h * p.L < (1ll << 31) && (long long)p.B * p.n_h * p.R < (1ll << 31);
}

int bwd_prep_groups(const Prob &p) { return (p.n_h + pr::kHeads - 1) / pr::kHeads; }

int bwd_head_groups(const Prob &p) {
    const long long items = (long long)((p.S + bw::kMK - 1) / bw::kMK) * p.B;
    // aim for about six waves on 148 SMs (shorter CTAs, smaller tail)
    int hg = 1;
    while (hg < p.n_h && items * hg < 6 * 148 && p.n_h % (hg * 2) == 0) hg *= 2;
    return hg;
}

cudaError_t launch_bwd_tc(const Prob &p, const void *q, const void *kc, const void *v, const int32_t *anchors,
                          const uint8_t *keep, const void *o, const float *lse, const void *dout, void *dq,
                          void *dkc, void *dkr, void *dv, const Ws &ws, cudaStream_t st) {
    if (p.B == 0) return cudaSuccess;
    const int HG = bwd_head_groups(p);
    if (p.N > 0) {
        count_launch();
        cudaError_t ep = cudaFuncSetAttribute(k_bwd_prep, cudaFuncAttributeMaxDynamicSharedMemorySize, pr::kSmem);
        if (ep != cudaSuccess) return ep;
        ep = launch_pdl(k_bwd_prep, dim3(p.N, bwd_prep_groups(p), p.B), dim3(pr::kThreads), pr::kSmem, st, p.n_h,
                        p.S, p.N, p.L, p.scale, p.scale_log2, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)kc,
                        (const __nv_bfloat16 *)ws.kr_rot, (const __nv_bfloat16 *)v, (const __nv_bfloat16 *)o,
                        (const __nv_bfloat16 *)dout, lse, (const int32_t *)ws.cnt, (const int32_t *)ws.sorted_n,
                        (const int32_t *)ws.sorted_a, (const float2 *)ws.rope, (__nv_bfloat16 *)ws.qs,
                        (__nv_bfloat16 *)ws.dos, ws.dvec, ws.lses, ws.dqacc, (__nv_bfloat16 *)dkc, ws.dkr_part,
                        (__nv_bfloat16 *)dv, ws.err, p.wait_ns);
        if (ep != cudaSuccess) return ep;
    }
    CUtensorMap m_kc3_64, m_kr64, m_v3_64, m_qs3_64, m_dos3_64;
    const uint64_t kv_rows = (uint64_t)p.B * p.n_h * p.L, q_rows = (uint64_t)p.B * p.n_h * p.R;
    if (!make_map3_bf16(&m_kc3_64, kc, kDC, kv_rows, 64) ||
        !make_map_bf16(&m_kr64, ws.kr_rot, kDR, (uint64_t)p.B * p.L, 64) || !make_map3_bf16(&m_v3_64, v, kDV, kv_rows, 64))
        return cudaErrorInvalidValue;
    if (p.N > 0 && q_rows > 0) {
        if (!make_map3_bf16(&m_qs3_64, ws.qs, kDQK, q_rows, 64) || !make_map3_bf16(&m_dos3_64, ws.dos, kDV, q_rows, 64))
            return cudaErrorInvalidValue;
    } else {  // maps over Q rows are never read: any valid map will do
        m_qs3_64 = m_dos3_64 = m_kc3_64;
    }
    BwdArgs a;
    a.B = p.B; a.n_h = p.n_h; a.S = p.S; a.N = p.N; a.W = p.W; a.L = p.L; a.R = p.R;
    a.scale_log2 = p.scale_log2;
    a.scale = p.scale;
    a.ds_ = ws.dvec;
    a.lses = ws.lses;
    a.cnt = ws.cnt;
    a.sorted_n = ws.sorted_n;
    a.sorted_a = ws.sorted_a;
    a.tab = ws.rope;
    a.dq = (__nv_bfloat16 *)dq;
    a.dkc = (__nv_bfloat16 *)dkc;
    a.dv = (__nv_bfloat16 *)dv;
    a.dkr_part = ws.dkr_part;
    a.dqacc = ws.dqacc;
    a.HG = HG;
    a.hpg = p.n_h / HG;
    a.n_ctx = (p.S + bw::kMK - 1) / bw::kMK;
    a.err = ws.err;
    a.wait_ns = p.wait_ns;
    const unsigned grid = (unsigned)((size_t)p.B * HG * a.n_ctx);
    constexpr int smem = bw::Smem<kRS>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(k_bwd_tc<kRS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    count_launch();
    if ((e = launch_pdl(k_bwd_tc<kRS>, dim3(grid), dim3(bw::kThreads), smem, st, m_kc3_64, m_kr64, m_v3_64, m_qs3_64,
                        m_dos3_64, a)) != cudaSuccess)
        return e;
    if (p.N > 0) {
        count_launch();
        if ((e = launch_pdl(k_bwd_dq_out, dim3(p.N, p.n_h, p.B), dim3(160), 0, st, p.n_h, p.N,
                            (const int32_t *)ws.cnt, (const int32_t *)ws.sorted_n, (const int32_t *)ws.sorted_a,
                            (const float2 *)ws.rope, (const float *)ws.dqacc, (__nv_bfloat16 *)dq)) != cudaSuccess)
            return e;
    }
    const size_t warps = (size_t)p.B * p.L;
    count_launch();
    return launch_pdl(k_bwd_dkr_reduce, dim3((unsigned)std::min<size_t>((warps + 7) / 8, 148 * 8)), dim3(256), 0, st,
                      p.B, p.S, p.N, p.L, HG, bwd_prep_groups(p), anchors, keep, (const float2 *)ws.rope,
                      (const float *)ws.dkr_part, (__nv_bfloat16 *)dkr);
}

}  // namespace dspark
