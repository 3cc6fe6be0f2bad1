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
// Launch sequence (one stream, no atomics, every output element written once):
//   1. k_bwd_prep      per kept block and head: rotated Q and dO copied into
//                      anchor-sorted row order, D, LSE*log2(e); padding rows 0.
//   2. k_bwd_pad       zeros for padding blocks' rows and draft keys.
//   3. k_bwd_dq_tc     query-major, one CTA per (b, h, 25 sorted blocks):
//                      64-key tiles of the group's key set; S and dP in TMEM,
//                      dS written over the S columns, dQ += dS K in TMEM.
//   4. k_bwd_kv_tc     key-major, one CTA per (b, 64-key tile, head group):
//                      rows of the blocks whose key sets meet the tile, in
//                      chunks of 64: S^T = K Q^T and dP^T = V dO^T in TMEM,
//                      P^T and dS^T through shared memory, dV += P^T dO and
//                      dK += dS^T Q accumulated in TMEM over the rows (M = 64
//                      accumulators: dK and dV share TMEM columns, one in each
//                      half of the lanes).
//   5. k_bwd_dkr_reduce sums the per-head-group rope-key partials, rotates
//                      them back and writes dK^R.
// Key tiles are either context tiles [t0, t0+64) or the draft keys of one
// group of 8 blocks; the blocks whose windows meet a context tile are a
// contiguous run of the anchor-sorted list (t0 < A <= t0 + 63 + W - 1).
#include <algorithm>

#include "dspark_tc_common.cuh"

namespace dspark {

namespace {

using namespace tc;

constexpr int kDC = 192, kDR = 64, kDQK = 256, kDV = 256;
constexpr int kG = 25;   // blocks per query group (query-major kernel)
constexpr int kGD = 8;   // blocks per draft-key tile of the key-major kernel (8 slots each: 64 keys)
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ prep
// One warp per row of a kept block (5 warps): rotated q -> qs, do -> dos,
// D = rowsum(dO * O), LSE * log2(e); rows past the kept blocks are zeroed so
// tiles that overhang them multiply finite values.
__global__ void __launch_bounds__(160) k_bwd_prep(int n_h, int N, const __nv_bfloat16 *__restrict__ q,
                                                  const __nv_bfloat16 *__restrict__ o,
                                                  const __nv_bfloat16 *__restrict__ dout,
                                                  const float *__restrict__ lse, const int32_t *__restrict__ cnt,
                                                  const int32_t *__restrict__ sorted_n,
                                                  const int32_t *__restrict__ sorted_a,
                                                  const float2 *__restrict__ tab, __nv_bfloat16 *__restrict__ qs,
                                                  __nv_bfloat16 *__restrict__ dos, float *__restrict__ ds_,
                                                  float *__restrict__ lses) {
    const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int j = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = kBlock * N;
    const size_t bh = (size_t)b * n_h + h;
    const size_t srow = bh * R + kBlock * i + j;
    uint4 *qd = reinterpret_cast<uint4 *>(qs + srow * kDQK) + lane;
    uint4 *dd = reinterpret_cast<uint4 *>(dos + srow * kDV) + lane;
    if (i >= cnt[b]) {
        *qd = make_uint4(0, 0, 0, 0);
        *dd = make_uint4(0, 0, 0, 0);
        if (lane == 0) {
            ds_[srow] = 0.f;
            lses[srow] = 0.f;
        }
        return;
    }
    const int n = sorted_n[(size_t)b * N + i], a = sorted_a[(size_t)b * N + i];
    const size_t orow = bh * R + kBlock * n + j;
    uint4 qv = __ldg(reinterpret_cast<const uint4 *>(q + orow * kDQK) + lane);
    if (lane >= 24) {
        const float2 *cs = tab + (size_t)(a + j) * (kDR / 2) + (lane - 24) * 4;
        uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
        for (int k = 0; k < 4; k++) {
            __nv_bfloat162 pr = *reinterpret_cast<__nv_bfloat162 *>(&w[k]);
            const float x0 = __bfloat162float(pr.x), x1 = __bfloat162float(pr.y);
            const float2 c = __ldg(cs + k);
            w[k] = pack_bf16x2(x0 * c.x - x1 * c.y, x0 * c.y + x1 * c.x);
        }
        qv = make_uint4(w[0], w[1], w[2], w[3]);
    }
    *qd = qv;
    const uint4 dv = __ldg(reinterpret_cast<const uint4 *>(dout + orow * kDV) + lane);
    const uint4 ov = __ldg(reinterpret_cast<const uint4 *>(o + orow * kDV) + lane);
    *dd = dv;
    const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w}, ow[4] = {ov.x, ov.y, ov.z, ov.w};
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162 *>(&dw[k]);
        const __nv_bfloat162 y = *reinterpret_cast<const __nv_bfloat162 *>(&ow[k]);
        acc = fmaf(__bfloat162float(x.x), __bfloat162float(y.x), acc);
        acc = fmaf(__bfloat162float(x.y), __bfloat162float(y.y), acc);
    }
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
        ds_[srow] = acc;
        lses[srow] = lse[orow] * kLog2e;
    }
}

// -------------------------------------------------------------- padding
// Padding blocks (keep = 0 or invalid anchor): dq rows and the block's own
// draft keys' dkc / dv get zeros (their dkr is zeroed by the reduction).
__global__ void __launch_bounds__(256) k_bwd_pad(int n_h, int S, int N, int L, const int32_t *anchors,
                                                 const uint8_t *keep, __nv_bfloat16 *dq, __nv_bfloat16 *dkc,
                                                 __nv_bfloat16 *dv) {
    const int n = blockIdx.x, b = blockIdx.y;
    const int a = anchors[(size_t)b * N + n];
    if (keep[(size_t)b * N + n] && a >= 0 && a <= S - 2) return;
    const int R = kBlock * N;
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int h = 0; h < n_h; h++) {
        const size_t bh = (size_t)b * n_h + h;
        uint4 *q4 = reinterpret_cast<uint4 *>(dq + (bh * R + kBlock * n) * kDQK);
        uint4 *k4 = reinterpret_cast<uint4 *>(dkc + (bh * L + S + kBlock * n) * kDC);
        uint4 *v4 = reinterpret_cast<uint4 *>(dv + (bh * L + S + kBlock * n) * kDV);
        for (int e = threadIdx.x; e < kBlock * kDQK / 8; e += blockDim.x) q4[e] = z;
        for (int e = threadIdx.x; e < kBlock * kDC / 8; e += blockDim.x) k4[e] = z;
        for (int e = threadIdx.x; e < kBlock * kDV / 8; e += blockDim.x) v4[e] = z;
    }
}

// ================================================================ dQ
// CTA = (group g of 25 sorted blocks, head h, batch b); warps 0-3 rows
// (thread t = row t = TMEM lane t), warp 4 producer, warp 5 MMA.
// Key tiles are 64 keys wide: an M = 128 MMA costs about the same for N = 32
// and N = 64, so the wider tile halves the MMA count per key.
// Q stays in shared memory (A operand of S = Q K^T); dO is moved into tensor
// memory once at the start (A operand of dP = dO V^T read from TMEM). TMEM:
// dQ 256 columns, S 64, dP 64, dO 128. The row warps write dS (bf16) over the
// S columns they have read, where dQ += dS K reads it as its A operand; the
// next tile's S and dP are issued after that MMA. Shared memory then holds
// only Q and the K / V stages: a K tile is held from its load until the dQ of
// its tile, so it gets three stages, V two. The 64 KB where dO first lands
// then holds the two V stages.
namespace dq {
constexpr int kM = 128, kBN = 64;
constexpr int kQChunk = kM * 128;      // 16 KB: 128 rows x 64 columns
constexpr int kKChunk = kBN * 128;     // 8 KB: 64 keys x 64 columns
constexpr int kTile = 4 * kKChunk;     // 32 KB
constexpr int kKS = 3, kVS = 2;        // K and V stages
// Draft tiles are block-major: block bb's 8 K^C rows (3 x 1 KB swizzled
// slices) at bb * 3 KB, its K^R rows at 24 KB + bb * 1 KB, its V rows
// (4 x 1 KB) at bb * 4 KB.
constexpr int kDraftKcBlock = 3 * 1024, kDraftKr = 3 * kKChunk, kDraftVBlock = 4 * 1024;
constexpr int oQ = 0, oK = oQ + 4 * kQChunk, oV = oK + kKS * kTile, oBar = oV + kVS * kTile;
constexpr int oDOStage = oV;           // dO lands here first
static_assert(kVS * kTile >= 4 * kQChunk, "dO staging area too small");
constexpr int kSmem = oBar + 512 + 1024;
static_assert(kSmem <= 232448, "dynamic shared memory above the sm_100 per-block limit");
constexpr int kThreads = 192;
constexpr uint32_t kColDQ = 0, kColS = 256, kColP = 320, kColDO = 384;  // dO: 384..511
}  // namespace dq

struct BwdArgs {
    int n_h, S, N, W, L, R;
    float scale_log2, scale;
    const __nv_bfloat16 *kc, *krr, *v;
    const __nv_bfloat16 *qs, *dos;
    const float *ds_, *lses;
    const int32_t *cnt, *sorted_n, *sorted_a;
    const float2 *tab;
    __nv_bfloat16 *dq, *dkc, *dv;
    float *dkr_part;
    int hpg;  // heads per head group (key-major kernel)
    int n_ctx_items;
    uint32_t *err;
};

__global__ void __launch_bounds__(dq::kThreads, 1)
    k_bwd_dq_tc(const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_kr,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_qs,
                const __grid_constant__ CUtensorMap tm_dos, const __grid_constant__ CUtensorMap tm_kc8,
                const __grid_constant__ CUtensorMap tm_kr8, const __grid_constant__ CUtensorMap tm_v8, const BwdArgs p) {
    using namespace dq;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + oBar);
    uint64_t *kfull = bars + 0, *kempty = bars + kKS, *vfull = bars + 2 * kKS, *vempty = bars + 2 * kKS + kVS;
    uint64_t *sfull = bars + 2 * (kKS + kVS), *dsready = sfull + 2, *dqdone = sfull + 4, *qfull = sfull + 6,
             *drain = sfull + 7, *dotmem = sfull + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sfull + 9);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sfull + 10);
    int *counters = reinterpret_cast<int *>(sfull + 11);  // K issued, V issued, K consumed, V consumed, q issued

    const int g = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int cnt = p.cnt[b];
    const int i0 = g * kG;
    if (i0 >= cnt) return;
    const int gcnt = min(kG, cnt - i0);
    const int nrows = kBlock * gcnt;
    const int32_t *sa = p.sorted_a + (size_t)b * p.N + i0;
    const int32_t *sn = p.sorted_n + (size_t)b * p.N + i0;
    const int ctx_lo = max(0, sa[0] - p.W + 1);
    const int ctx_hi = sa[gcnt - 1];
    const int n_ctx = ctx_hi > ctx_lo ? (ctx_hi - ctx_lo + kBN - 1) / kBN : 0;
    constexpr int kDraftBlocks = kBN / 8;  // draft tiles: 8 key slots per block
    const int n_draft = (gcnt + kDraftBlocks - 1) / kDraftBlocks;
    const int T = n_ctx + n_draft;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t bh = (size_t)b * p.n_h + h;
    const size_t srow0 = bh * p.R + (size_t)kBlock * i0;  // first sorted row of the group

    // K stages start zeroed (masked key slots must hold finite values)
    for (int e = threadIdx.x; e < (oV - oK) / 16; e += blockDim.x)
        reinterpret_cast<uint4 *>(sm + oK)[e] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kKS; s++) {
            mbar_init(&kfull[s], 1);
            mbar_init(&kempty[s], 1);
        }
        for (int s = 0; s < kVS; s++) {
            mbar_init(&vfull[s], 1);
            mbar_init(&vempty[s], 1);
        }
        mbar_init(sfull, 1);
        mbar_init(dsready, 4);
        for (int s = 0; s < 2; s++) mbar_init(&dqdone[s], 1);
        mbar_init(qfull, 1);
        mbar_init(drain, 1);
        mbar_init(dotmem, 4);
        *abort_flag = 0;
        for (int c = 0; c < 5; c++) counters[c] = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ------------------------------------------------------- producer
        if (lane == 0) {
            mbar_arrive_expect_tx(qfull, 8 * kQChunk);
            tma_load_3d(sm + oQ, &tm_qs, qfull, 0, (int)srow0, 0);
            tma_load_3d(sm + oDOStage, &tm_dos, qfull, 0, (int)srow0, 0);
            counters[4] = 1;
        }
        // lane l holds the block index of group block l (l < gcnt)
        const int my_n = lane < gcnt ? sn[lane] : 0;
        for (int t = 0; t < T; ++t) {
            const int ks = t % kKS, vs = t % kVS;
            uint8_t *kt = sm + oK + ks * kTile;
            uint8_t *vt = sm + oV + vs * kTile;
            if (t >= kKS && !warp_all(mbar_wait(&kempty[ks], ((t / kKS) - 1) & 1, abort_flag))) break;
            if (t < n_ctx) {
                const int pos0 = ctx_lo + t * kBN;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&kfull[ks], kTile);
                    tma_load_3d(kt, &tm_kc, &kfull[ks], 0, (int)(bh * p.L + pos0), 0);
                    tma_load_2d(kt + 3 * kKChunk, &tm_kr, &kfull[ks], 0, (int)((size_t)b * p.L + pos0));
                }
            } else {
                // draft tile: 8 key slots per block (its 5 keys, then 3 masked rows)
                const int d = t - n_ctx;
                const int nb = min(kDraftBlocks, gcnt - d * kDraftBlocks);
                if (lane == 0) mbar_arrive_expect_tx(&kfull[ks], nb * 8 * kDQK * 2);
                for (int bb = 0; bb < nb; ++bb) {
                    const int n = __shfl_sync(0xffffffffu, my_n, d * kDraftBlocks + bb);
                    if (lane == 0) {
                        const int row = p.S + kBlock * n;
                        tma_load_3d(kt + bb * kDraftKcBlock, &tm_kc8, &kfull[ks], 0, (int)(bh * p.L + row), 0);
                        tma_load_2d(kt + kDraftKr + bb * 1024, &tm_kr8, &kfull[ks], 0, (int)((size_t)b * p.L + row));
                    }
                }
            }
            if (lane == 0) counters[0] = t + 1;
            // the V stages hold dO until the row warps have moved it to TMEM
            if (t == 0 && !warp_all(mbar_wait(dotmem, 0, abort_flag))) break;
            if (t >= kVS && !warp_all(mbar_wait(&vempty[vs], ((t / kVS) - 1) & 1, abort_flag))) break;
            if (t < n_ctx) {
                const int pos0 = ctx_lo + t * kBN;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&vfull[vs], kTile);
                    tma_load_3d(vt, &tm_v, &vfull[vs], 0, (int)(bh * p.L + pos0), 0);
                }
            } else {
                const int d = t - n_ctx;
                const int nb = min(kDraftBlocks, gcnt - d * kDraftBlocks);
                if (lane == 0) mbar_arrive_expect_tx(&vfull[vs], nb * 8 * kDV * 2);
                for (int bb = 0; bb < nb; ++bb) {
                    const int n = __shfl_sync(0xffffffffu, my_n, d * kDraftBlocks + bb);
                    if (lane == 0) {
                        const int row = p.S + kBlock * n;
                        tma_load_3d(vt + bb * kDraftVBlock, &tm_v8, &vfull[vs], 0, (int)(bh * p.L + row), 0);
                    }
                }
            }
            if (lane == 0) counters[1] = t + 1;
        }
    } else if (warp == 5) {
        // ----------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idS = idesc_bf16(kM, kBN, 0);    // S, dP: B = K / V tile, K-major
            const uint32_t idQ = idesc_bf16(kM, kDQK, 1);   // dQ: B = K tile, MN-major
            const SDesc qd = sdesc_split(sdesc_sw128(smem_u32(sm + oQ), 16, 1024));
            bool ok = mbar_wait(qfull, 0, abort_flag);
            if (ok) ok = mbar_wait(dotmem, 0, abort_flag);
            const uint32_t idQc = idesc_bf16(kM, kDC, 1);   // draft tiles: dQ^C and dQ^R separately
            const uint32_t idQr = idesc_bf16(kM, kDR, 1);
            auto issue_sdp = [&](int t) {
                const bool ctx = t < n_ctx;
                const uint32_t kb = smem_u32(sm + oK + (t % kKS) * kTile), vb = smem_u32(sm + oV + (t % kVS) * kTile);
                // B operands: context tile slices 8 KB apart with keys 128 B
                // apart; draft tile block-major (K^C / V 8-key groups 3 KB / 4 KB
                // apart, slices 1 KB apart; K^R at 24 KB)
                const uint32_t step = ctx ? kKChunk : 1024;
                const SDesc kd = sdesc_split(sdesc_sw128(kb, 16, ctx ? 1024 : kDraftKcBlock));
                const SDesc krd = sdesc_split(sdesc_sw128(kb + kDraftKr, 16, 1024));
                const SDesc vd = sdesc_split(sdesc_sw128(vb, 16, ctx ? 1024 : kDraftVBlock));
                const uint32_t dS = tmem + kColS, dP = tmem + kColP;
                // S and dP interleaved: two independent accumulation chains
#pragma unroll
                for (int k = 0; k < kDQK / 16; ++k) {
                    const int c = k >> 2;
                    const uint32_t sub = (k & 3) * 2;
                    const uint32_t qo = ((k >> 2) * kQChunk + (k & 3) * 32) >> 4;
                    const uint64_t kbd = c < 3 ? kd.at(((c * step) >> 4) + sub) : krd.at(sub);
                    mma_bf16_ss(dS, qd.at(qo), kbd, idS, k > 0 ? 1u : 0u);
                    mma_bf16_ts(dP, tmem + kColDO + 8 * k, vd.at(((c * step) >> 4) + sub), idS, k > 0 ? 1u : 0u);
                }
                mma_commit(sfull);
                mma_commit(&vempty[t % kVS]);
            };
            // Issue whichever is ready first: S/dP of tile ns (its K and V
            // landed, and the dQ of tile ns - 1, which reads the dS written
            // over the S columns, is issued) or dQ of tile nq (its dS is in
            // TMEM).
            int ns = 0, nq = 0;
            uint64_t t_idle = 0;
            if (ok) tc_fence_after();
            while (ok && nq < T) {
                bool issued = false;
                if (ns < T && ns <= nq) {
                    if (mbar_test(&kfull[ns % kKS], (ns / kKS) & 1) && mbar_test(&vfull[ns % kVS], (ns / kVS) & 1)) {
                        counters[2] = ns + 1;
                        counters[3] = ns + 1;
                        tc_fence_after();
                        issue_sdp(ns);
                        ++ns;
                        issued = true;
                    }
                }
                if (!issued && nq < ns && mbar_test(dsready, nq & 1)) {
                    const int s = nq & 1;
                    tc_fence_after();
                    const uint32_t da = tmem + kColS;  // dS: 64 keys as 32 columns of bf16 pairs
                    const uint32_t kb = smem_u32(sm + oK + (nq % kKS) * kTile);
                    if (nq < n_ctx) {  // B: all 256 columns, slices 8 KB apart, 16 keys = 2 KB
                        const SDesc kd = sdesc_split(sdesc_sw128(kb, kKChunk, 1024));
                        mma_bf16_ts(tmem + kColDQ, da, kd.at(0), idQ, nq > 0 ? 1u : 0u);
#pragma unroll
                        for (int k = 1; k < kBN / 16; ++k) mma_bf16_ts(tmem + kColDQ, da + 8 * k, kd.at(128 * k), idQ, 1u);
                    } else {  // block-major: K^C (slices 1 KB apart, 2 blocks = 6 KB) and K^R (2 KB)
                        const SDesc kdc = sdesc_split(sdesc_sw128(kb, 1024, kDraftKcBlock));
                        const SDesc kdr = sdesc_split(sdesc_sw128(kb + kDraftKr, 1024, 1024));
#pragma unroll
                        for (int k = 0; k < kBN / 16; ++k) {
                            const uint32_t acc = (nq > 0 || k > 0) ? 1u : 0u;
                            mma_bf16_ts(tmem + kColDQ, da + 8 * k, kdc.at(((2 * kDraftKcBlock) >> 4) * k), idQc, acc);
                            mma_bf16_ts(tmem + kColDQ + kDC, da + 8 * k, kdr.at(128 * k), idQr, acc);
                        }
                    }
                    mma_commit(&kempty[nq % kKS]);
                    mma_commit(&dqdone[s]);
                    ++nq;
                    issued = true;
                }
                if (issued) {
                    t_idle = 0;
                } else {
                    const uint64_t now = globaltimer();
                    if (t_idle == 0) t_idle = now;
                    if (*abort_flag) ok = false;
                    else if (now - t_idle > kWaitTimeoutNs) {
                        *abort_flag = 1;
                        ok = false;
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------ rows (warps 0-3)
        const int r = threadIdx.x;
        const bool live = r < nrows;
        int A = 0, n = 0, j = 0, lo = 0;
        float lse2 = 0.f, Dr = 0.f;
        if (live) {
            A = sa[r / kBlock];
            n = sn[r / kBlock];
            j = r % kBlock;
            lo = max(0, A - p.W + 1);
            lse2 = p.lses[srow0 + r];
            Dr = p.ds_[srow0 + r];
        }
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        bool ok = warp_all(mbar_wait(qfull, 0, abort_flag));
        {
            // dO row r: shared memory (128-byte swizzled, 64-column chunks) ->
            // TMEM lane r, columns kColDO.. (bf16 pairs, 8 per 16-byte unit)
#pragma unroll 1
            for (int c = 0; c < 4; c++) {
                uint32_t w[32];
#pragma unroll
                for (int u = 0; u < 8; u++) {
                    const uint4 val = *reinterpret_cast<const uint4 *>(sm + oDOStage + c * kQChunk + sw128(r, u));
                    w[4 * u + 0] = val.x;
                    w[4 * u + 1] = val.y;
                    w[4 * u + 2] = val.z;
                    w[4 * u + 3] = val.w;
                }
                tmem_st32u(trow + kColDO + 32 * c, w);
            }
            // the V stages now hold dO rows or zero fill: finite, as masked
            // key slots of draft tiles need
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dotmem);
        }
        for (int t = 0; t < T && ok; ++t) {
            const int s = t & 1;
            ok = warp_all(mbar_wait(sfull, t & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            float sv[64], pv[64];
            {
                float a0[32], a1[32], b0[32], b1[32];
                tmem_ld32(trow + kColS, a0);
                tmem_ld32(trow + kColS + 32, a1);
                tmem_ld32(trow + kColP, b0);
                tmem_ld32(trow + kColP + 32, b1);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; c++) {
                    sv[c] = a0[c];
                    sv[32 + c] = a1[c];
                    pv[c] = b0[c];
                    pv[32 + c] = b1[c];
                }
            }
            (void)s;
            // the row's keys in this tile: one contiguous column range [clo, chi)
            int clo, chi;
            if (t < n_ctx) {
                const int c0 = ctx_lo + t * kBN;
                clo = lo - c0;
                chi = A - c0;
            } else {
                clo = 8 * (r / kBlock) - (t - n_ctx) * kBN;
                chi = clo + kBlock;
            }
            if (!live) chi = clo;
            uint32_t dsw[kBN / 2];  // dS as bf16 pairs, over the S columns just read
#pragma unroll
            for (int c = 0; c < kBN; c += 2) {
                float e[2];
#pragma unroll
                for (int d = 0; d < 2; d++) {
                    const float pp = (c + d >= clo && c + d < chi) ? ex2(fmaf(sv[c + d], p.scale_log2, -lse2)) : 0.f;
                    e[d] = pp * (pv[c + d] - Dr) * p.scale;
                }
                dsw[c / 2] = pack_bf16x2(e[0], e[1]);
            }
            tmem_st32u(trow + kColS, dsw);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dsready);
        }
        if (ok) ok = warp_all(mbar_wait(&dqdone[(T - 1) & 1], ((T - 1) >> 1) & 1, abort_flag));
        if (ok) {
            tc_fence_after();
            // dQ row (rope slice rotated back by A + j) -> staging in the idle
            // K stages (unit u of row r at u ^ (r & 31)) -> one 512-byte row
            // per warp instruction
            uint8_t *stage = sm + oK + warp * (32 * kDQK * 2);
#pragma unroll 1
            for (int c = 0; c < kDQK; c += 32) {
                float v[32];
                tmem_ld32(trow + kColDQ + c, v);
                tmem_wait_ld();
                if (c >= kDC) {  // rope slice: rotate back by the query position A + j
                    const float2 *cs = p.tab + (size_t)(A + j) * (kDR / 2) + (c - kDC) / 2;
#pragma unroll
                    for (int k = 0; k < 16; k++) {
                        const float2 t2 = live ? __ldg(cs + k) : make_float2(1.f, 0.f);
                        const float x0 = v[2 * k], x1 = v[2 * k + 1];
                        v[2 * k] = x0 * t2.x + x1 * t2.y;
                        v[2 * k + 1] = x1 * t2.x - x0 * t2.y;
                    }
                }
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    const int u = c / 8 + k;
                    *reinterpret_cast<uint4 *>(stage + lane * 512 + ((u ^ lane) << 4)) = make_uint4(
                        pack_bf16x2(v[8 * k + 0], v[8 * k + 1]), pack_bf16x2(v[8 * k + 2], v[8 * k + 3]),
                        pack_bf16x2(v[8 * k + 4], v[8 * k + 5]), pack_bf16x2(v[8 * k + 6], v[8 * k + 7]));
                }
            }
            __syncwarp();
            for (int i = 0; i < 32; i++) {
                const int rr = warp * 32 + i;
                if (rr >= nrows) break;  // uniform
                const int ni = __shfl_sync(0xffffffffu, n, i), ji = __shfl_sync(0xffffffffu, j, i);
                const uint4 val = *reinterpret_cast<const uint4 *>(stage + i * 512 + ((lane ^ i) << 4));
                *reinterpret_cast<uint4 *>(p.dq + (bh * p.R + kBlock * ni + ji) * kDQK + 8 * lane) = val;
            }
        }
    }

    __syncthreads();
    if (*abort_flag) {
        volatile int never = 0;
        if (warp == 4 && lane == 0) {
            if (counters[4]) mbar_wait(qfull, 0, (volatile int *)&never);
            for (int t = counters[2]; t < counters[0]; ++t)
                mbar_wait(&kfull[t % kKS], (t / kKS) & 1, (volatile int *)&never);
            for (int t = counters[3]; t < counters[1]; ++t)
                mbar_wait(&vfull[t % kVS], (t / kVS) & 1, (volatile int *)&never);
        }
        if (warp == 5 && lane == 0) {
            mma_commit(drain);
            mbar_wait(drain, 0, (volatile int *)&never);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x == 0 && *abort_flag) atomicOr(p.err, kErrTimeout);
}

// ============================================================== dK / dV
// Key tile = 64 keys (MMA M = 64); dK and dV of the tile in one CTA, so K, V
// and every row of Q and dO that sees the tile cross into shared memory once.
// With M = 64 an accumulator occupies lanes 0-15 of each 32-lane TMEM
// sub-partition, and a second one addressed at lane offset 16 the lanes 16-31
// of the same columns: dK (offset 0) and dV (offset 16) share columns 0..255,
// S^T (0) and dP^T (16) share a 64-column buffer (two buffers, columns 256 and
// 320). dK's columns 192..255 are the rope slice: it is summed over the heads
// of the group, so that part of the accumulator is never reset between heads.
// Per head: the K^C and V tiles (one stage, reloaded once the head's last
// S^T / dP^T completed; the rope-key tile is the same for all heads and is
// loaded once), then the rows that see the tile in chunks of 64 (Q and dO,
// two stages): S^T = K Q^T and dP^T = V dO^T, P^T and dS^T (bf16) through one
// shared-memory buffer, dV += P^T dO, dK += dS^T Q.
// Key warps: warp w covers keys 16 (w & 3) .. + 15 (TMEM sub-partition w & 3)
// and rows 32 (w >> 2) .. + 31 of a chunk. Lane l < 16 loads S^T of its key,
// lane l + 16 dP^T of the same key; the two swap halves, so each lane holds
// both for 16 rows. At a head's end they copy the accumulators, as bf16, into
// the 128 free TMEM columns (the stash), which frees them for the next head;
// four store warps write the stash out to dK^C / dV while the next head runs.
namespace kv {
constexpr int kMK = 64;                    // keys per tile (MMA M)
constexpr int kRC = 64;                    // rows per chunk (MMA N of S^T / dP^T, K of the accumulations)
constexpr int kSlice = 64 * 128;           // 8 KB: 64 keys or rows x 64 columns, 128-byte swizzled
// Draft tiles are block-major: block bb's 8 K^C rows (3 x 1 KB swizzled
// slices) at bb * 3 KB, its K^R rows at bb * 1 KB of the rope-key tile, its V
// rows (4 x 1 KB) at bb * 4 KB: 8-key groups 3 KB / 4 KB apart, 64-column
// slices 1 KB apart.
constexpr int kDraftKcBlock = 3 * 1024, kDraftVBlock = 4 * 1024;
constexpr int oKr = 0, oKc = oKr + kSlice, oV = oKc + 3 * kSlice;
constexpr int kRowStage = 8 * kSlice;      // Q chunk (4 slices), then dO chunk (4 slices)
constexpr int oRow = oV + 4 * kSlice;
constexpr int oPT = oRow + 2 * kRowStage;  // P^T, then dS^T: [64 keys][64 rows] bf16 each
constexpr int oStage = oPT + 2 * kSlice;   // epilogue staging, 2 KB per store warp
constexpr int oMeta = oStage + 4 * 2048;   // per row stage: (LSE * log2 e, D) of each row
constexpr int oBar = oMeta + 2 * kRC * 8;
constexpr int kSmem = oBar + 256 + 1024;
static_assert(kSmem <= 232448, "dynamic shared memory above the sm_100 per-block limit");
constexpr int kKeyWarps = 8;
constexpr int kWarpKV = kKeyWarps, kWarpRow = kKeyWarps + 1, kWarpMma = kKeyWarps + 2;
constexpr int kWarpSt = kKeyWarps + 3;     // four store warps, one per TMEM sub-partition
constexpr int kThreads = (kKeyWarps + 7) * 32;
constexpr uint32_t kColAcc = 0, kColS = 256;  // S^T / dP^T buffer s at kColS + 64 s
constexpr uint32_t kColStash = 384;           // a finished head's dK / dV as bf16 pairs (128 columns)
constexpr uint32_t kHi = 16u << 16;           // lane offset of the second M = 64 accumulator
}  // namespace kv

// One CTA per (64-key tile, head group, batch row).
__global__ void __launch_bounds__(kv::kThreads, 1)
    k_bwd_kv_tc(const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_kr,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_qs,
                const __grid_constant__ CUtensorMap tm_dos, const __grid_constant__ CUtensorMap tm_kc8,
                const __grid_constant__ CUtensorMap tm_kr8, const __grid_constant__ CUtensorMap tm_v8,
                const BwdArgs p) {
    using namespace kv;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + oBar);
    uint64_t *kvfull = bars + 0, *kvfree = bars + 1, *rowfull = bars + 2, *rowfree = bars + 4, *sfull = bars + 6,
             *dsready = bars + 8, *ptfree = bars + 9, *drain = bars + 10, *stashfull = bars + 11,
             *stashfree = bars + 12;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 13);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    // K/V heads issued, row chunks issued, K/V heads consumed, row chunks consumed
    int *counters = reinterpret_cast<int *>(tmem_slot + 2);
    int *band = counters + 4;  // first sorted row, row count

    const int item = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cnt = p.cnt[b];
    const bool is_ctx = item < p.n_ctx_items;
    int t0 = 0, gcnt = 0, i0 = 0;
    if (is_ctx) {
        t0 = item * kMK;
    } else {
        i0 = (item - p.n_ctx_items) * kGD;
        if (i0 >= cnt) return;  // uniform: fewer draft tiles in this batch row
        gcnt = min(kGD, cnt - i0);
    }
    const int32_t *sa = p.sorted_a + (size_t)b * p.N;
    const int32_t *sn = p.sorted_n + (size_t)b * p.N;
    if (threadIdx.x == 0) {
        int r0, nr;
        if (is_ctx) {
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
            r0 = kBlock * lo;
            nr = kBlock * (lo2 - lo);
        } else {
            r0 = kBlock * i0;
            nr = kBlock * gcnt;
        }
        band[0] = r0;
        band[1] = nr;
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
    bool key_valid = false;
    size_t key_pos = 0;
    if (warp < kKeyWarps || warp >= kWarpSt) {
        if (is_ctx) {
            key_valid = t0 + kk < p.S;
            key_pos = (size_t)t0 + kk;
        } else {  // 8 key slots per block: its 5 keys, then 3 masked rows
            key_valid = kk / 8 < gcnt && kk % 8 < kBlock;
            if (key_valid) key_pos = (size_t)p.S + kBlock * sn[i0 + kk / 8] + kk % 8;
        }
    }
    float *dkr_part_row = p.dkr_part + (((size_t)hg * gridDim.z + b) * p.L + key_pos) * kDR;

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
    for (int e = threadIdx.x; e < (oRow - oKr) / 16; e += blockDim.x)
        reinterpret_cast<uint4 *>(sm + oKr)[e] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        mbar_init(kvfull, 1);
        mbar_init(kvfree, 1);
        for (int s = 0; s < 2; s++) {
            mbar_init(&rowfull[s], 1);
            mbar_init(&rowfree[s], 1);
            mbar_init(&sfull[s], 1);
        }
        mbar_init(dsready, kKeyWarps);
        mbar_init(ptfree, 1);
        mbar_init(drain, 1);
        mbar_init(stashfull, kKeyWarps);
        mbar_init(stashfree, 4);
        *abort_flag = 0;
        for (int c = 0; c < 4; c++) counters[c] = 0;
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
        const int my_n = (!is_ctx && lane < gcnt) ? sn[i0 + lane] : 0;
        for (int hh = 0; hh < H; ++hh) {
            const size_t bh = (size_t)b * p.n_h + h0 + hh;
            if (hh >= 1 && !warp_all(mbar_wait(kvfree, (hh - 1) & 1, abort_flag))) break;
            if (is_ctx) {
                if (lane == 0) {
                    mbar_arrive_expect_tx(kvfull, (hh == 0 ? 8 : 7) * kSlice);
                    if (hh == 0) tma_load_2d(sm + oKr, &tm_kr, kvfull, 0, (int)((size_t)b * p.L + t0));
                    tma_load_3d(sm + oKc, &tm_kc, kvfull, 0, (int)(bh * p.L + t0), 0);
                    tma_load_3d(sm + oV, &tm_v, kvfull, 0, (int)(bh * p.L + t0), 0);
                }
            } else {
                if (lane == 0) mbar_arrive_expect_tx(kvfull, gcnt * 8 * ((hh == 0 ? kDQK : kDC) + kDV) * 2);
                for (int bb = 0; bb < gcnt; ++bb) {
                    const int nb = __shfl_sync(0xffffffffu, my_n, bb);
                    if (lane == 0) {
                        const int row = p.S + kBlock * nb;
                        tma_load_3d(sm + oKc + bb * kDraftKcBlock, &tm_kc8, kvfull, 0, (int)(bh * p.L + row), 0);
                        if (hh == 0)
                            tma_load_2d(sm + oKr + bb * 1024, &tm_kr8, kvfull, 0, (int)((size_t)b * p.L + row));
                        tma_load_3d(sm + oV + bb * kDraftVBlock, &tm_v8, kvfull, 0, (int)(bh * p.L + row), 0);
                    }
                }
            }
            if (lane == 0) counters[0] = hh + 1;
        }
    } else if (warp == kWarpRow) {
        // ---------------------------- producer of Q / dO chunks and row data
        for (int q = 0; q < QT; ++q) {
            const int hh = q / nchunks, c = q % nchunks, s = q & 1;
            const size_t bh = (size_t)b * p.n_h + h0 + hh;
            const int r0 = row0 + c * kRC;
            if (q >= 2 && !warp_all(mbar_wait(&rowfree[s], ((q >> 1) - 1) & 1, abort_flag))) break;
            float2 *mLD = reinterpret_cast<float2 *>(sm + oMeta + s * kRC * 8);
#pragma unroll
            for (int jj = 0; jj < kRC; jj += 32) {
                const int rowi = r0 + jj + lane;
                mLD[jj + lane] = rowi < row0 + nrows ? make_float2(p.lses[bh * p.R + rowi], p.ds_[bh * p.R + rowi])
                                                     : make_float2(0.f, 0.f);
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_expect_tx(&rowfull[s], kRowStage);
                tma_load_3d(sm + oRow + s * kRowStage, &tm_qs, &rowfull[s], 0, (int)(bh * p.R + r0), 0);
                tma_load_3d(sm + oRow + s * kRowStage + 4 * kSlice, &tm_dos, &rowfull[s], 0, (int)(bh * p.R + r0), 0);
                counters[1] = q + 1;
            }
        }
    } else if (warp == kWarpMma) {
        // ----------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idS = idesc_bf16(kMK, kRC, 0);   // S^T, dP^T: B = Q / dO chunk, K-major
            const uint32_t idV = idesc_bf16(kMK, kDV, 1);   // dV: B = dO chunk, MN-major
            const uint32_t idKc = idesc_bf16(kMK, kDC, 1);  // dK^C: B = Q^C columns
            const uint32_t idKr = idesc_bf16(kMK, kDR, 1);  // dK^R: B = Q^R columns
            // A operands: K^C / V slices kcStep / vStep bytes apart (context
            // tile: 8 KB slices of 64 keys; draft tile: block-major)
            const uint32_t kcStep = is_ctx ? kSlice : 1024, vStep = is_ctx ? kSlice : 1024;
            const SDesc kad = sdesc_split(sdesc_sw128(smem_u32(sm + oKc), 16, is_ctx ? 1024 : kDraftKcBlock));
            const SDesc krd = sdesc_split(sdesc_sw128(smem_u32(sm + oKr), 16, 1024));
            const SDesc vad = sdesc_split(sdesc_sw128(smem_u32(sm + oV), 16, is_ctx ? 1024 : kDraftVBlock));
            const SDesc ptd = sdesc_split(sdesc_sw128(smem_u32(sm + oPT), 16, 1024));
            const SDesc dsd = sdesc_split(sdesc_sw128(smem_u32(sm + oPT + kSlice), 16, 1024));
            bool ok = true;
            auto issue_s = [&](int q) {
                const int c = q % nchunks, s = q & 1;
                tc_fence_after();
                const uint32_t rs = smem_u32(sm + oRow + s * kRowStage);
                const SDesc qd = sdesc_split(sdesc_sw128(rs, 16, 1024));
                const SDesc dod = sdesc_split(sdesc_sw128(rs + 4 * kSlice, 16, 1024));
                const uint32_t dS = tmem + kColS + 64 * s, dP = dS + kHi;
                // S^T = K Q^T and dP^T = V dO^T interleaved: two independent chains
#pragma unroll
                for (int k16 = 0; k16 < kDQK / 16; ++k16) {
                    const int cc = k16 >> 2;
                    const uint32_t sub = (k16 & 3) * 2;  // 32 bytes, in 16-byte units
                    const uint64_t ka = cc < 3 ? kad.at(((cc * kcStep) >> 4) + sub) : krd.at(sub);
                    const uint32_t ro = (cc * kSlice + (k16 & 3) * 32) >> 4;
                    mma_bf16_ss(dS, ka, qd.at(ro), idS, k16 > 0 ? 1u : 0u);
                    mma_bf16_ss(dP, vad.at(((cc * vStep) >> 4) + sub), dod.at(ro), idS, k16 > 0 ? 1u : 0u);
                }
                mma_commit(&sfull[s]);
                if (c == nchunks - 1) mma_commit(kvfree);
            };
            auto issue_acc = [&](int q) {
                const int c = q % nchunks, s = q & 1;
                tc_fence_after();
                const uint32_t rs = smem_u32(sm + oRow + s * kRowStage);
                const SDesc qb = sdesc_split(sdesc_sw128(rs, kSlice, 1024));            // MN-major
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
                mma_commit(ptfree);
            };
            // Issue whichever is ready: the S^T stage of chunk ns (its K/V tile
            // and row operands landed; at most one chunk ahead, so its S^T /
            // dP^T buffer was read by the key warps before they signalled chunk
            // ns - 2) or the accumulation of chunk na (P^T / dS^T written; at a
            // head's first chunk the key warps have also read the previous
            // head's accumulators, which precedes that signal).
            int ns = 0, na = 0;
            uint64_t t_idle = 0;
            while (ok && na < QT) {
                bool issued = false;
                if (ns < QT && ns <= na + 1) {
                    const int hh = ns / nchunks, c = ns % nchunks;
                    if ((c != 0 || mbar_test(kvfull, hh & 1)) && mbar_test(&rowfull[ns & 1], (ns >> 1) & 1)) {
                        if (c == 0) counters[2] = hh + 1;
                        counters[3] = ns + 1;
                        issue_s(ns);
                        ++ns;
                        issued = true;
                    }
                }
                if (!issued && na < ns && mbar_test(dsready, na & 1)) {
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
                    else if (now - t_idle > kWaitTimeoutNs) {
                        *abort_flag = 1;
                        ok = false;
                    }
                }
            }
        }
    } else if (warp >= kWarpSt) {
        // ------------------------------------------------ store warps
        // Sub-partition warp & 3: keys 16 (warp & 3) .. + 15, lanes 0-15 their
        // dK, lanes 16-31 their dV. Per head: the stash (128 columns of bf16
        // pairs: accumulator columns 128 hr + 32 rd .. + 31 at stash column
        // 64 hr + 16 rd) in eight rounds of 32 values; each thread stages its
        // 64 bytes (16-byte unit u at u ^ (lane & 3)), then the warp writes 8
        // rows' 64-byte segments per instruction. dK columns 192..255 (the
        // rope slice) are not written: they stay in TMEM, summed over heads.
        const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        uint8_t *stage = sm + oStage + (warp - kWarpSt) * 2048;
        for (int hh = 0; hh < H; ++hh) {
            if (!warp_all(mbar_wait(stashfull, hh & 1, abort_flag))) break;
            tc_fence_after();
            const size_t bh = (size_t)b * p.n_h + h0 + hh;
#pragma unroll 1
            for (int rr = 0; rr < 4; rr++) {
                float v[32];
                tmem_ld32(trow + kColStash + 32 * rr, v);
                tmem_wait_ld();
                if (rr == 3) {  // the stash is free for the next head
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(stashfree);
                }
#pragma unroll
                for (int sub = 0; sub < 2; sub++) {
                    const int col = (rr >> 1) * 128 + ((rr & 1) * 2 + sub) * 32;
                    const bool rope = col >= kDC;
#pragma unroll
                    for (int u = 0; u < 4; u++)
                        *reinterpret_cast<uint4 *>(stage + lane * 64 + ((u ^ (lane & 3)) << 4)) =
                            make_uint4(__float_as_uint(v[16 * sub + 4 * u]), __float_as_uint(v[16 * sub + 4 * u + 1]),
                                       __float_as_uint(v[16 * sub + 4 * u + 2]),
                                       __float_as_uint(v[16 * sub + 4 * u + 3]));
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        const int kl = 8 * i + (lane >> 2), u = lane & 3;  // source lane, unit
                        const int kvl = __shfl_sync(0xffffffffu, (int)key_valid, kl);
                        const long long kposl = __shfl_sync(0xffffffffu, (long long)key_pos, kl);
                        const bool is_v = kl >= 16;
                        if (kvl && (is_v || !rope)) {
                            const uint4 val =
                                *reinterpret_cast<const uint4 *>(stage + kl * 64 + ((u ^ (kl & 3)) << 4));
                            __nv_bfloat16 *dst = is_v ? p.dv + (bh * p.L + (size_t)kposl) * kDV + col + 8 * u
                                                      : p.dkc + (bh * p.L + (size_t)kposl) * kDC + col + 8 * u;
                            *reinterpret_cast<uint4 *>(dst) = val;
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
            if (is_ctx) {
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
            } else {
                rlo = kBlock * (kk / 8);
                rhi = rlo + kBlock;
            }
        }
        // this key's row of the P^T / dS^T tiles (128-byte swizzle) and the
        // two 16-byte units that hold rows rb .. rb + 15
        const uint32_t prow = (uint32_t)((kk >> 3) * 1024 + (kk & 7) * 128);
        const uint32_t pu0 = prow + ((((uint32_t)rb >> 3) ^ (kk & 7)) << 4);
        const uint32_t pu1 = prow + (((((uint32_t)rb >> 3) + 1) ^ (kk & 7)) << 4);
        bool ok = true;
        for (int q = 0; q < QT && ok; ++q) {
            const int hh = q / nchunks, c = q % nchunks, s = q & 1;
            ok = warp_all(mbar_wait(&rowfull[s], (q >> 1) & 1, abort_flag));  // row data
            if (ok) ok = warp_all(mbar_wait(&sfull[s], (q >> 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            float v[32];
            tmem_ld32(trow + kColS + 64 * s + 32 * hr, v);
            tmem_wait_ld();
            float sv[16], pv[16];
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const float send = dlane ? v[i] : v[16 + i];
                const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
                sv[i] = dlane ? recv : v[i];
                pv[i] = dlane ? v[16 + i] : recv;
            }
            const float2 *mLD = reinterpret_cast<const float2 *>(sm + oMeta + s * kRC * 8) + rb;
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
            // the P^T / dS^T buffer is free once the accumulation of chunk q - 1 completed
            if (q >= 1) {
                ok = warp_all(mbar_wait(ptfree, (q - 1) & 1, abort_flag));
                if (!ok) break;
            }
            *reinterpret_cast<uint4 *>(sm + oPT + pu0) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
            *reinterpret_cast<uint4 *>(sm + oPT + pu1) = make_uint4(pw[4], pw[5], pw[6], pw[7]);
            *reinterpret_cast<uint4 *>(sm + oPT + kSlice + pu0) = make_uint4(dw[0], dw[1], dw[2], dw[3]);
            *reinterpret_cast<uint4 *>(sm + oPT + kSlice + pu1) = make_uint4(dw[4], dw[5], dw[6], dw[7]);
            fence_proxy_async_smem();  // visible to the MMAs that read them
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dsready);
            if (c != nchunks - 1) continue;
            // head end, once its accumulations completed and the store warps
            // have read the previous head's stash: accumulator columns
            // [128 hr, 128 hr + 128) (lanes 0-15 dK, 16-31 dV) -> bf16 pairs in
            // stash columns [64 hr, 64 hr + 64). The accumulator is then free
            // for the next head.
            ok = warp_all(mbar_wait(ptfree, q & 1, abort_flag));
            if (ok && hh >= 1) ok = warp_all(mbar_wait(stashfree, (hh - 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int rd = 0; rd < 4; rd++) {
                tmem_ld32(trow + kColAcc + hr * 128 + rd * 32, v);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; i++) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
                tmem_st16u(trow + kColStash + hr * 64 + rd * 16, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(stashfull);
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
            for (int t = counters[2]; t < counters[0]; ++t) mbar_wait(kvfull, t & 1, (volatile int *)&never);
        }
        if (warp == kWarpRow && lane == 0) {
            for (int t = counters[3]; t < counters[1]; ++t)
                mbar_wait(&rowfull[t & 1], (t >> 1) & 1, (volatile int *)&never);
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

// ------------------------------------------------------------ dK^R reduce
// One warp per (b, key): sum the head-group partials (rotated frame), rotate
// back by the key's position, write dkr. Draft keys of padding blocks: 0.
__global__ void __launch_bounds__(256) k_bwd_dkr_reduce(int B, int S, int N, int L, int HG,
                                                        const int32_t *anchors, const uint8_t *keep,
                                                        const float2 *tab, const float *part,
                                                        __nv_bfloat16 *dkr) {
    const size_t wid = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (wid >= (size_t)B * L) return;
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
        for (int g = 0; g < HG; g++) {
            const float2 v = *reinterpret_cast<const float2 *>(part + (((size_t)g * B + b) * L + key) * kDR + 2 * lane);
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

}  // namespace

bool bwd_tc_supported(const Prob &p) {
    return p.dtype == DSPARK_BF16 && p.d_c == kDC && p.d_r == kDR && p.d_v == kDV &&
           (long long)p.B * p.n_h * p.L < (1ll << 31) && (long long)p.B * p.n_h * p.R < (1ll << 31);
}

int bwd_head_groups(const Prob &p) {
    const long long items = (long long)((p.S + kv::kMK - 1) / kv::kMK + (p.N + kGD - 1) / kGD) * p.B;
    // aim for about eight waves on 148 SMs (shorter CTAs, smaller tail)
    int hg = 1;
    while (hg < p.n_h && items * hg < 8 * 148 && p.n_h % (hg * 2) == 0) hg *= 2;
    return hg;
}

cudaError_t launch_bwd_tc(const Prob &p, const void *q, const void *kc, const void *v, const int32_t *anchors,
                          const uint8_t *keep, const void *o, const float *lse, const void *dout, void *dq,
                          void *dkc, void *dkr, void *dv, const Ws &ws, cudaStream_t st) {
    if (p.B == 0) return cudaSuccess;
    const int HG = bwd_head_groups(p);
    if (p.N > 0) {
        count_launch();
        k_bwd_prep<<<dim3(p.N, p.n_h, p.B), 160, 0, st>>>(
            p.n_h, p.N, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)o, (const __nv_bfloat16 *)dout, lse, ws.cnt,
            ws.sorted_n, ws.sorted_a, ws.rope, (__nv_bfloat16 *)ws.qs, (__nv_bfloat16 *)ws.dos, ws.dvec, ws.lses);
        count_launch();
        k_bwd_pad<<<dim3(p.N, p.B), 256, 0, st>>>(p.n_h, p.S, p.N, p.L, anchors, keep, (__nv_bfloat16 *)dq,
                                                   (__nv_bfloat16 *)dkc, (__nv_bfloat16 *)dv);
    }
    CUtensorMap m_kc3_64, m_kr64, m_v3_64, m_qs3_128, m_dos3_128, m_qs3_64, m_dos3_64, m_kr8, m_kc3_8, m_v3_8;
    const uint64_t kv_rows = (uint64_t)p.B * p.n_h * p.L, q_rows = (uint64_t)p.B * p.n_h * p.R;
    const void *qs = ws.qs, *dos = ws.dos;
    if (!make_map3_bf16(&m_kc3_64, kc, kDC, kv_rows, 64) ||
        !make_map_bf16(&m_kr64, ws.kr_rot, kDR, (uint64_t)p.B * p.L, 64) ||
        !make_map3_bf16(&m_v3_64, v, kDV, kv_rows, 64) ||
        !make_map_bf16(&m_kr8, ws.kr_rot, kDR, (uint64_t)p.B * p.L, 8) ||
        !make_map3_bf16(&m_kc3_8, kc, kDC, kv_rows, 8) || !make_map3_bf16(&m_v3_8, v, kDV, kv_rows, 8))
        return cudaErrorInvalidValue;
    if (p.N > 0 && q_rows > 0) {
        if (!make_map3_bf16(&m_qs3_128, qs, kDQK, q_rows, 128) || !make_map3_bf16(&m_dos3_128, dos, kDV, q_rows, 128) ||
            !make_map3_bf16(&m_qs3_64, qs, kDQK, q_rows, 64) || !make_map3_bf16(&m_dos3_64, dos, kDV, q_rows, 64))
            return cudaErrorInvalidValue;
    } else {  // maps over Q rows are never read: any valid map will do
        m_qs3_128 = m_dos3_128 = m_qs3_64 = m_dos3_64 = m_kc3_64;
    }
    BwdArgs a;
    a.n_h = p.n_h; a.S = p.S; a.N = p.N; a.W = p.W; a.L = p.L; a.R = p.R;
    a.scale_log2 = p.scale_log2;
    a.scale = p.scale;
    a.kc = (const __nv_bfloat16 *)kc;
    a.krr = (const __nv_bfloat16 *)ws.kr_rot;
    a.v = (const __nv_bfloat16 *)v;
    a.qs = (const __nv_bfloat16 *)ws.qs;
    a.dos = (const __nv_bfloat16 *)ws.dos;
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
    a.hpg = p.n_h / HG;
    a.n_ctx_items = (p.S + kv::kMK - 1) / kv::kMK;
    a.err = ws.err;
    cudaError_t e;
    if (p.N > 0) {
        e = cudaFuncSetAttribute(k_bwd_dq_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, dq::kSmem);
        if (e != cudaSuccess) return e;
        count_launch();
        k_bwd_dq_tc<<<dim3((p.N + kG - 1) / kG, p.n_h, p.B), dq::kThreads, dq::kSmem, st>>>(
            m_kc3_64, m_kr64, m_v3_64, m_qs3_128, m_dos3_128, m_kc3_8, m_kr8, m_v3_8, a);
    }
    const dim3 kv_grid(a.n_ctx_items + (p.N + kGD - 1) / kGD, HG, p.B);
    e = cudaFuncSetAttribute(k_bwd_kv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kv::kSmem);
    if (e != cudaSuccess) return e;
    count_launch();
    k_bwd_kv_tc<<<kv_grid, kv::kThreads, kv::kSmem, st>>>(m_kc3_64, m_kr64, m_v3_64, m_qs3_64, m_dos3_64, m_kc3_8,
                                                        m_kr8, m_v3_8, a);
    const size_t warps = (size_t)p.B * p.L;
    count_launch();
    k_bwd_dkr_reduce<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(p.B, p.S, p.N, p.L, HG, anchors, keep, ws.rope,
                                                                   ws.dkr_part, (__nv_bfloat16 *)dkr);
    return cudaGetLastError();
}

}  // namespace dspark
