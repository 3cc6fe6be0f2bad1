// Tensor-core (tcgen05 / TMEM / TMA) forward of the DSpark draft attention for
// the page's head widths (d_c = 192, d_r = 64, d_v = 256), bf16.
//
// Work item: (batch b, head h, group of up to 25 kept blocks that are
// consecutive in anchor order) = up to 125 query rows, the M = 128 of one
// MMA. The group's key set is the union of its blocks' context windows,
// [max(0, A_first - W + 1), A_last), walked in 64-key tiles, followed by the
// group's own draft keys (5 per block, in 8 key slots) gathered into tiles of
// 8 blocks (up to 4 more tiles).
// Each row masks every key that is not in its own key set (page "GLM 5.2
// DSpark speculative-training design", §3: window [A-W+1, A) shared by the 5
// offsets, own block bidirectional, other blocks invisible). Because blocks
// are sorted by anchor, neighbouring items read overlapping windows close
// together in time, so the overlap is served by L2.
//
// Persistent: one CTA per SM; each takes its next work item from a global
// counter (items in the order of item_at), so all CTAs stay busy until the
// items run out. K/V tiles, S buffers and pipeline phases are counted over all of a CTA's
// items, so the K/V stream runs on across item boundaries; the next item's
// raw Q rows are staged (and their rope slice rotated) while the current item
// runs, moved into TMEM as soon as its last QK has completed, and the finished
// item's O leaves TMEM through the same staging area, one bulk copy per block,
// while the next item's first QK runs.
// Q lives in tensor memory (A operand of S = Q K^T read from TMEM), and P is
// written over its own S columns (A operand of O += P V read from TMEM).
// TMEM: O 0..255, S 256..319 / 320..383, Q 384..511. Shared memory: two K
// and two V stages, the 64 KB staging area, the softmax pair exchange.
//
// Warp roles (384 threads):
//   warps 0-7  softmax: warps w and w + 4 share TMEM sub-partition w % 4, so
//              query rows 32 (w % 4) .. + 31 (thread = row = TMEM lane), and
//              split each 64-key tile into two 32-column halves. They move
//              the row's half of Q from the staging area into TMEM,
//              turn each S tile into P with an online softmax whose row max
//              the pair exchanges through shared memory, rescale their half
//              of the O row when the running max grows by more than 2^8,
//              stage O and write LSE.
//   warp 8     K producer: TMA loads of context K tiles (K^C as one 3-D box,
//              plus the pre-rotated shared K^R) and of draft-key tiles (per
//              block one 3-D box of its 8 K^C rows and one of its K^R rows).
//   warp 9     TMEM owner and MMA issuer (one thread): S = Q K^T into two
//              alternating S buffers, O += P V, each issued as soon as its
//              inputs are ready (an S buffer is reused only after the P V
//              that reads the P written over it; an item's first QK after
//              its Q is in TMEM, its first P V after the previous item's O
//              has been read out).
//   warp 10    V producer.
//   warp 11    raw Q loader (one bulk copy per block of 5 rows), which then
//              RoPE-rotates the staged rows' rope slice in place, and O writer
//              (one bulk copy per block of 5 staged O rows).
// Every mbarrier wait is bounded; on time-out the CTA raises an abort flag,
// all roles leave their loops, in-flight copies and MMAs are drained with a
// bounded wait, TMEM is freed and the workspace error word gets kErrTimeout.
#include <algorithm>

#include "dspark_tc_common.cuh"

namespace dspark {

namespace {

using namespace tc;

constexpr int kG = 25;    // blocks per work item
constexpr int kM = 128;   // query rows per work item (MMA M)
constexpr int kBN = 64;   // keys per tile
constexpr int kDC = 192, kDR = 64, kDQK = 256, kDV = 256;

constexpr int kKChunk = kBN * 128;  // one 64-column slice of a K or V tile
constexpr int kKBytes = 4 * kKChunk;
constexpr int kVBytes = 4 * kKChunk;
constexpr int kKS = 2, kVS = 2;     // K and V stages

// Shared memory: K0 K1 V0 V1, then the staging area (the next item's raw Q
// rows; then, once they are in TMEM, the finished item's O rows on their way
// to global memory, in the same layout), then the softmax pair exchange and
// the barriers.
constexpr int oStage = 4 * kKBytes;
constexpr int kStageBytes = 64 * 1024;
constexpr int oX = oStage + kStageBytes;  // pair exchange: tile max [2][2][128], row sum [2][128] (floats)
constexpr int oBar = oX + 3 * 1024;
__device__ __forceinline__ int k_stage_off(int s) { return s * kKBytes; }
__device__ __forceinline__ int v_stage_off(int s) { return (2 + s) * kKBytes; }
// Raw Q and O: one bulk copy per block (5 rows of 512 B), blocks 2576 B
// apart, so the rows that the threads of a warp access at once fall on at
// most 5 rows per bank group.
constexpr int kStageBlockPitch = kBlock * kDQK * 2 + 16;
static_assert(kG * kStageBlockPitch <= kStageBytes, "staging area too small for raw Q and O rows");
static_assert(kDQK == kDV, "raw Q and O rows share the staging layout");
constexpr int kDraftBlocksPerTile = kBN / 8;  // 8 key slots per block
// Draft tiles are block-major: block bb's 8 K^C rows (3 x 1 KB swizzled
// slices) at bb * 3 KB, its K^R rows at 24 KB + bb * 1 KB; its V rows (4 x 1 KB)
// at bb * 4 KB. As MMA operands: K^C with 8-row groups 3 KB apart, V with
// 64-column slices 1 KB apart and 8-key groups 4 KB apart.
constexpr int kDraftKcBlock = 3 * 1024, kDraftKr = 3 * kKChunk, kDraftVBlock = 4 * 1024;
constexpr int kSmemBytes = oBar + 512 + 1024;  // barriers + alignment slack
// barrier words: K and V full/empty per stage, 28 more, 6 counters, one more
// barrier, the item ring's 2 x kRing barriers and its kRing slots
constexpr int kRing = 4;
static_assert((2 * (kKS + kVS) + 32 + 2 * kRing + kRing / 2) * 8 <= 512, "barrier area too small");
static_assert(kSmemBytes <= 232448, "dynamic shared memory above the sm_100 per-block limit");

constexpr int kSoftWarps = 8;
constexpr int kWarpK = 8, kWarpMma = 9, kWarpV = 10, kWarpQ = 11;
// roles that read the item ring: K and V producers, the MMA issuer, the softmax warps
constexpr int kItemReaders = 3 + kSoftWarps;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;
constexpr uint32_t kColS = 256;  // two S buffers: 256..319, 320..383 (P over the first 16 columns of each half)
constexpr uint32_t kColQ = 384;  // Q: 256 bf16 per row as 128 columns
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLn2 = 0.6931471805599453f;

struct FwdArgs {
    int n_h, S, N, W, L, R;
    float scale_log2;
    const __nv_bfloat16 *q, *kc, *krr, *v;
    const int32_t *cnt, *sorted_n, *sorted_a;
    const float2 *tab;
    __nv_bfloat16 *o;
    float *lse;
    uint32_t *err;
    int B;
    int n_groups;  // groups of kG blocks per batch row (work items per (b, h))
    int n_items;   // n_groups * n_h * B
    int n_work;    // counter values that name an item: n_items + n_h * B
    int *sched;    // work-item counter, 0 at launch
    uint64_t wait_ns;  // limit of the pipeline waits (ns)
};

// A bf16 pair (x0 low, x1 high) of a rope slice rotated by (c, s).
__device__ __forceinline__ uint32_t rope_rot(uint32_t w, float c, float s) {
    const float x0 = __uint_as_float(w << 16), x1 = __uint_as_float(w & 0xffff0000u);
    return pack_bf16x2(x0 * c - x1 * s, x0 * s + x1 * c);
}
// 1-D bulk copy shared -> global (16-byte aligned addresses, size a multiple
// of 16), tracked by this thread's bulk async-group.
__device__ __forceinline__ void bulk_store(void *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// this thread's bulk stores have read their shared-memory source
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// this thread's bulk stores are complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Work items in the order the CTAs take them from the counter: first every
// full group of kG blocks, w = (group g, head h, batch b) with g fastest
// (neighbouring groups of one head read overlapping context windows, close
// together in time, so the overlap is served by L2); then, from w = n_items
// on, the last, partial group of each (b, h) whose kept count is not a
// multiple of kG. Small items at the end even out the CTAs' finishing times.
struct Item {
    int b, gcnt, nrows, ctx_lo, n_ctx, T;
    size_t bh;
    const int32_t *sa, *sn;
};
__device__ __forceinline__ bool item_at(const FwdArgs &p, int w, Item &it) {
    int g, h, b, cnt;
    if (w < p.n_items) {
        g = w % p.n_groups;
        h = (w / p.n_groups) % p.n_h;
        b = w / (p.n_groups * p.n_h);
        cnt = p.cnt[b];
        if (g * kG + kG > cnt) return false;  // past the row's blocks, or its partial group
    } else {
        const int r = w - p.n_items;
        h = r % p.n_h;
        b = r / p.n_h;
        cnt = p.cnt[b];
        if (cnt % kG == 0) return false;  // no partial group
        g = cnt / kG;
    }
    const int i0 = g * kG;
    it.b = b;
    it.gcnt = min(kG, cnt - i0);
    it.nrows = kBlock * it.gcnt;
    it.sa = p.sorted_a + (size_t)b * p.N + i0;
    it.sn = p.sorted_n + (size_t)b * p.N + i0;
    it.ctx_lo = max(0, it.sa[0] - p.W + 1);
    const int ctx_hi = it.sa[it.gcnt - 1];
    it.n_ctx = ctx_hi > it.ctx_lo ? (ctx_hi - it.ctx_lo + kBN - 1) / kBN : 0;
    it.T = it.n_ctx + (it.gcnt + kDraftBlocksPerTile - 1) / kDraftBlocksPerTile;
    it.bh = (size_t)b * p.n_h + h;
    return true;
}

// Persistent: one CTA per SM. The loader warp takes the CTA's next work item
// from a global counter (so every CTA stays busy until the items run out) and
// publishes it in a ring of kRing slots in shared memory, from which the other
// roles read the same sequence. Tiles, S buffers and pipeline phases are
// counted over all of the CTA's items, so K/V loads run on across item
// boundaries.
__global__ void __launch_bounds__(kThreads, 1)
    k_fwd_tc(const __grid_constant__ CUtensorMap tm_kc3, const __grid_constant__ CUtensorMap tm_kr,
             const __grid_constant__ CUtensorMap tm_v3, const __grid_constant__ CUtensorMap tm_kc38,
             const __grid_constant__ CUtensorMap tm_kr8, const __grid_constant__ CUtensorMap tm_v38, const FwdArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + oBar);
    uint64_t *kfull = bars, *kempty = kfull + kKS, *vfull = kempty + kKS, *vempty = vfull + kVS;
    uint64_t *sfull = vempty + kVS, *pready = sfull + 2, *pvdone = sfull + 4;
    // per item: raw Q landed, Q in TMEM, raw Q read (all softmax warps), O
    // read out of TMEM, staging area free again
    uint64_t *qraw = sfull + 6, *qready = sfull + 7, *qdone = sfull + 8, *ofree = sfull + 9, *stgfree = sfull + 10;
    // per item: O rows staged (softmax warps), O rows read out (loader warp)
    uint64_t *drain = sfull + 11, *ostaged = sfull + 26, *oread = sfull + 27;
    // softmax pair exchange: per TMEM sub-partition and S buffer the tile max,
    // per sub-partition the row sum (two arrivals each: one per warp)
    uint64_t *xbar = sfull + 12, *lbar = sfull + 20;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sfull + 24);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sfull + 25);
    const uint64_t wlim = p.wait_ns;
    // [0] K tiles issued, [1] V tiles issued, [2] K tiles consumed by an MMA, [3] V tiles consumed,
    // [4] raw Q loads issued, [5] raw Q loads consumed
    int *counters = reinterpret_cast<int *>(sfull + 28);
    // per item: the staged raw Q rows' rope slice rotated (loader warp)
    uint64_t *qrot = sfull + 31;
    // item ring: slot published (loader warp), slot read by every reader role
    uint64_t *ifull = sfull + 32, *ifree = ifull + kRing;
    volatile int *ring = reinterpret_cast<volatile int *>(ifree + kRing);
    float *xm = reinterpret_cast<float *>(sm + oX);         // [s][half][row]
    float *xl = reinterpret_cast<float *>(sm + oX + 2048);  // [half][row]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // K/V stages start zeroed: masked key slots of a tile are multiplied by a
    // zero weight, and must not hold stale non-finite bits.
    for (int e = threadIdx.x; e < oStage / 16; e += blockDim.x)
        reinterpret_cast<uint4 *>(sm)[e] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kKS; s++) {
            mbar_init(&kfull[s], 1);
            mbar_init(&kempty[s], 1);
        }
        for (int s = 0; s < kVS; s++) {
            mbar_init(&vfull[s], 1);
            mbar_init(&vempty[s], 1);
        }
        for (int s = 0; s < 2; s++) {
            mbar_init(&sfull[s], 1);
            mbar_init(&pready[s], kSoftWarps);
            mbar_init(&pvdone[s], 1);
        }
        mbar_init(qraw, 1);
        mbar_init(qrot, 1);
        mbar_init(qready, kSoftWarps);
        mbar_init(qdone, kSoftWarps);
        mbar_init(ofree, kSoftWarps);
        mbar_init(stgfree, kSoftWarps);
        mbar_init(ostaged, kSoftWarps);
        mbar_init(oread, 1);
        mbar_init(drain, 1);
        for (int s = 0; s < kRing; s++) {
            mbar_init(&ifull[s], 1);
            mbar_init(&ifree[s], kItemReaders);
        }
        for (int i = 0; i < 8; i++) mbar_init(&xbar[i], 2);
        for (int i = 0; i < 4; i++) mbar_init(&lbar[i], 2);
        *abort_flag = 0;
        for (int c = 0; c < 6; c++) counters[c] = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    fence_proxy_async_smem();  // the zeroed stages are read by TMA-fed MMAs
    tc_fence_before();
    pdl_wait();  // the kernels before this one (rotated rope keys, item counter) have completed
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Item k of the CTA's sequence from ring slot k % kRing: 1 = an item, 0 =
    // past the last one, -1 = the wait gave up. take_w is called by a whole
    // warp, take_1 by one thread; release: this reader is done with the slot.
    auto take_w = [&](int k, Item &it) -> int {
        const int s = k % kRing;
        if (!warp_all(mbar_wait(&ifull[s], (k / kRing) & 1, abort_flag, wlim))) return -1;
        const int w = ring[s];
        __syncwarp();
        if (lane == 0) mbar_arrive(&ifree[s]);
        return w >= 0 && item_at(p, w, it) ? 1 : 0;
    };
    auto take_1 = [&](int k, Item &it, bool release) -> int {
        const int s = k % kRing;
        if (!mbar_wait(&ifull[s], (k / kRing) & 1, abort_flag, wlim)) return -1;
        const int w = ring[s];
        if (release) mbar_arrive(&ifree[s]);
        return w >= 0 && item_at(p, w, it) ? 1 : 0;
    };

    if (warp == kWarpK || warp == kWarpV) {
        // ------------------------------------------------------ producers
        const bool isk = warp == kWarpK;
        if (isk && lane == 0) {
            tma_prefetch_desc(&tm_kc3);
            tma_prefetch_desc(&tm_kr);
            tma_prefetch_desc(&tm_v3);
        }
        int tt = 0;  // tiles over all items
        bool ok = true;
        Item it;
        for (int k = 0; ok; ++k) {
            const int f = take_w(k, it);
            if (f < 0) ok = false;
            if (f <= 0) break;
            // lane l holds the block index of group block l
            const int my_n = lane < it.gcnt ? it.sn[lane] : 0;
            for (int t = 0; t < it.T; ++t, ++tt) {
                const int nst = isk ? kKS : kVS;
                const int s = tt % nst;
                if (tt >= nst && !warp_all(mbar_wait(isk ? &kempty[s] : &vempty[s], ((tt / nst) - 1) & 1, abort_flag, wlim))) {
                    ok = false;
                    break;
                }
                uint64_t *full = isk ? &kfull[s] : &vfull[s];
                uint8_t *dst = sm + (isk ? k_stage_off(s) : v_stage_off(s));
                if (t < it.n_ctx) {
                    const int pos0 = it.ctx_lo + t * kBN;
                    if (lane == 0) {
                        if (isk) {
                            mbar_arrive_expect_tx(full, kKBytes);
                            tma_load_3d(dst, &tm_kc3, full, 0, (int)(it.bh * p.L + pos0), 0);
                            tma_load_2d(dst + 3 * kKChunk, &tm_kr, full, 0, (int)((size_t)it.b * p.L + pos0));
                        } else {
                            mbar_arrive_expect_tx(full, kVBytes);
                            tma_load_3d(dst, &tm_v3, full, 0, (int)(it.bh * p.L + pos0), 0);
                        }
                    }
                } else {
                    // draft tile: 8 key slots per block, its 5 keys first (the 3
                    // rows after them are other keys, masked out)
                    const int d = t - it.n_ctx;
                    const int nb = min(kDraftBlocksPerTile, it.gcnt - d * kDraftBlocksPerTile);
                    if (lane == 0) mbar_arrive_expect_tx(full, nb * 8 * (isk ? kDQK : kDV) * 2);
                    __syncwarp();
                    for (int bb = 0; bb < nb; ++bb) {
                        const int n = __shfl_sync(0xffffffffu, my_n, d * kDraftBlocksPerTile + bb);
                        if (lane == 0) {
                            const int row = p.S + kBlock * n;
                            if (isk) {
                                tma_load_3d(dst + bb * kDraftKcBlock, &tm_kc38, full, 0, (int)(it.bh * p.L + row), 0);
                                tma_load_2d(dst + kDraftKr + bb * 1024, &tm_kr8, full, 0,
                                            (int)((size_t)it.b * p.L + row));
                            } else {
                                tma_load_3d(dst + bb * kDraftVBlock, &tm_v38, full, 0, (int)(it.bh * p.L + row), 0);
                            }
                        }
                    }
                }
                if (lane == 0) counters[isk ? 0 : 1] = tt + 1;
            }
        }
    } else if (warp == kWarpQ) {
        // ------------------------------------ raw Q loader and O writer
        // The staging area holds item ic's raw Q rows until they are in TMEM,
        // then item ic - 1's O rows (staged by the softmax warps), which this
        // warp stores before loading item ic + 1's raw Q rows.
        auto load_q = [&](const Item &q_it, int ic) {
            const int my_n = lane < q_it.gcnt ? q_it.sn[lane] : 0;
            fence_proxy_async_smem();  // this warp's reads of the staging area precede the copy
            __syncwarp();
            if (lane == 0) {
                // each block's 5 rows are one contiguous 2560-byte run
                mbar_arrive_expect_tx(qraw, q_it.nrows * kDQK * 2);
                counters[4] = ic + 1;
            }
            __syncwarp();
            if (lane < q_it.gcnt)
                bulk_load(sm + oStage + lane * kStageBlockPitch, p.q + (q_it.bh * p.R + (size_t)kBlock * my_n) * kDQK,
                          kBlock * kDQK * 2, qraw);
        };
        // Once they have landed, the rope slice (the last 64 columns) of every
        // staged row is rotated in place to the row's position A + j: lane i
        // turns frequency i (one bf16 pair) of each row, 25 rows per round of
        // table loads. This runs while the item before is still in flight, so
        // the softmax warps only copy the rows into TMEM at the item switch.
        auto rotate_q = [&](const Item &q_it, int ic) -> bool {
            if (!warp_all(mbar_wait(qraw, ic & 1, abort_flag, wlim))) return false;
            if (lane == 0) counters[5] = ic + 1;
            const int my_a = lane < q_it.gcnt ? q_it.sa[lane] : 0;
            for (int b0 = 0; b0 < q_it.gcnt; b0 += 5) {
                float2 cs[5][kBlock];
#pragma unroll
                for (int bb = 0; bb < 5; bb++) {
                    const int a = __shfl_sync(0xffffffffu, my_a, b0 + bb);  // b0 + bb <= 28
#pragma unroll
                    for (int j = 0; j < kBlock; j++)
                        cs[bb][j] = b0 + bb < q_it.gcnt ? __ldg(p.tab + (size_t)(a + j) * (kDR / 2) + lane)
                                                        : make_float2(1.f, 0.f);
                }
#pragma unroll
                for (int bb = 0; bb < 5; bb++) {
                    if (b0 + bb < q_it.gcnt) {
                        uint32_t *row = reinterpret_cast<uint32_t *>(sm + oStage + (b0 + bb) * kStageBlockPitch + kDC * 2);
#pragma unroll
                        for (int j = 0; j < kBlock; j++) {
                            uint32_t *wp = row + j * (kDQK / 2) + lane;
                            *wp = rope_rot(*wp, cs[bb][j].x, cs[bb][j].y);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(qrot);
            return true;
        };
        // Item k of the CTA's sequence: the next valid item from the global
        // counter, published in ring slot k % kRing once every reader is done
        // with the item kRing before it (1 = an item, 0 = none left, published
        // as -1, -1 = a wait gave up). Called by the whole warp.
        auto fetch = [&](int k, Item &it) -> int {
            const int s = k % kRing;
            if (k >= kRing && !warp_all(mbar_wait(&ifree[s], ((k / kRing) - 1) & 1, abort_flag, wlim))) return -1;
            int w = -1;
            if (lane == 0) {
                Item probe;
                for (;;) {
                    const int x = atomicAdd(p.sched, 1);
                    if (x >= p.n_work) break;
                    if (item_at(p, x, probe)) {
                        w = x;
                        break;
                    }
                }
                ring[s] = w;
                mbar_arrive(&ifull[s]);
            }
            w = __shfl_sync(0xffffffffu, w, 0);
            return w >= 0 && item_at(p, w, it) ? 1 : 0;
        };
        Item it, nx;
        int ic = 0;
        int f = fetch(0, it);
        bool ok = f >= 0, has = f > 0, hasn = false;
        if (has) {
            load_q(it, 0);
            ok = rotate_q(it, 0);
        }
        if (ok && has) {
            f = fetch(1, nx);
            ok = f >= 0;
            hasn = f > 0;
        }
        if (ok && hasn) {  // item 1's raw Q once item 0's is in TMEM
            ok = warp_all(mbar_wait(stgfree, 0, abort_flag, wlim));
            if (ok) {
                load_q(nx, 1);
                ok = rotate_q(nx, 1);
            }
        }
        while (ok && has) {
            // item ic's O rows: each block's 5 rows (contiguous in global
            // memory) with one bulk copy; the staging area is free again once
            // the copies have read it
            ok = warp_all(mbar_wait(ostaged, ic & 1, abort_flag, wlim));
            if (!ok) break;
            if (lane < it.gcnt)
                bulk_store(p.o + (it.bh * p.R + (size_t)kBlock * it.sn[lane]) * kDV, sm + oStage + lane * kStageBlockPitch,
                           kBlock * kDV * 2);
            bulk_commit();
            bulk_wait_read_all();
            __syncwarp();
            if (lane == 0) mbar_arrive(oread);
            // the item after next: its raw Q into the staging area
            Item n2;
            bool has2 = false;
            if (hasn) {
                f = fetch(ic + 2, n2);
                if (f < 0) {
                    ok = false;
                    break;
                }
                has2 = f > 0;
            }
            if (has2) {
                load_q(n2, ic + 2);
                ok = rotate_q(n2, ic + 2);
            }
            ++ic;
            it = nx;
            has = hasn;
            nx = n2;
            hasn = has2;
        }
        bulk_wait_all();  // the O stores are complete before the CTA ends
    } else if (warp == kWarpMma) {
        // ----------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idS = idesc_bf16(kM, kBN, 0);
            const uint32_t idO = idesc_bf16(kM, kDV, 1);
            auto issue_qk = [&](int tg, int t, int n_ctx) {
                const int s = tg & 1;
                const uint32_t kb = smem_u32(sm + k_stage_off(tg % kKS));
                const uint32_t dS = tmem + kColS + s * kBN;
                if (t < n_ctx) {
                    const SDesc kd = sdesc_split(sdesc_sw128(kb, 16, 1024));
#pragma unroll
                    for (int k = 0; k < kDQK / 16; ++k) {
                        const uint32_t ko = ((k >> 2) * kKChunk + (k & 3) * 32) >> 4;
                        mma_bf16_ts(dS, tmem + kColQ + 8 * k, kd.at(ko), idS, k > 0 ? 1u : 0u);
                    }
                } else {
                    const SDesc kdc = sdesc_split(sdesc_sw128(kb, 16, kDraftKcBlock));
                    const SDesc kdr = sdesc_split(sdesc_sw128(kb + kDraftKr, 16, 1024));
#pragma unroll
                    for (int k = 0; k < kDC / 16; ++k) {
                        const uint32_t ko = ((k >> 2) * 1024 + (k & 3) * 32) >> 4;
                        mma_bf16_ts(dS, tmem + kColQ + 8 * k, kdc.at(ko), idS, k > 0 ? 1u : 0u);
                    }
#pragma unroll
                    for (int k = kDC / 16; k < kDQK / 16; ++k)
                        mma_bf16_ts(dS, tmem + kColQ + 8 * k, kdr.at(((k & 3) * 32) >> 4), idS, 1u);
                }
                mma_commit(&sfull[s]);
                mma_commit(&kempty[tg % kKS]);
                counters[2] = tg + 1;
            };
            auto issue_pv = [&](int tg, int t, int n_ctx) {
                const int s = tg & 1;
                const uint32_t vb = smem_u32(sm + v_stage_off(tg % kVS));
                const bool ctx = t < n_ctx;
                // context tile: 64-column slices 8 KB apart, keys 128 B apart;
                // draft tile: slices 1 KB apart, 8-key groups 4 KB apart
                const SDesc vd = sdesc_split(ctx ? sdesc_sw128(vb, kKChunk, 1024) : sdesc_sw128(vb, 1024, kDraftVBlock));
                const uint32_t kstep = ctx ? 128u : 512u;  // 16 keys, in 16-byte units
                // P of keys 16 k .. 16 k + 15: half k / 2 of the S buffer, its
                // columns 8 (k % 2) ..; the item's first tile overwrites O
                const uint32_t pa = tmem + kColS + s * kBN;
                mma_bf16_ts(tmem + kColO, pa, vd.at(0), idO, t > 0 ? 1u : 0u);
                mma_bf16_ts(tmem + kColO, pa + 8, vd.at(kstep), idO, 1u);
                mma_bf16_ts(tmem + kColO, pa + 32, vd.at(2 * kstep), idO, 1u);
                mma_bf16_ts(tmem + kColO, pa + 40, vd.at(3 * kstep), idO, 1u);
                mma_commit(&vempty[tg % kVS]);
                mma_commit(&pvdone[s]);
            };
            // Two cursors over the CTA's items: QK of tile nk (item icK, local
            // tile tK) and P V of tile np (item icP, local tile tP). Issue
            // whichever is ready: QK when its K landed, the P V that reads the
            // P written over its S buffer (tile nk - 2) is issued and, at an
            // item's first tile, the item's Q is in TMEM; P V when its P is in
            // TMEM and its V landed and, at an item's first tile, the previous
            // item's O has been read out.
            // (the QK cursor reads each item first; the P V cursor releases it)
            Item ik, ip;
            int f = take_1(0, ik, false);
            bool ok = f >= 0, hk = f > 0, hp = false;
            if (ok) {
                f = take_1(0, ip, true);
                ok = f >= 0;
                hp = f > 0;
            }
            int nk = 0, np = 0, icK = 0, icP = 0, tK = 0, tP = 0;
            uint64_t t_idle = 0;
            while (ok && hp) {
                bool issued = false;
                if (hk && np >= nk - 1 && mbar_test(&kfull[nk % kKS], (nk / kKS) & 1) &&
                    (tK != 0 || mbar_test(qready, icK & 1))) {
                    tc_fence_after();
                    issue_qk(nk, tK, ik.n_ctx);
                    ++nk;
                    if (++tK == ik.T) {
                        tK = 0;
                        ++icK;
                        const int g = take_1(icK, ik, false);
                        if (g < 0) ok = false;
                        hk = g > 0;
                    }
                    issued = true;
                }
                if (!issued && np < nk && mbar_test(&pready[np & 1], (np >> 1) & 1) &&
                    mbar_test(&vfull[np % kVS], (np / kVS) & 1) && (tP != 0 || icP == 0 || mbar_test(ofree, (icP - 1) & 1))) {
                    counters[3] = np + 1;
                    tc_fence_after();
                    issue_pv(np, tP, ip.n_ctx);
                    ++np;
                    if (++tP == ip.T) {
                        tP = 0;
                        ++icP;
                        const int g = take_1(icP, ip, true);
                        if (g < 0) ok = false;
                        hp = g > 0;
                    }
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
    } else if (warp < kSoftWarps) {
        // ------------------------------------------------ softmax (rows)
        const int q4 = warp & 3, hf = warp >> 2;  // TMEM sub-partition, column half
        const int r = q4 * 32 + lane;               // query row = TMEM lane
        const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
        bool ok = true;
        // Q row r of an item, this thread's half (columns 128 hf .. + 127),
        // from the staging area (rope slice already rotated by the loader
        // warp) -> TMEM lane r, columns kColQ + 64 hf .. + 63. Rows past the
        // item's blocks are zero.
        auto move_q = [&](const Item &q_it, int ic) {
            const bool live = r < q_it.nrows;
            ok = warp_all(mbar_wait(qrot, ic & 1, abort_flag, wlim));
            const bool have = live && ok;
            const uint4 *src = reinterpret_cast<const uint4 *>(sm + oStage + (r / kBlock) * kStageBlockPitch +
                                                               (r % kBlock) * (kDQK * 2) + hf * 256);
#pragma unroll
            for (int part = 0; part < 2; part++) {  // 8 units (64 bf16) per TMEM store
                uint32_t w[32];
#pragma unroll
                for (int uu = 0; uu < 8; uu++) {
                    const uint4 val = have ? src[part * 8 + uu] : make_uint4(0, 0, 0, 0);
                    w[4 * uu + 0] = val.x;
                    w[4 * uu + 1] = val.y;
                    w[4 * uu + 2] = val.z;
                    w[4 * uu + 3] = val.w;
                }
                tmem_st32u(trow + kColQ + 64 * hf + 32 * part, w);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(qready);
        };

        int tg = 0;  // tiles over all items
        int ic = 0;
        Item it, nx;
        const int f0 = take_w(0, it);
        ok = f0 >= 0;
        bool has = f0 > 0;
        if (has) {
            move_q(it, 0);
            __syncwarp();
            if (lane == 0) mbar_arrive(stgfree);  // item 1's raw Q may load
        }
        while (ok && has) {
            const bool live = r < it.nrows;
            int A = 0, n = 0, j = 0, lo = 0;
            if (live) {
                A = it.sa[r / kBlock];
                n = it.sn[r / kBlock];
                j = r % kBlock;
                lo = max(0, A - p.W + 1);
            }
            float m_used = -INFINITY, l = 0.f;  // l: this half's share of the row sum
            for (int t = 0; t < it.T && ok; ++t, ++tg) {
                const int s = tg & 1;
                ok = warp_all(mbar_wait(&sfull[s], (tg >> 1) & 1, abort_flag, wlim));
                if (!ok) break;
                tc_fence_after();
                // every row's keys in a tile form one contiguous column range
                // [clo, chi): the window [lo, A) for context tiles, its block's 5
                // key slots for draft tiles; this warp holds columns 32 hf .. +31
                int clo, chi;
                if (t < it.n_ctx) {
                    const int c0 = it.ctx_lo + t * kBN;
                    clo = lo - c0;
                    chi = A - c0;
                } else {
                    clo = 8 * (r / kBlock) - (t - it.n_ctx) * kBN;
                    chi = clo + kBlock;
                }
                if (!live) chi = clo;
                clo -= 32 * hf;
                chi -= 32 * hf;
                // Rows are anchor-sorted, so for most (warp, half tile) pairs no
                // row of the warp sees any of the 32 keys: such a half tile only
                // contributes P = 0 (uniform over the warp, no S read).
                const bool act = __any_sync(0xffffffffu, clo < chi && clo < 32 && chi > 0);
                float sv[32];
                float mx[4];
#pragma unroll
                for (int k = 0; k < 4; k++) mx[k] = -INFINITY;
                if (act) {
                    tmem_ld32(trow + kColS + s * kBN + 32 * hf, sv);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; c++) {
                        sv[c] = (c >= clo && c < chi) ? sv[c] : -INFINITY;
                        mx[c & 3] = fmaxf(mx[c & 3], sv[c]);
                    }
                }
                // the pair's tile max, exchanged through shared memory
                const float mhalf = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                xm[(s * 2 + hf) * kM + r] = mhalf;
                __syncwarp();
                if (lane == 0) mbar_arrive(&xbar[2 * q4 + s]);
                ok = warp_all(mbar_wait(&xbar[2 * q4 + s], (tg >> 1) & 1, abort_flag, wlim));
                if (!ok) break;
                const float mother = xm[(s * 2 + (hf ^ 1)) * kM + r];
                const float mt = fmaxf(mhalf, mother) * p.scale_log2;
                bool resc = false;
                float alpha = 1.f;
                if (mt > m_used + kRescaleThreshold) {
                    if (m_used != -INFINITY) {
                        resc = true;
                        alpha = ex2(m_used - mt);
                    }
                    m_used = mt;
                }
                float psum[4];
#pragma unroll
                for (int k = 0; k < 4; k++) psum[k] = 0.f;
                const bool any = m_used != -INFINITY;
                const float mneg = any ? -m_used : 0.f;
                uint32_t pw[16];  // this half's 32 P values as bf16 pairs
                if (act) {
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        const float e0 = any ? ex2(fmaf(sv[c], p.scale_log2, mneg)) : 0.f;
                        const float e1 = any ? ex2(fmaf(sv[c + 1], p.scale_log2, mneg)) : 0.f;
                        psum[c & 3] += e0;
                        psum[(c + 1) & 3] += e1;
                        pw[c / 2] = pack_bf16x2(e0, e1);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 16; c++) pw[c] = 0u;
                }
                // P over this half's first 16 S columns (the S values are in registers)
                tmem_st16u(trow + kColS + s * kBN + 32 * hf, pw);
                l = l * alpha + ((psum[0] + psum[1]) + (psum[2] + psum[3]));
                if (__any_sync(0xffffffffu, resc)) {
                    // (never at an item's first tile: m_used starts at -inf)
                    ok = warp_all(mbar_wait(&pvdone[(tg - 1) & 1], ((tg - 1) >> 1) & 1, abort_flag, wlim));
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 128 * hf; c < 128 * hf + 128; c += 32) {  // this half's O columns
                        float ov[32];
                        tmem_ld32(trow + kColO + c, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; i++) ov[i] *= alpha;
                        tmem_st32(trow + kColO + c, ov);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&pready[s]);
            }
            if (!ok) break;
            // The next item's Q into TMEM (its raw rows are staged; every QK of
            // this item has completed, as all its S tiles have been read), so
            // that its QK can start while this item's O is written out.
            const int fn = take_w(ic + 1, nx);
            if (fn < 0) {
                ok = false;
                break;
            }
            const bool hasn = fn > 0;
            if (hasn) {
                move_q(nx, ic + 1);
                if (!ok) break;
                if (lane == 0) mbar_arrive(qdone);
            }
            ok = warp_all(mbar_wait(&pvdone[(tg - 1) & 1], ((tg - 1) >> 1) & 1, abort_flag, wlim));
            if (ok) {
                // the row sum: both halves' shares, exchanged like the tile max
                xl[hf * kM + r] = l;
                __syncwarp();
                if (lane == 0) mbar_arrive(&lbar[q4]);
                ok = warp_all(mbar_wait(&lbar[q4], ic & 1, abort_flag, wlim));
            }
            // the staging area: every warp has read the next item's raw Q rows,
            // and the loader warp's bulk copies have read the previous item's O rows
            if (ok && hasn) ok = warp_all(mbar_wait(qdone, ic & 1, abort_flag, wlim));
            if (ok && ic >= 1) ok = warp_all(mbar_wait(oread, (ic - 1) & 1, abort_flag, wlim));
            if (!ok) break;
            tc_fence_after();
            const float ltot = l + xl[(hf ^ 1) * kM + r];
            const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
            // this half of the O row (columns 128 hf .. +127) -> the staging
            // area in the raw Q layout (block r / 5 at r / 5 * 2576, row r % 5
            // at + 512 (r % 5)); rows past the item's blocks are not staged
            uint8_t *orow = sm + oStage + (live ? (r / kBlock) * kStageBlockPitch + (r % kBlock) * (kDV * 2) : 0) + hf * 256;
#pragma unroll 1
            for (int c = 0; c < 128; c += 32) {
                float ov[32];
                tmem_ld32(trow + kColO + 128 * hf + c, ov);
                tmem_wait_ld();
                if (live) {
#pragma unroll
                    for (int k = 0; k < 4; k++)
                        *reinterpret_cast<uint4 *>(orow + (c / 8 + k) * 16) =
                            make_uint4(pack_bf16x2(ov[8 * k + 0] * inv, ov[8 * k + 1] * inv),
                                       pack_bf16x2(ov[8 * k + 2] * inv, ov[8 * k + 3] * inv),
                                       pack_bf16x2(ov[8 * k + 4] * inv, ov[8 * k + 5] * inv),
                                       pack_bf16x2(ov[8 * k + 6] * inv, ov[8 * k + 7] * inv));
                }
            }
            // O is out of TMEM: the next item's first P V may overwrite it; the
            // loader warp stores the staged rows with bulk copies (async proxy)
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(ofree);
                mbar_arrive(ostaged);
            }
            if (live && hf == 0) p.lse[it.bh * p.R + kBlock * n + j] = (m_used + log2f(ltot)) * kLn2;
            ++ic;
            it = nx;
            has = hasn;
        }
    }

    // ---------------------------------------------------------- teardown
    pdl_trigger();
    __syncthreads();
    if (*abort_flag) {
        // Drain what may still be in flight, each wait bounded on its own.
        volatile int never = 0;
        if (warp == kWarpK && lane == 0) {
            // loads issued but not yet consumed complete in order, one phase each
            for (int t = counters[2]; t < counters[0]; ++t)
                mbar_wait(&kfull[t % kKS], (t / kKS) & 1, (volatile int *)&never);
            for (int t = counters[3]; t < counters[1]; ++t)
                mbar_wait(&vfull[t % kVS], (t / kVS) & 1, (volatile int *)&never);
            for (int t = counters[5]; t < counters[4]; ++t) mbar_wait(qraw, t & 1, (volatile int *)&never);
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
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0 && *abort_flag) atomicOr(p.err, kErrTimeout);
}

}  // namespace

bool fwd_tc_supported(const Prob &p) {
    // TMA row coordinates are 32-bit: every (batch, head, position) row must fit
    return p.dtype == DSPARK_BF16 && p.d_c == kDC && p.d_r == kDR && p.d_v == kDV &&
           (long long)p.B * p.n_h * p.L < (1ll << 31);
}

cudaError_t launch_fwd_tc(const Prob &p, const void *q, const void *kc, const void *v, const int32_t *anchors,
                          const uint8_t *keep, void *o, float *lse, const Ws &ws, cudaStream_t st) {
    // (padding blocks' rows are written by the rope-key rotation launch before this one)
    if (p.B == 0 || p.N == 0) return cudaSuccess;
    CUtensorMap m_kc3, m_kr, m_v3, m_kc38, m_kr8, m_v38;
    const uint64_t kv_rows = (uint64_t)p.B * p.n_h * p.L, kr_rows = (uint64_t)p.B * p.L;
    if (!make_map3_bf16(&m_kc3, kc, kDC, kv_rows, 64) || !make_map_bf16(&m_kr, ws.kr_rot, kDR, kr_rows, 64) ||
        !make_map3_bf16(&m_v3, v, kDV, kv_rows, 64) || !make_map3_bf16(&m_kc38, kc, kDC, kv_rows, 8) ||
        !make_map_bf16(&m_kr8, ws.kr_rot, kDR, kr_rows, 8) || !make_map3_bf16(&m_v38, v, kDV, kv_rows, 8))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(k_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    FwdArgs a;
    a.n_h = p.n_h; a.S = p.S; a.N = p.N; a.W = p.W; a.L = p.L; a.R = p.R;
    a.scale_log2 = p.scale_log2;
    a.q = (const __nv_bfloat16 *)q;
    a.kc = (const __nv_bfloat16 *)kc;
    a.krr = (const __nv_bfloat16 *)ws.kr_rot;
    a.v = (const __nv_bfloat16 *)v;
    a.cnt = ws.cnt;
    a.sorted_n = ws.sorted_n;
    a.sorted_a = ws.sorted_a;
    a.tab = ws.rope;
    a.o = (__nv_bfloat16 *)o;
    a.lse = lse;
    a.err = ws.err;
    a.wait_ns = p.wait_ns;
    a.B = p.B;
    a.sched = ws.sched;
    a.n_groups = (p.N + kG - 1) / kG;
    a.n_items = a.n_groups * p.n_h * p.B;
    a.n_work = a.n_items + p.n_h * p.B;
    int dev = 0, nsm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    count_launch();
    return launch_pdl(k_fwd_tc, dim3(std::min(a.n_items, nsm)), dim3(kThreads), kSmemBytes, st, m_kc3, m_kr, m_v3,
                      m_kc38, m_kr8, m_v38, a);
}

}  // namespace dspark
