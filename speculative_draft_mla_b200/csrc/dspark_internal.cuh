// Internal declarations shared by the translation units of the DSpark
// attention library: problem view, workspace layout, error bits and the
// launch functions of each kernel family.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dspark_attn.h"

namespace dspark {

constexpr int kBlock = 5;  // draft block length (block_size = 5)

// Device error word bits (workspace offset 0).
constexpr uint32_t kErrAnchor = 1u;   // kept anchor outside [0, S-2]
constexpr uint32_t kErrTimeout = 2u;  // a bounded mbarrier wait gave up
// Default (and largest) time a bounded wait lasts before it gives up, in ns.
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;

struct Prob {
    int B, n_h, S, N, W, d_c, d_r, d_v;
    int dqk;   // d_c + d_r
    int R;     // 5N query rows per (b, h)
    int L;     // S + 5N kv positions
    int P;     // rope table positions (S + 8)
    double base;
    int dtype;
    float scale_log2;  // (d_c + d_r)^(-1/2) * log2(e)
    float scale;       // (d_c + d_r)^(-1/2)
    uint64_t wait_ns;  // limit of the kernels' pipeline waits (ns)
};

// Workspace layout (byte offsets, each 256-aligned).
struct WsLayout {
    size_t err;       // uint32 error word; at +128 the tensor-core forward's int32 work-item counter
    size_t cnt;       // int32 [B]     kept blocks per batch row
    size_t sorted_n;  // int32 [B, N]  block index of the i-th smallest anchor
    size_t sorted_a;  // int32 [B, N]  its anchor
    size_t rope;      // float2 [P, d_r/2] (cos, sin) of pos * base^(-2i/d_r)
    size_t kr_rot;    // dtype [B, L, d_r] rotated rope keys
    size_t fwd_total; // the forward needs only the sections above
    size_t dvec;      // float [B, n_h, 5N] D = rowsum(dO * O)
    // tensor-core backward only (empty otherwise)
    size_t lses;      // float [B, n_h, 5N] LSE * log2(e), anchor-sorted rows
    size_t qs;        // bf16 [B, n_h, 5N, 256] rotated Q, anchor-sorted rows
    size_t dos;       // bf16 [B, n_h, 5N, 256] dO, anchor-sorted rows
    size_t dkr_part;  // float [max(HG, HGd), B, L, d_r] rope-key gradient per head group
    size_t dqacc;     // float [B, n_h, 5N, d_c + d_r] dQ accumulator, anchor-sorted rows
    size_t total;
};

bool bwd_tc_supported(const Prob &p);
int bwd_head_groups(const Prob &p);  // head groups of the tensor-core backward (context keys)
int bwd_prep_groups(const Prob &p);  // head groups of its preparation (draft keys)
size_t fwd_workspace_size(const dspark_problem *p);

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(const Prob &p) {
    WsLayout w;
    size_t off = 0;
    size_t esz = p.dtype == DSPARK_BF16 ? 2 : 4;
    w.err = off;       off = align256(off + 256);
    w.cnt = off;       off = align256(off + sizeof(int32_t) * (size_t)p.B);
    w.sorted_n = off;  off = align256(off + sizeof(int32_t) * (size_t)p.B * p.N);
    w.sorted_a = off;  off = align256(off + sizeof(int32_t) * (size_t)p.B * p.N);
    w.rope = off;      off = align256(off + sizeof(float2) * (size_t)p.P * (p.d_r / 2));
    w.kr_rot = off;    off = align256(off + esz * (size_t)p.B * p.L * p.d_r);
    w.fwd_total = off;
    w.dvec = off;      off = align256(off + sizeof(float) * (size_t)p.B * p.n_h * p.R);
    const bool tc = bwd_tc_supported(p);
    const size_t rows = tc ? (size_t)p.B * p.n_h * p.R : 0;
    w.lses = off;      off = align256(off + sizeof(float) * rows);
    w.qs = off;        off = align256(off + 2 * rows * p.dqk);
    w.dos = off;       off = align256(off + 2 * rows * p.d_v);
    w.dkr_part = off;
    const int groups = tc ? (bwd_head_groups(p) > bwd_prep_groups(p) ? bwd_head_groups(p) : bwd_prep_groups(p)) : 0;
    off = align256(off + sizeof(float) * (size_t)groups * p.B * p.L * p.d_r);
    w.dqacc = off;     off = align256(off + sizeof(float) * rows * p.dqk);
    w.total = off;
    return w;
}

// Typed views of the workspace.
struct Ws {
    uint32_t *err;
    int32_t *sched;  // work-item counter of the tensor-core forward (in the error word's section)
    int32_t *cnt, *sorted_n, *sorted_a;
    float2 *rope;
    void *kr_rot;
    float *dvec;
    float *lses;
    void *qs, *dos;
    float *dkr_part;
    float *dqacc;
};

inline Ws ws_view(const Prob &p, void *base) {
    WsLayout l = ws_layout(p);
    char *c = (char *)base;
    Ws w;
    w.err = (uint32_t *)(c + l.err);
    w.sched = (int32_t *)(c + l.err + 128);
    w.cnt = (int32_t *)(c + l.cnt);
    w.sorted_n = (int32_t *)(c + l.sorted_n);
    w.sorted_a = (int32_t *)(c + l.sorted_a);
    w.rope = (float2 *)(c + l.rope);
    w.kr_rot = (void *)(c + l.kr_rot);
    w.dvec = (float *)(c + l.dvec);
    w.lses = (float *)(c + l.lses);
    w.qs = (void *)(c + l.qs);
    w.dos = (void *)(c + l.dos);
    w.dkr_part = (float *)(c + l.dkr_part);
    w.dqacc = (float *)(c + l.dqacc);
    return w;
}

// ---- element conversions -------------------------------------------------
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// ---- programmatic dependent launch ----------------------------------------
// The kernels of one call (and of consecutive calls) form a chain in the
// stream. Launched with programmatic stream serialization, a kernel may start
// (its CTAs be scheduled, its prologue touching only shared and tensor memory
// run) while the kernel before it finishes; pdl_wait() then blocks until that
// kernel has completed and its memory operations are visible, so every such
// kernel calls it before its first access to global memory. pdl_trigger()
// lets the next kernel start early (it is scheduled once every CTA of this
// one has triggered or exited); only the short single-wave kernels ahead of a
// kernel with a real prologue call it early (early dependents parked beside a
// long multi-wave kernel's last wave slowed it down), the others trigger by
// exiting. Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

// ---- launch accounting -----------------------------------------------------
// Every kernel launch goes through count_launch() so that the launch counter of
// the C ABI reports the device work a caller issued.
void count_launch(unsigned n = 1);

// ---- launch functions ------------------------------------------------------
// descriptor: sort kept blocks by anchor, validate anchors, rope table
cudaError_t launch_build_descriptor(const Prob &p, const int32_t *anchors, const uint8_t *keep, const Ws &ws,
                                    cudaStream_t st);
// Rows of padding blocks (keep = 0 or an invalid anchor, page §3: such a block
// sees nothing) that the rope-key rotation launch zeroes as well, so that the
// tensor-core paths need no launch of their own for them. Up to three bf16
// tensors laid out [B, n_h, rows, width]; block n owns rows first + 5 n ..
// first + 5 n + 4 of each. Unused entries have t = NULL.
struct PadRows {
    void *t[3];
    int rows[3];   // rows per (b, h)
    int first[3];  // row of block 0's first position (0 for query rows, S for draft keys)
    int width[3];  // elements per row, a multiple of 8
    float *lse;    // [B, n_h, 5N] fp32: -inf for the block's rows (NULL = none)
    int32_t *clear;  // a word set to 0 (the forward's work-item counter; NULL = none)
};

// rotated rope keys for all kv positions; with pad != NULL, also the padding
// blocks' rows described by *pad
cudaError_t launch_rotate_kr(const Prob &p, const void *kr, const int32_t *anchors, const uint8_t *keep,
                             const PadRows *pad, const Ws &ws, cudaStream_t st);

// SIMT (CUDA-core) forward / backward, any supported dims, fp32 or bf16
cudaError_t launch_fwd_simt(const Prob &p, const void *q, const void *kc, const void *v, const int32_t *anchors,
                            const uint8_t *keep, void *o, float *lse, const Ws &ws, cudaStream_t st);
cudaError_t launch_bwd_simt(const Prob &p, const void *q, const void *kc, const void *v, const int32_t *anchors,
                            const uint8_t *keep, const void *o, const float *lse, const void *dout, void *dq,
                            void *dkc, void *dkr, void *dv, const Ws &ws, cudaStream_t st);

// tcgen05 backward for bf16 at the page's head widths
cudaError_t launch_bwd_tc(const Prob &p, const void *q, const void *kc, const void *v, const int32_t *anchors,
                          const uint8_t *keep, const void *o, const float *lse, const void *dout, void *dq,
                          void *dkc, void *dkr, void *dv, const Ws &ws, cudaStream_t st);

// tcgen05 forward for bf16 at the page's head widths (192 + 64 / 256)
bool fwd_tc_supported(const Prob &p);
cudaError_t launch_fwd_tc(const Prob &p, const void *q, const void *kc, const void *v, const int32_t *anchors,
                          const uint8_t *keep, void *o, float *lse, const Ws &ws, cudaStream_t st);

}  // namespace dspark
