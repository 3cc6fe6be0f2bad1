// C ABI of the DSpark draft attention library: host-side argument checks,
// workspace layout, and the launch sequence of each entry point.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "dspark_steps.cuh"

using namespace dspark;

namespace dspark {
static std::atomic<uint64_t> g_launches{0};
static std::atomic<uint64_t> g_wait_ns{kWaitTimeoutNs};  // pipeline-wait limit of later launches
void count_launch(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
}  // namespace dspark

namespace {

bool make_prob(const dspark_problem *pp, Prob *out, dspark_status *why) {
    if (!pp) { *why = DSPARK_ERR_NULL; return false; }
    const dspark_problem &p = *pp;
    if (p.dtype != DSPARK_F32 && p.dtype != DSPARK_BF16) { *why = DSPARK_ERR_DTYPE; return false; }
    if (p.reserved != 0 || p.B < 0 || p.n_h < 1 || p.S < 1 || p.N < 0 || p.W < 1 || p.d_c < 0 || p.d_r < 0 ||
        p.d_v < 1 || (p.d_r & 1) || p.d_c + p.d_r < 1 || !(p.rope_base > 0.0) || !std::isfinite(p.rope_base)) {
        *why = DSPARK_ERR_SHAPE;
        return false;
    }
    if (p.W > 4096 || p.N > 8192 || p.d_c + p.d_r > 256 || p.d_v > 256) { *why = DSPARK_ERR_UNSUPPORTED; return false; }
    const long long L = (long long)p.S + (long long)kBlock * p.N;
    const long long widest = p.d_c > p.d_v ? (p.d_c > p.d_r ? p.d_c : p.d_r) : (p.d_v > p.d_r ? p.d_v : p.d_r);
    if (L * (long long)p.n_h * widest >= (1ll << 31) || (long long)p.S + 8 >= (1ll << 30)) {
        *why = DSPARK_ERR_UNSUPPORTED;
        return false;
    }
    Prob r;
    r.B = p.B; r.n_h = p.n_h; r.S = p.S; r.N = p.N; r.W = p.W;
    r.d_c = p.d_c; r.d_r = p.d_r; r.d_v = p.d_v;
    r.dqk = p.d_c + p.d_r;
    r.R = kBlock * p.N;
    r.L = (int)L;
    r.P = p.S + 8;
    r.base = p.rope_base;
    r.dtype = p.dtype;
    r.scale = (float)(1.0 / std::sqrt((double)r.dqk));
    r.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)r.dqk));
    r.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
    *out = r;
    return true;
}

bool aligned16(const void *x) { return ((uintptr_t)x & 15u) == 0; }

// need_bwd: the backward uses the whole layout, the forward and the
// descriptor only its leading sections.
dspark_status check_ws(const Prob &p, void *ws, size_t bytes, bool need_bwd) {
    if (!ws) return DSPARK_ERR_WORKSPACE;
    if (((uintptr_t)ws & 255u) != 0) return DSPARK_ERR_WORKSPACE;
    const WsLayout l = ws_layout(p);
    if (bytes < (need_bwd ? l.total : l.fwd_total)) return DSPARK_ERR_WORKSPACE;
    return DSPARK_OK;
}

// Tensor pointers may be NULL only when the tensor has no elements.
dspark_status check_tensor(const void *ptr, size_t elems) {
    if (elems == 0) return DSPARK_OK;
    if (!ptr) return DSPARK_ERR_NULL;
    if (!aligned16(ptr)) return DSPARK_ERR_ALIGN;
    return DSPARK_OK;
}

#define DSPARK_TRY(x)                          \
    do {                                       \
        dspark_status _s = (x);                \
        if (_s != DSPARK_OK) return _s;        \
    } while (0)

// With DSPARK_VERBOSE set in the environment, failing CUDA calls are printed
// to stderr with the call that failed.
bool verbose() {
    static const bool v = getenv("DSPARK_VERBOSE") != nullptr;
    return v;
}

#define DSPARK_CUDA(x)                                                                           \
    do {                                                                                         \
        const cudaError_t _e = (x);                                                              \
        if (_e != cudaSuccess) {                                                                 \
            if (verbose()) fprintf(stderr, "dspark: %s failed: %s\n", #x, cudaGetErrorString(_e)); \
            return DSPARK_ERR_CUDA;                                                              \
        }                                                                                        \
    } while (0)

struct Sizes {
    size_t q, kc, kr, v, o, lse, ab;
};

Sizes sizes(const Prob &p) {
    Sizes s;
    s.q = (size_t)p.B * p.n_h * p.R * p.dqk;
    s.kc = (size_t)p.B * p.n_h * p.L * p.d_c;
    s.kr = (size_t)p.B * p.L * p.d_r;
    s.v = (size_t)p.B * p.n_h * p.L * p.d_v;
    s.o = (size_t)p.B * p.n_h * p.R * p.d_v;
    s.lse = (size_t)p.B * p.n_h * p.R;
    s.ab = (size_t)p.B * p.N;
    return s;
}

dspark_status check_inputs(const Prob &p, const void *q, const void *kc, const void *kr, const void *v,
                           const int32_t *anchors, const uint8_t *keep) {
    const Sizes s = sizes(p);
    DSPARK_TRY(check_tensor(q, s.q));
    DSPARK_TRY(check_tensor(kc, s.kc));
    DSPARK_TRY(check_tensor(kr, s.kr));
    DSPARK_TRY(check_tensor(v, s.v));
    if (s.ab && (!anchors || !keep)) return DSPARK_ERR_NULL;
    if (s.ab && ((uintptr_t)anchors & 3u)) return DSPARK_ERR_ALIGN;
    return DSPARK_OK;
}

dspark_status build(const Prob &p, const int32_t *anchors, const uint8_t *keep, const Ws &w, cudaStream_t st) {
    DSPARK_CUDA(launch_build_descriptor(p, anchors, keep, w, st));
    return DSPARK_OK;
}

}  // namespace

namespace dspark {
// Workspace bytes the forward alone needs (a prefix of the full layout); 0 if
// the problem is invalid.
size_t fwd_workspace_size(const dspark_problem *pp) {
    Prob p;
    dspark_status why;
    if (!make_prob(pp, &p, &why)) return 0;
    return ws_layout(p).fwd_total;
}
}  // namespace dspark

extern "C" {

size_t dspark_workspace_size(const dspark_problem *pp) {
    Prob p;
    dspark_status why;
    if (!make_prob(pp, &p, &why)) return 0;
    return ws_layout(p).total;
}

dspark_status dspark_build_descriptor(const dspark_problem *pp, const int32_t *anchors, const uint8_t *keep,
                                      void *workspace, size_t workspace_bytes, void *stream) {
    Prob p;
    dspark_status why;
    if (!make_prob(pp, &p, &why)) return why;
    DSPARK_TRY(check_ws(p, workspace, workspace_bytes, false));
    if ((size_t)p.B * p.N != 0 && (!anchors || !keep)) return DSPARK_ERR_NULL;
    cudaStream_t st = (cudaStream_t)stream;
    return build(p, anchors, keep, ws_view(p, workspace), st);
}

dspark_status dspark_attn_fwd(const dspark_problem *pp, const void *q, const void *kc, const void *kr,
                              const void *v, const int32_t *anchors, const uint8_t *keep, void *o, float *lse,
                              void *workspace, size_t workspace_bytes, uint32_t flags, void *stream) {
    Prob p;
    dspark_status why;
    if (!make_prob(pp, &p, &why)) return why;
    DSPARK_TRY(check_ws(p, workspace, workspace_bytes, false));
    DSPARK_TRY(check_inputs(p, q, kc, kr, v, anchors, keep));
    const Sizes s = sizes(p);
    DSPARK_TRY(check_tensor(o, s.o));
    DSPARK_TRY(check_tensor(lse, s.lse));
    cudaStream_t st = (cudaStream_t)stream;
    const Ws w = ws_view(p, workspace);
    if (!(flags & DSPARK_FLAG_REUSE_DESCRIPTOR)) DSPARK_TRY(build(p, anchors, keep, w, st));
    const bool tc = fwd_tc_supported(p);
    // the tensor-core forward leaves padding blocks' rows to this launch: O = 0, LSE = -inf
    PadRows pad{};
    pad.t[0] = o;
    pad.rows[0] = p.R;
    pad.width[0] = p.d_v;
    pad.lse = lse;
    pad.clear = w.sched;  // the tensor-core forward takes its work items from this counter
    DSPARK_CUDA(launch_rotate_kr(p, kr, anchors, keep, tc ? &pad : nullptr, w, st));
    if (tc)
        DSPARK_CUDA(launch_fwd_tc(p, q, kc, v, anchors, keep, o, lse, w, st));
    else
        DSPARK_CUDA(launch_fwd_simt(p, q, kc, v, anchors, keep, o, lse, w, st));
    return DSPARK_OK;
}

dspark_status dspark_attn_bwd(const dspark_problem *pp, const void *q, const void *kc, const void *kr,
                              const void *v, const int32_t *anchors, const uint8_t *keep, const void *o,
                              const float *lse, const void *do_, void *dq, void *dkc, void *dkr, void *dv,
                              void *workspace, size_t workspace_bytes, uint32_t flags, void *stream) {
    Prob p;
    dspark_status why;
    if (!make_prob(pp, &p, &why)) return why;
    DSPARK_TRY(check_ws(p, workspace, workspace_bytes, true));
    DSPARK_TRY(check_inputs(p, q, kc, kr, v, anchors, keep));
    const Sizes s = sizes(p);
    DSPARK_TRY(check_tensor(o, s.o));
    DSPARK_TRY(check_tensor(lse, s.lse));
    DSPARK_TRY(check_tensor(do_, s.o));
    DSPARK_TRY(check_tensor(dq, s.q));
    DSPARK_TRY(check_tensor(dkc, s.kc));
    DSPARK_TRY(check_tensor(dkr, s.kr));
    DSPARK_TRY(check_tensor(dv, s.v));
    cudaStream_t st = (cudaStream_t)stream;
    const Ws w = ws_view(p, workspace);
    if (!(flags & DSPARK_FLAG_REUSE_DESCRIPTOR)) DSPARK_TRY(build(p, anchors, keep, w, st));
    const bool tc = bwd_tc_supported(p);
    // the tensor-core backward leaves padding blocks' dq rows and their own
    // draft keys' dK^C and dV to this launch (zeros; their dK^R is zeroed by the
    // backward's rope-key reduction)
    PadRows pad{};
    pad.t[0] = dq;
    pad.rows[0] = p.R;
    pad.width[0] = p.dqk;
    pad.t[1] = dkc;
    pad.rows[1] = p.L;
    pad.first[1] = p.S;
    pad.width[1] = p.d_c;
    pad.t[2] = dv;
    pad.rows[2] = p.L;
    pad.first[2] = p.S;
    pad.width[2] = p.d_v;
    DSPARK_CUDA(launch_rotate_kr(p, kr, anchors, keep, tc ? &pad : nullptr, w, st));
    if (tc)
        DSPARK_CUDA(launch_bwd_tc(p, q, kc, v, anchors, keep, o, lse, do_, dq, dkc, dkr, dv, w, st));
    else
        DSPARK_CUDA(launch_bwd_simt(p, q, kc, v, anchors, keep, o, lse, do_, dq, dkc, dkr, dv, w, st));
    return DSPARK_OK;
}

dspark_status dspark_get_error(void *workspace, void *stream) {
    if (!workspace) return DSPARK_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t word = 0;
    // The error word sits at offset 0 of every workspace layout.
    if (cudaStreamSynchronize(st) != cudaSuccess) return DSPARK_ERR_CUDA;
    if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return DSPARK_ERR_CUDA;
    if (word) {
        const uint32_t zero = 0;
        if (cudaMemcpy(workspace, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return DSPARK_ERR_CUDA;
    }
    if (word & kErrTimeout) return DSPARK_ERR_DEVICE;
    if (word & kErrAnchor) return DSPARK_ERR_ANCHOR;
    return DSPARK_OK;
}

uint64_t dspark_launch_counter(void) { return g_launches.load(std::memory_order_relaxed); }

static bool aligned4(const void *x) { return ((uintptr_t)x & 3u) == 0; }

dspark_status dspark_sample_anchors_gpu(const uint8_t *loss_mask, int32_t B, int32_t S, int32_t N, uint64_t seed,
                                        int32_t *anchors, uint8_t *keep, void *stream) {
    if (B < 0 || S < 1 || N < 0) return DSPARK_ERR_SHAPE;
    if (S >= (1 << 30) || N > 8192) return DSPARK_ERR_UNSUPPORTED;
    if ((int64_t)B * N == 0) return DSPARK_OK;
    if (!loss_mask || !anchors || !keep) return DSPARK_ERR_NULL;
    if (!aligned4(anchors)) return DSPARK_ERR_ALIGN;
    DSPARK_CUDA(launch_sample_anchors(loss_mask, B, S, N, seed, anchors, keep, (cudaStream_t)stream));
    return DSPARK_OK;
}

dspark_status dspark_build_draft_inputs(const int32_t *input_ids, const uint8_t *loss_mask, int32_t B, int32_t S,
                                        int32_t N, const int32_t *anchors, const uint8_t *keep, int32_t mask_id,
                                        int32_t *draft_ids, int32_t *position_ids, int32_t *labels,
                                        int32_t *prev_ids, uint8_t *eval_mask, void *stream) {
    if (B < 0 || S < 1 || N < 0) return DSPARK_ERR_SHAPE;
    if (S >= (1 << 30) || N > 8192) return DSPARK_ERR_UNSUPPORTED;
    if ((int64_t)B * N == 0) return DSPARK_OK;
    if (!input_ids || !loss_mask || !anchors || !keep || !draft_ids || !position_ids || !labels || !prev_ids ||
        !eval_mask)
        return DSPARK_ERR_NULL;
    if (!aligned4(input_ids) || !aligned4(anchors) || !aligned4(draft_ids) || !aligned4(position_ids) ||
        !aligned4(labels) || !aligned4(prev_ids))
        return DSPARK_ERR_ALIGN;
    DSPARK_CUDA(launch_build_draft_inputs(input_ids, loss_mask, B, S, N, anchors, keep, mask_id, draft_ids,
                                          position_ids, labels, prev_ids, eval_mask, (cudaStream_t)stream));
    return DSPARK_OK;
}

size_t dspark_loss_workspace_size(int32_t R) { return R < 0 ? 0 : loss_workspace_size(R); }

dspark_status dspark_loss_fwd_bwd(int32_t R, int32_t V, const void *student_logits, const void *teacher_logits,
                                  const int32_t *labels, const float *conf_logits, const uint8_t *eval_mask,
                                  float ce_alpha, float l1_alpha, float conf_alpha, float *loss_out,
                                  void *grad_logits, float *grad_conf, void *workspace, size_t workspace_bytes,
                                  void *stream) {
    if (R < 0 || V < 8 || (V % 8) != 0) return DSPARK_ERR_SHAPE;
    if (V > 229376 || (int64_t)R * V >= (1ll << 40)) return DSPARK_ERR_UNSUPPORTED;  // two row slices per CTA
    if (!loss_out || !workspace || (R > 0 && (!student_logits || !teacher_logits || !labels || !conf_logits ||
                                              !eval_mask)))
        return DSPARK_ERR_NULL;
    if (workspace_bytes < loss_workspace_size(R) || ((uintptr_t)workspace & 255u)) return DSPARK_ERR_WORKSPACE;
    if ((R > 0 && (!aligned16(student_logits) || !aligned16(teacher_logits))) ||
        (grad_logits && !aligned16(grad_logits)) || !aligned4(loss_out) || (labels && !aligned4(labels)) ||
        (conf_logits && !aligned4(conf_logits)) || (grad_conf && !aligned4(grad_conf)))
        return DSPARK_ERR_ALIGN;
    DSPARK_CUDA(launch_loss(R, V, student_logits, teacher_logits, labels, conf_logits, eval_mask, ce_alpha, l1_alpha,
                            conf_alpha, loss_out, grad_logits, grad_conf, workspace,
                            g_wait_ns.load(std::memory_order_relaxed), (cudaStream_t)stream));
    return DSPARK_OK;
}

uint64_t dspark_set_wait_limit_ns(uint64_t ns) {
    if (ns == 0 || ns > kWaitTimeoutNs) ns = kWaitTimeoutNs;
    return g_wait_ns.exchange(ns, std::memory_order_relaxed);
}

const char *dspark_status_string(dspark_status s) {
    switch (s) {
        case DSPARK_OK: return "ok";
        case DSPARK_ERR_NULL: return "a required pointer is NULL";
        case DSPARK_ERR_SHAPE: return "a size is out of range or inconsistent";
        case DSPARK_ERR_DTYPE: return "unknown dtype";
        case DSPARK_ERR_ANCHOR: return "a kept anchor is outside [0, S-2]";
        case DSPARK_ERR_WORKSPACE: return "workspace missing, too small or not 256-byte aligned";
        case DSPARK_ERR_CUDA: return "a CUDA call or kernel launch failed";
        case DSPARK_ERR_DEVICE: return "a bounded device-side wait gave up";
        case DSPARK_ERR_ALIGN: return "a tensor pointer is not 16-byte aligned";
        case DSPARK_ERR_UNSUPPORTED: return "sizes outside what the kernels implement";
    }
    return "unknown status";
}

}  // extern "C"
