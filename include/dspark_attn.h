/*
 * dspark_attn.h — C ABI of the B200 (sm_100a) DSpark draft MLA attention.
 *
 * The operation (page "GLM 5.2 DSpark speculative-training design"):
 *   The KV axis is [S context positions | N draft blocks x 5 positions]
 *   (§2 "QKV construction"). The queries are the 5N draft positions. A query of
 *   block n, anchor A = anchors[b][n], sees exactly
 *     - the context window max(0, A-W+1) <= kv < A, shared by the 5 offsets of
 *       the block and excluding position A (§3 "attention mask"), and
 *     - the 5 positions of its own block, bidirectionally (§3);
 *   a block with keep[b][n] = 0 (block_keep_mask, a padding block) sees nothing.
 *   Per head the query is [q^C ; q^R] and the key [k^C ; k^R], where the rope key
 *   k^R is one d_r-wide vector per position shared by all heads (§4 "MLA").
 *   RoPE rotates only the rope slice, interleaved adjacent pairs (2i, 2i+1), by
 *   angle pos * rope_base^(-2i/d_r); positions are 0..S-1 for context and
 *   A_n .. A_n+4 for block n (§2, §4 "RoPE").
 *   O = softmax(Q K^T / sqrt(d_c + d_r) + Lambda(M)) V with Lambda = -inf off the
 *   mask (appendix "Attention implementation"). Rows of padding blocks give
 *   O = 0, LSE = -inf and zero gradients.
 *
 * Layouts (contiguous, row-major; "dtype" is fp32 or bf16 as given by
 * dspark_problem.dtype; all tensors on the CUDA device unless stated):
 *   q   [B, n_h, 5N, d_c + d_r]  dtype   query, rope slice last, NOT rotated
 *   kc  [B, n_h, S + 5N, d_c]    dtype   per-head key, non-rope part
 *   kr  [B, S + 5N, d_r]         dtype   rope key shared by heads, NOT rotated
 *   v   [B, n_h, S + 5N, d_v]    dtype
 *   anchors [B, N] int32; keep [B, N] uint8 (0 = padding block)
 *   o   [B, n_h, 5N, d_v]        dtype;  lse [B, n_h, 5N] fp32 (natural log)
 *   do_ like o; dq like q; dkc like kc; dkr like kr; dv like v
 *   (gradients are with respect to the un-rotated inputs).
 * Row r = 5n + j of q / o is offset j of block n. Every element of every output
 * is written (zeros included).
 *
 * Ownership: the caller allocates and owns every buffer, the workspace
 * included. The library allocates no device memory, launches only on the
 * given stream (a cudaStream_t passed as void*, NULL = legacy default stream)
 * and never synchronises, except dspark_get_error.
 *
 * Errors: argument checks run on the host before any launch and return a
 * status without touching device memory. A kept anchor outside [0, S-2] can
 * only be seen on the device: that block is then treated as a padding block
 * and a bit is set in the workspace error word, read by dspark_get_error.
 */
#ifndef DSPARK_ATTN_H
#define DSPARK_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSPARK_API __attribute__((visibility("default")))
#else
#define DSPARK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSPARK_OK = 0,
    DSPARK_ERR_NULL = 1,        /* a required pointer is NULL */
    DSPARK_ERR_SHAPE = 2,       /* a size is out of range or inconsistent */
    DSPARK_ERR_DTYPE = 3,       /* unknown dtype */
    DSPARK_ERR_ANCHOR = 4,      /* (device) a kept anchor outside [0, S-2] */
    DSPARK_ERR_WORKSPACE = 5,   /* workspace NULL, too small or misaligned */
    DSPARK_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed */
    DSPARK_ERR_DEVICE = 7,      /* (device) a bounded wait gave up */
    DSPARK_ERR_ALIGN = 8,       /* a tensor pointer is not 16-byte aligned */
    DSPARK_ERR_UNSUPPORTED = 9  /* sizes outside what the kernels implement */
} dspark_status;

typedef enum { DSPARK_F32 = 0, DSPARK_BF16 = 1 } dspark_dtype;

/* Problem sizes (page notation). Limits checked on the host:
 *   B >= 0, n_h >= 1, S >= 1, N >= 0, 1 <= W <= 4096, N <= 8192,
 *   d_c >= 0, d_r >= 0 even, d_v >= 1, d_c + d_r >= 1, d_c + d_r <= 256,
 *   d_v <= 256, (S + 5N) * n_h * max(d_c, d_v) < 2^31, rope_base > 0. */
typedef struct {
    int32_t B;          /* batch */
    int32_t n_h;        /* heads */
    int32_t S;          /* context positions */
    int32_t N;          /* draft blocks (5 positions each) */
    int32_t W;          /* sliding window: W-1 context positions visible */
    int32_t d_c;        /* per-head non-rope query/key width */
    int32_t d_r;        /* rope width (shared rope key) */
    int32_t d_v;        /* per-head value width */
    double rope_base;   /* RoPE base, e.g. 10000 */
    int32_t dtype;      /* dspark_dtype of q, kc, kr, v, o, do, dq, dkc, dkr, dv */
    int32_t reserved;   /* must be 0 */
} dspark_problem;

/* Flags of dspark_attn_fwd / dspark_attn_bwd. */
#define DSPARK_FLAG_REUSE_DESCRIPTOR 1u /* the workspace already holds the
        descriptor built by dspark_build_descriptor (or by an earlier fwd/bwd)
        for the same anchors, keep and sizes: skip rebuilding it. The page's
        mask is built once and shared by the three draft layers (§3, §4). */

/* Bytes of device workspace needed for problem *p (0 if *p is invalid): the
 * size dspark_attn_bwd requires. dspark_build_descriptor and dspark_attn_fwd
 * use only a leading part of it, so a workspace of this size serves every
 * entry point. The workspace must be 256-byte aligned. */
DSPARK_API size_t dspark_workspace_size(const dspark_problem *p);

/* Build the mask descriptor into the workspace: kept blocks of each batch row
 * sorted by anchor (ties by block index), per-row kept counts, and the RoPE
 * cos/sin table for positions 0 .. S+7. Validates kept anchors on the device
 * (see dspark_get_error). Clears the workspace error word first, so the word
 * reports what happened since the last descriptor build.
 * anchors, keep: device pointers [B, N]. */
DSPARK_API dspark_status dspark_build_descriptor(const dspark_problem *p, const int32_t *anchors, const uint8_t *keep,
                                      void *workspace, size_t workspace_bytes, void *stream);

/* Forward: o and lse (layouts above). Builds the descriptor first unless
 * flags has DSPARK_FLAG_REUSE_DESCRIPTOR. */
DSPARK_API dspark_status dspark_attn_fwd(const dspark_problem *p, const void *q, const void *kc, const void *kr,
                              const void *v, const int32_t *anchors, const uint8_t *keep, void *o, float *lse,
                              void *workspace, size_t workspace_bytes, uint32_t flags, void *stream);

/* Forward without a caller workspace. The page has no counterpart to this
 * entry point: it exists for callers that get only their input and output
 * buffers and may not allocate device memory (a plugin inside another
 * framework's execution hook, whose device memory that framework already owns;
 * a latency-bound loop that cannot afford the device synchronisation of
 * cudaMalloc/cudaFree). It runs the dspark_attn_fwd sequence with the
 * workspace in a device array compiled into the library, so it allocates
 * nothing at run time; every GPU that loads the library keeps that array,
 * DSPARK_NOALLOC_SCRATCH_BYTES (16 MiB), until the process exits.
 *   - Arguments and layouts as dspark_attn_fwd. error_word (device pointer,
 *     may be NULL) receives, in stream order, the error word of this call
 *     (bit 0: a kept anchor was out of range and its block treated as padding;
 *     bit 1: a bounded device-side wait gave up).
 *   - Returns DSPARK_ERR_UNSUPPORTED when the forward needs more scratch than
 *     the array holds; other statuses as dspark_attn_fwd.
 *   - Every call outside a stream capture looks up the array's device address
 *     (cudaGetSymbolAddress, with the stream's device current), so a
 *     cudaDeviceReset between calls is harmless; a call on a stream that is
 *     being captured reuses the address of the last uncaptured call on that
 *     device. Make the first call on a device before any stream capture.
 *   - All calls share the one array, which keeps the last call's contents: two
 *     calls whose work overlaps on the GPU (different streams, or different
 *     host threads on the same device) race on it. Serialise them. */
#define DSPARK_NOALLOC_SCRATCH_BYTES (16u << 20)
DSPARK_API dspark_status dspark_attn_fwd_noalloc(const dspark_problem *p, const void *q, const void *kc,
                                                 const void *kr, const void *v, const int32_t *anchors,
                                                 const uint8_t *keep, void *o, float *lse, uint32_t *error_word,
                                                 void *stream);

/* Backward of the forward for a loss L with dL/dO = do_: writes dq, dkc, dkr,
 * dv. o and lse are the forward's outputs for the same inputs. Builds the
 * descriptor first unless flags has DSPARK_FLAG_REUSE_DESCRIPTOR. */
DSPARK_API dspark_status dspark_attn_bwd(const dspark_problem *p, const void *q, const void *kc, const void *kr,
                              const void *v, const int32_t *anchors, const uint8_t *keep, const void *o,
                              const float *lse, const void *do_, void *dq, void *dkc, void *dkr, void *dv,
                              void *workspace, size_t workspace_bytes, uint32_t flags, void *stream);

/* Synchronises the stream, reads and clears the workspace error word.
 * Returns DSPARK_OK, DSPARK_ERR_ANCHOR (a kept anchor was out of range) or
 * DSPARK_ERR_DEVICE (a bounded wait in a kernel gave up). */
DSPARK_API dspark_status dspark_get_error(void *workspace, void *stream);

/* Static description of a status code. */
DSPARK_API const char *dspark_status_string(dspark_status s);

/* Number of kernels this library has launched in the calling process since it
 * was loaded (host-side count, incremented at every launch; monotonic). Lets a
 * caller count the device work of a timed region. */
DSPARK_API uint64_t dspark_launch_counter(void);

/* Time after which a bounded wait inside a kernel gives up (ns; default and
 * maximum 2 s). Every pipeline wait of the tensor-core kernels (a consumer
 * waiting for a copy or an MMA, a producer waiting for a free stage, the MMA
 * issuer waiting for any operand) gives up after this long, raises its CTA's
 * abort flag, and the call then reports DSPARK_ERR_DEVICE through
 * dspark_get_error; the outputs of such a call are unspecified. The waits that
 * let copies and MMAs already issued complete before a CTA exits keep the 2 s
 * limit whatever is set here. Process-wide, read by each fwd / bwd call when
 * it launches. ns = 0, or a value above 2 s, sets the default. Returns the
 * limit in effect before the call. A limit far below the kernels' own
 * latencies makes the waits run out on purpose, so the time-out path (error
 * report, copies drained, TMEM released, context usable afterwards) can be
 * exercised without a stalled device. */
DSPARK_API uint64_t dspark_set_wait_limit_ns(uint64_t ns);

/* Host helper, page §2 "anchor sampling": for each batch row, the candidates
 * are A in [0, S-2] with loss_mask[A] = loss_mask[A+1] = 1, where
 * loss_mask[S-1] is read as 0 (appendix A: the last position is neither an
 * anchor nor a label). Draws min(N, #candidates) of them uniformly without
 * replacement (a Fisher-Yates shuffle driven by SplitMix64 seeded with
 * seed + row), writes them in draw order, and pads the rest with anchor 0,
 * keep 0 (padding blocks, §3). All pointers are host memory:
 * loss_mask [B, S] uint8, anchors_out [B, N] int32, keep_out [B, N] uint8.
 * Returns the total number of kept blocks, or -1 on bad arguments. */
DSPARK_API int64_t dspark_sample_anchors(const uint8_t *loss_mask, int32_t B, int32_t S, int32_t N, uint64_t seed,
                              int32_t *anchors_out, uint8_t *keep_out);

/* GPU anchor sampler, page §2 "anchor sampling": for each batch row b the
 * candidates are A in [0, S-2] with loss_mask[A] = loss_mask[A+1] = 1, where
 * loss_mask[S-1] is read as 0 (§6). Each candidate gets the key k_A = output A
 * (counted from 0) of SplitMix64 started from state seed + b, and the
 * min(N, #candidates) candidates with the smallest (k_A, A) are kept (a uniform
 * draw without replacement), written in ascending order of A; the remaining
 * entries are padding blocks, anchor 0 and keep 0 (§3). Deterministic for a
 * given seed. This draw differs from dspark_sample_anchors' (a shuffle, in draw
 * order); both are uniform.
 *   loss_mask [B, S] uint8, anchors [B, N] int32 (4-byte aligned),
 *   keep [B, N] uint8: device pointers, owned by the caller.
 * Limits: B >= 0, 1 <= S < 2^30, 0 <= N <= 8192. Launches one kernel on the
 * stream; returns a status from the host checks (nothing is written on error)
 * or DSPARK_ERR_CUDA if the launch fails. */
DSPARK_API dspark_status dspark_sample_anchors_gpu(const uint8_t *loss_mask, int32_t B, int32_t S, int32_t N,
                                                   uint64_t seed, int32_t *anchors, uint8_t *keep, void *stream);

/* Draft-block inputs for anchors / keep [B, N] (page §2 "Draft block", §5
 * Markov head, §6 "Label" and "eval_mask"). For block n with anchor A and
 * offset j = 0..4, row 5n + j of each [B, 5N] output holds
 *   draft_ids    x_A at j = 0, mask_id at j = 1..4 (the page's MASK is 154821)
 *   position_ids A + j (the block's RoPE positions on the KV axis)
 *   labels       y_j = x_{A+j+1}
 *   prev_ids     x_{A+j} (the anchor, then the gold tokens: the Markov head's
 *                predecessors)
 *   eval_mask    1 while every step j' <= j has A+j'+1 < S, loss_mask[A+j'+1] = 1
 *                (loss_mask[S-1] read as 0) and keep = 1 (a prefix product
 *                along the block), else 0.
 * Positions outside [0, S) read as mask_id (draft_ids, prev_ids) and -1
 * (labels); such steps have eval_mask 0.
 *   input_ids [B, S] int32, loss_mask [B, S] uint8, anchors [B, N] int32,
 *   keep [B, N] uint8; outputs int32 except eval_mask (uint8). Device pointers
 *   owned by the caller; int32 arrays 4-byte aligned.
 * Limits, errors and launches as dspark_sample_anchors_gpu. */
DSPARK_API dspark_status dspark_build_draft_inputs(const int32_t *input_ids, const uint8_t *loss_mask, int32_t B,
                                                   int32_t S, int32_t N, const int32_t *anchors, const uint8_t *keep,
                                                   int32_t mask_id, int32_t *draft_ids, int32_t *position_ids,
                                                   int32_t *labels, int32_t *prev_ids, uint8_t *eval_mask,
                                                   void *stream);

/* Bytes of device workspace dspark_loss_fwd_bwd needs for R rows (256-byte
 * aligned). */
DSPARK_API size_t dspark_loss_workspace_size(int32_t R);

/* The DSpark training loss over R draft steps and its gradient (page §6).
 * Row r holds student logits L_r = student_logits[r] and teacher logits
 * T_r = teacher_logits[r] over the vocabulary (V entries each), the label
 * y_r = labels[r], the confidence-head logit c_r = conf_logits[r] and
 * m_r = eval_mask[r] (0 / 1). With p = softmax(L_r), q = softmax(T_r):
 *   CE_r  = logsumexp(L_r) - L_r[y_r]
 *   L1_r  = sum_i |p_i - q_i|
 *   a_r   = clip(1 - L1_r / 2, 0, 1)            (a target: no gradient)
 *   BCE_r = max(c_r, 0) - c_r a_r + log(1 + exp(-|c_r|))
 *   loss  = ce_alpha CE + l1_alpha L1 + conf_alpha BCE, each the sum over the
 *           counted steps (m_r = 1) divided by their number M (the page's
 *           coefficients are 1, 0.9 and 1).
 * Writes loss_out[4] = {loss, CE mean, L1 mean, BCE mean} and, when given,
 *   grad_logits[r][i] = (m_r / M) (ce_alpha (p_i - [i = y_r])
 *                                  + l1_alpha p_i (s_i - sum_j s_j p_j)),
 *       s = sign(p - q) (0 where p = q), rounded to bf16 (every element of
 *       every row is written, zeros for uncounted rows),
 *   grad_conf[r] = (m_r / M) conf_alpha (sigmoid(c_r) - a_r).
 * M = 0 gives a zero loss and zero gradients; a label outside [0, V) adds no
 * CE term. Teacher logits get no gradient.
 *   student_logits, teacher_logits, grad_logits: [R, V] bf16, 16-byte aligned;
 *   labels [R] int32, conf_logits [R] float, eval_mask [R] uint8, grad_conf [R]
 *   float, loss_out [4] float: device pointers owned by the caller;
 *   grad_logits and grad_conf may be NULL (loss only).
 * Limits: R >= 0, V >= 8 and a multiple of 8, V <= 229376. Host checks return
 * before any launch; a bounded wait that gives up is reported through the
 * workspace as in dspark_get_error (DSPARK_ERR_DEVICE). Launches four
 * operations on the stream (a count, the loss kernel in clusters of 8 CTAs, a
 * fixed-order reduction and a memset). */
DSPARK_API dspark_status dspark_loss_fwd_bwd(int32_t R, int32_t V, const void *student_logits,
                                             const void *teacher_logits, const int32_t *labels,
                                             const float *conf_logits, const uint8_t *eval_mask, float ce_alpha,
                                             float l1_alpha, float conf_alpha, float *loss_out, void *grad_logits,
                                             float *grad_conf, void *workspace, size_t workspace_bytes,
                                             void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DSPARK_ATTN_H */
