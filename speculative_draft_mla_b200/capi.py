"""Python binding of the C ABI in include/dspark_attn.h (argument marshalling only).

Every step of the attention runs in the CUDA library ``libdspark_attn.so``
built in-tree by ``speculative_draft_mla_b200.build``. There is no fallback:
if the library is missing or the tensors are not CUDA tensors, the calls raise.
Function names follow the C entry points without the ``dspark_`` prefix.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdspark_attn.so")

F32, BF16 = 0, 1
FLAG_REUSE_DESCRIPTOR = 1
STATUS = {0: "OK", 1: "ERR_NULL", 2: "ERR_SHAPE", 3: "ERR_DTYPE", 4: "ERR_ANCHOR", 5: "ERR_WORKSPACE",
          6: "ERR_CUDA", 7: "ERR_DEVICE", 8: "ERR_ALIGN", 9: "ERR_UNSUPPORTED"}
EXPORTS = ("dspark_workspace_size", "dspark_build_descriptor", "dspark_attn_fwd", "dspark_attn_bwd",
           "dspark_get_error", "dspark_status_string", "dspark_sample_anchors", "dspark_launch_counter",
           "dspark_set_wait_limit_ns", "dspark_sample_anchors_gpu", "dspark_build_draft_inputs",
           "dspark_loss_workspace_size", "dspark_loss_fwd_bwd")
MASK_ID = 154821  # the page's MASK token id


class Problem(ctypes.Structure):
    """Mirror of dspark_problem."""
    _fields_ = [("B", ctypes.c_int32), ("n_h", ctypes.c_int32), ("S", ctypes.c_int32), ("N", ctypes.c_int32),
                ("W", ctypes.c_int32), ("d_c", ctypes.c_int32), ("d_r", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("rope_base", ctypes.c_double), ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class DsparkError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s (%s)" % (where, STATUS.get(status, status), status_string(status)))


_lib = None


def load():
    """Load the CUDA library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libdspark_attn.so is not built; run `python -m speculative_draft_mla_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, u32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint32
    pp = ctypes.POINTER(Problem)
    lib.dspark_workspace_size.argtypes = [pp]
    lib.dspark_workspace_size.restype = sz
    lib.dspark_build_descriptor.argtypes = [pp, vp, vp, vp, sz, vp]
    lib.dspark_attn_fwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, u32, vp]
    lib.dspark_attn_bwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, u32, vp]
    lib.dspark_get_error.argtypes = [vp, vp]
    lib.dspark_status_string.argtypes = [ctypes.c_int]
    lib.dspark_status_string.restype = ctypes.c_char_p
    lib.dspark_sample_anchors.argtypes = [vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_uint64, vp, vp]
    lib.dspark_sample_anchors.restype = ctypes.c_int64
    lib.dspark_attn_fwd_noalloc.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.dspark_attn_fwd_noalloc.restype = ctypes.c_int
    lib.dspark_launch_counter.argtypes = []
    lib.dspark_launch_counter.restype = ctypes.c_uint64
    i32 = ctypes.c_int32
    lib.dspark_sample_anchors_gpu.argtypes = [vp, i32, i32, i32, ctypes.c_uint64, vp, vp, vp]
    lib.dspark_sample_anchors_gpu.restype = ctypes.c_int
    lib.dspark_build_draft_inputs.argtypes = [vp, vp, i32, i32, i32, vp, vp, i32, vp, vp, vp, vp, vp, vp]
    lib.dspark_build_draft_inputs.restype = ctypes.c_int
    lib.dspark_loss_workspace_size.argtypes = [i32]
    lib.dspark_loss_workspace_size.restype = sz
    f32 = ctypes.c_float
    lib.dspark_loss_fwd_bwd.argtypes = [i32, i32, vp, vp, vp, vp, vp, f32, f32, f32, vp, vp, vp, vp, sz, vp]
    lib.dspark_loss_fwd_bwd.restype = ctypes.c_int
    lib.dspark_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.dspark_set_wait_limit_ns.restype = ctypes.c_uint64
    for f in ("dspark_build_descriptor", "dspark_attn_fwd", "dspark_attn_bwd", "dspark_get_error"):
        getattr(lib, f).restype = ctypes.c_int
    _lib = lib
    return lib


def status_string(status):
    return load().dspark_status_string(int(status)).decode()


def problem(B, n_h, S, N, W, d_c, d_r, d_v, rope_base=10000.0, dtype=BF16):
    return Problem(B, n_h, S, N, W, d_c, d_r, d_v, float(rope_base), int(dtype), 0)


def dtype_code(t):
    if t == torch.float32:
        return F32
    if t == torch.bfloat16:
        return BF16
    raise TypeError("unsupported dtype %s" % t)


def _ptr(t):
    return None if t is None or t.numel() == 0 else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status, where):
    if status != 0:
        raise DsparkError(status, where)


def workspace_size(prob):
    return int(load().dspark_workspace_size(ctypes.byref(prob)))


def alloc_workspace(prob, device):
    n = workspace_size(prob)
    if n == 0:
        raise DsparkError(2, "workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def problem_of(q, kc, kr, v, anchors, S, W, rope_base):
    B, n_h, R, dqk = q.shape
    return problem(B, n_h, S, R // 5, W, kc.shape[-1], kr.shape[-1], v.shape[-1], rope_base, dtype_code(q.dtype))


def build_descriptor(prob, anchors, keep, workspace, stream=None):
    _cuda(anchors, keep, workspace)
    st = _stream(stream, workspace.device)
    _check(load().dspark_build_descriptor(ctypes.byref(prob), _ptr(anchors), _ptr(keep), _ptr(workspace),
                                          workspace.numel(), st), "dspark_build_descriptor")


def attn_fwd(q, kc, kr, v, anchors, keep, S, W, rope_base=10000.0, workspace=None, flags=0, out=None, stream=None):
    """Returns (o, lse, workspace). ``out`` may pass preallocated (o, lse)."""
    _cuda(q, kc, kr, v, anchors, keep)
    prob = problem_of(q, kc, kr, v, anchors, S, W, rope_base)
    if workspace is None:
        workspace = alloc_workspace(prob, q.device)
    if out is None:
        o = torch.empty(q.shape[:3] + (v.shape[-1],), dtype=q.dtype, device=q.device)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    _cuda(o, lse, workspace)
    st = _stream(stream, q.device)
    _check(load().dspark_attn_fwd(ctypes.byref(prob), _ptr(q), _ptr(kc), _ptr(kr), _ptr(v), _ptr(anchors),
                                  _ptr(keep), _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel(), flags, st),
           "dspark_attn_fwd")
    return o, lse, workspace


def attn_bwd(q, kc, kr, v, anchors, keep, o, lse, dout, S, W, rope_base=10000.0, workspace=None, flags=0,
             out=None, stream=None):
    """Returns (dq, dkc, dkr, dv). ``out`` may pass preallocated gradients."""
    _cuda(q, kc, kr, v, anchors, keep, o, lse, dout)
    prob = problem_of(q, kc, kr, v, anchors, S, W, rope_base)
    if workspace is None:
        workspace = alloc_workspace(prob, q.device)
    if out is None:
        dq, dkc, dkr, dv = (torch.empty_like(q), torch.empty_like(kc), torch.empty_like(kr), torch.empty_like(v))
    else:
        dq, dkc, dkr, dv = out
    _cuda(dq, dkc, dkr, dv, workspace)
    st = _stream(stream, q.device)
    _check(load().dspark_attn_bwd(ctypes.byref(prob), _ptr(q), _ptr(kc), _ptr(kr), _ptr(v), _ptr(anchors),
                                  _ptr(keep), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dkc), _ptr(dkr),
                                  _ptr(dv), _ptr(workspace), workspace.numel(), flags, st), "dspark_attn_bwd")
    return dq, dkc, dkr, dv


def attn_fwd_noalloc(q, kc, kr, v, anchors, keep, S, W, rope_base=10000.0, out=None, error_word=None,
                     stream=None):
    """Forward through dspark_attn_fwd_noalloc (no workspace argument: the
    library's built-in scratch array is used). Returns (o, lse)."""
    _cuda(q, kc, kr, v, anchors, keep, error_word)
    prob = problem_of(q, kc, kr, v, anchors, S, W, rope_base)
    if out is None:
        o = torch.empty(q.shape[:3] + (v.shape[-1],), dtype=q.dtype, device=q.device)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    _cuda(o, lse)
    st = _stream(stream, q.device)
    _check(load().dspark_attn_fwd_noalloc(ctypes.byref(prob), _ptr(q), _ptr(kc), _ptr(kr), _ptr(v), _ptr(anchors),
                                          _ptr(keep), _ptr(o), _ptr(lse), _ptr(error_word), st),
           "dspark_attn_fwd_noalloc")
    return o, lse


def get_error(workspace, stream=None):
    """Synchronise and read (and clear) the device error word; raises on error."""
    st = _stream(stream, workspace.device)
    _check(load().dspark_get_error(_ptr(workspace), st), "dspark_get_error")


def launch_counter():
    """Kernels the library has launched in this process so far."""
    return int(load().dspark_launch_counter())


def set_wait_limit_ns(ns):
    """Limit (ns) of the kernels' pipeline waits for later calls; 0 restores
    the default (2 s). Returns the previous limit."""
    return int(load().dspark_set_wait_limit_ns(int(ns)))


def sample_anchors_gpu(loss_mask, N, seed, stream=None):
    """GPU anchor sampler: loss_mask uint8 [B, S] (CUDA) -> (anchors int32 [B, N], keep uint8 [B, N])."""
    _cuda(loss_mask)
    if loss_mask.dtype != torch.uint8:
        raise TypeError("loss_mask must be uint8")
    B, S = loss_mask.shape
    anchors = torch.empty(B, N, dtype=torch.int32, device=loss_mask.device)
    keep = torch.empty(B, N, dtype=torch.uint8, device=loss_mask.device)
    _check(load().dspark_sample_anchors_gpu(_ptr(loss_mask), B, S, N, ctypes.c_uint64(seed & (2 ** 64 - 1)),
                                            _ptr(anchors), _ptr(keep), _stream(stream, loss_mask.device)),
           "dspark_sample_anchors_gpu")
    return anchors, keep


def build_draft_inputs(input_ids, loss_mask, anchors, keep, mask_id=MASK_ID, stream=None):
    """Draft-block inputs: input_ids int32 [B, S], loss_mask uint8 [B, S], anchors int32 / keep uint8
    [B, N] (CUDA) -> dict of [B, 5N] tensors: draft_ids, position_ids, labels, prev_ids (int32) and
    eval_mask (uint8)."""
    _cuda(input_ids, loss_mask, anchors, keep)
    if input_ids.dtype != torch.int32 or anchors.dtype != torch.int32 or loss_mask.dtype != torch.uint8 or \
            keep.dtype != torch.uint8:
        raise TypeError("input_ids / anchors int32, loss_mask / keep uint8")
    B, S = input_ids.shape
    N = anchors.shape[1]
    dev = input_ids.device
    out = {k: torch.empty(B, 5 * N, dtype=torch.int32, device=dev)
           for k in ("draft_ids", "position_ids", "labels", "prev_ids")}
    out["eval_mask"] = torch.empty(B, 5 * N, dtype=torch.uint8, device=dev)
    _check(load().dspark_build_draft_inputs(_ptr(input_ids), _ptr(loss_mask), B, S, N, _ptr(anchors), _ptr(keep),
                                            int(mask_id), _ptr(out["draft_ids"]), _ptr(out["position_ids"]),
                                            _ptr(out["labels"]), _ptr(out["prev_ids"]), _ptr(out["eval_mask"]),
                                            _stream(stream, dev)), "dspark_build_draft_inputs")
    return out


CE_ALPHA, L1_ALPHA, CONF_ALPHA = 1.0, 0.9, 1.0  # the page's loss coefficients


def dspark_loss(student_logits, teacher_logits, labels, conf_logits, eval_mask, with_grad=True,
                alphas=(CE_ALPHA, L1_ALPHA, CONF_ALPHA), workspace=None, stream=None):
    """DSpark loss over R draft steps: bf16 [R, V] logits, int32 labels, float conf logits, uint8
    eval_mask (CUDA). Returns (loss [4] float: total, CE, L1, BCE means; grad_logits or None;
    grad_conf or None; workspace)."""
    _cuda(student_logits, teacher_logits, labels, conf_logits, eval_mask)
    if student_logits.dtype != torch.bfloat16 or teacher_logits.dtype != torch.bfloat16:
        raise TypeError("logits must be bf16")
    R, V = student_logits.shape
    dev = student_logits.device
    if workspace is None:
        workspace = torch.empty(int(load().dspark_loss_workspace_size(R)), dtype=torch.uint8, device=dev)
    out = torch.empty(4, dtype=torch.float32, device=dev)
    grad = torch.empty_like(student_logits) if with_grad else None
    gconf = torch.empty(R, dtype=torch.float32, device=dev) if with_grad else None
    _check(load().dspark_loss_fwd_bwd(R, V, _ptr(student_logits), _ptr(teacher_logits), _ptr(labels),
                                      _ptr(conf_logits), _ptr(eval_mask), float(alphas[0]), float(alphas[1]),
                                      float(alphas[2]), _ptr(out), _ptr(grad), _ptr(gconf), _ptr(workspace),
                                      workspace.numel(), _stream(stream, dev)), "dspark_loss_fwd_bwd")
    return out, grad, gconf, workspace


def sample_anchors(loss_mask, N, seed):
    """Host anchor sampler: loss_mask uint8 [B, S] (CPU) -> (anchors int32, keep uint8), CPU."""
    lm = loss_mask.to(torch.uint8).contiguous().cpu()
    B, S = lm.shape
    anchors = torch.empty(B, N, dtype=torch.int32)
    keep = torch.empty(B, N, dtype=torch.uint8)
    rc = load().dspark_sample_anchors(_ptr(lm), B, S, N, ctypes.c_uint64(seed), _ptr(anchors), _ptr(keep))
    if rc < 0:
        raise DsparkError(2, "dspark_sample_anchors")
    return anchors, keep
