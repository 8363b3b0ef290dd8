"""ctypes binding of liblwm_attn.so (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: it checks that tensors are CUDA tensors of the right
shape, allocates outputs and workspace with torch (device memory is torch's
job), passes raw pointers and the current stream, and turns a non-zero
status into an exception.  If the shared library is missing the import fails
loudly; there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblwm_attn.so")

LWM_OK = 0
LWM_DTYPE_BF16 = 0
LWM_DTYPE_FP32 = 1

STATUS_NAMES = {
    0: "LWM_OK", -1: "LWM_ERR_INVALID_ARG", -2: "LWM_ERR_UNSUPPORTED", -3: "LWM_ERR_ALIGNMENT",
    -4: "LWM_ERR_WORKSPACE", -5: "LWM_ERR_CUDA", -6: "LWM_ERR_TIMEOUT",
}

ENTRY_POINTS = ("lwm_attn_workspace_size", "lwm_attn_fwd", "lwm_attn_bwd", "lwm_rope_apply",
                "lwm_attn_read_status", "lwm_status_string", "lwm_attn_set_timing_events",
                "lwm_attn_kernel_launches", "lwm_attn_fwd_noalloc",
                "lwm_attn_decode_workspace_size", "lwm_attn_decode", "lwm_attn_selftest_wait",
                "lwm_rope_apply_at", "lwm_attn_merge", "lwm_accumulate", "lwm_convert_f32",
                "lwm_attn_fwd_pair", "lwm_attn_bwd_pair", "lwm_packed_ce_workspace_size",
                "lwm_packed_cross_entropy", "lwm_attn_fwd_noalloc_read_status",
                "lwm_attn_fwd_pair_f32", "lwm_attn_bwd_pair_f32")
DECODE_MAX_NEW = 16


class LwmAttnDesc(ctypes.Structure):
    """Mirror of lwm_attn_desc in include/lwm_attn.h."""
    _fields_ = [
        ("batch", ctypes.c_int64),
        ("seqlen", ctypes.c_int64),
        ("heads", ctypes.c_int64),
        ("head_dim", ctypes.c_int64),
        ("dtype", ctypes.c_int32),
        ("causal", ctypes.c_int32),
        ("rope_theta", ctypes.c_double),
        ("softmax_scale", ctypes.c_float),
        ("segment_ids", ctypes.c_void_p),
    ]


class LwmError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({lwm_status_string(status)})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m long_context_causal_attention_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    lib.lwm_attn_workspace_size.argtypes = [ctypes.POINTER(LwmAttnDesc), ctypes.c_int]
    lib.lwm_attn_workspace_size.restype = ctypes.c_size_t
    lib.lwm_attn_fwd.argtypes = [ctypes.POINTER(LwmAttnDesc), P, P, P, P, P, P, ctypes.c_size_t, P]
    lib.lwm_attn_fwd.restype = ctypes.c_int
    lib.lwm_attn_bwd.argtypes = [ctypes.POINTER(LwmAttnDesc), P, P, P, P, P, P, P, P, P, P,
                                 ctypes.c_size_t, P]
    lib.lwm_attn_bwd.restype = ctypes.c_int
    lib.lwm_rope_apply.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_int32, ctypes.c_double, P, P, ctypes.c_int, P]
    lib.lwm_rope_apply.restype = ctypes.c_int
    lib.lwm_attn_read_status.argtypes = [P, P]
    lib.lwm_attn_read_status.restype = ctypes.c_int
    lib.lwm_status_string.argtypes = [ctypes.c_int]
    lib.lwm_status_string.restype = ctypes.c_char_p
    lib.lwm_attn_set_timing_events.argtypes = [P, P, P, P, P]
    lib.lwm_attn_set_timing_events.restype = None
    lib.lwm_attn_fwd_noalloc.argtypes = [ctypes.POINTER(LwmAttnDesc), P, P, P, P, P, P]
    lib.lwm_attn_fwd_noalloc.restype = ctypes.c_int
    lib.lwm_attn_fwd_noalloc_read_status.argtypes = [P]
    lib.lwm_attn_fwd_noalloc_read_status.restype = ctypes.c_int
    lib.lwm_attn_decode_workspace_size.argtypes = [ctypes.POINTER(LwmAttnDesc), ctypes.c_int64]
    lib.lwm_attn_decode_workspace_size.restype = ctypes.c_size_t
    lib.lwm_attn_decode.argtypes = [ctypes.POINTER(LwmAttnDesc), ctypes.c_int64, P, P, P, P, P, P,
                                    ctypes.c_size_t, P]
    lib.lwm_attn_decode.restype = ctypes.c_int
    lib.lwm_attn_selftest_wait.argtypes = [P, ctypes.c_size_t, ctypes.c_int64, ctypes.c_int, P]
    lib.lwm_attn_selftest_wait.restype = ctypes.c_int
    lib.lwm_packed_ce_workspace_size.argtypes = [ctypes.c_int64, ctypes.c_int64]
    lib.lwm_packed_ce_workspace_size.restype = ctypes.c_size_t
    lib.lwm_packed_cross_entropy.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                             ctypes.c_int32, P, P, P, P, P, P, ctypes.c_size_t, P]
    lib.lwm_packed_cross_entropy.restype = ctypes.c_int
    lib.lwm_attn_fwd_pair.argtypes = [ctypes.POINTER(LwmAttnDesc), P, P, P, P, P, P, P,
                                      ctypes.c_size_t, P]
    lib.lwm_attn_fwd_pair.restype = ctypes.c_int
    lib.lwm_attn_bwd_pair.argtypes = [ctypes.POINTER(LwmAttnDesc), P, P, P, P, P, P, P, P, P, P,
                                      P, ctypes.c_size_t, P]
    lib.lwm_attn_bwd_pair.restype = ctypes.c_int
    lib.lwm_attn_fwd_pair_f32.argtypes = lib.lwm_attn_fwd_pair.argtypes
    lib.lwm_attn_fwd_pair_f32.restype = ctypes.c_int
    lib.lwm_attn_bwd_pair_f32.argtypes = lib.lwm_attn_bwd_pair.argtypes
    lib.lwm_attn_bwd_pair_f32.restype = ctypes.c_int
    lib.lwm_rope_apply_at.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_int64, ctypes.c_int32, ctypes.c_double,
                                      ctypes.c_int64, P, P, ctypes.c_int, P]
    lib.lwm_rope_apply_at.restype = ctypes.c_int
    lib.lwm_attn_merge.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_int32, P, P, P, P, P]
    lib.lwm_attn_merge.restype = ctypes.c_int
    lib.lwm_accumulate.argtypes = [ctypes.c_int64, ctypes.c_int32, P, P, P]
    lib.lwm_accumulate.restype = ctypes.c_int
    lib.lwm_convert_f32.argtypes = [ctypes.c_int64, ctypes.c_int32, P, P, P]
    lib.lwm_convert_f32.restype = ctypes.c_int
    lib.lwm_attn_kernel_launches.argtypes = []
    lib.lwm_attn_kernel_launches.restype = ctypes.c_uint64
    return lib


_lib = _load()


def lib():
    return _lib


def lwm_status_string(status: int) -> str:
    return _lib.lwm_status_string(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return LWM_DTYPE_BF16
    if t.dtype == torch.float32:
        return LWM_DTYPE_FP32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


def _cuda(t: torch.Tensor, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def make_desc(q: torch.Tensor, segment_ids=None, causal=True, rope_theta=1e4,
              softmax_scale=0.0) -> LwmAttnDesc:
    if q.dim() != 4:
        raise ValueError("q must be [B, S, H, D]")
    B, S, H, D = q.shape
    seg_ptr = None
    if segment_ids is not None:
        _cuda(segment_ids, "segment_ids")
        if segment_ids.dtype != torch.int32 or tuple(segment_ids.shape) != (B, S):
            raise ValueError("segment_ids must be int32 [B, S]")
        seg_ptr = segment_ids.data_ptr()
    return LwmAttnDesc(B, S, H, D, _dtype_code(q), 1 if causal else 0, float(rope_theta),
                       float(softmax_scale), seg_ptr)


def lwm_attn_workspace_size(desc: LwmAttnDesc, is_bwd: bool) -> int:
    return int(_lib.lwm_attn_workspace_size(ctypes.byref(desc), 1 if is_bwd else 0))


def alloc_workspace(desc: LwmAttnDesc, is_bwd: bool, device) -> torch.Tensor:
    n = lwm_attn_workspace_size(desc, is_bwd)
    if n == 0:
        raise LwmError(-1, "lwm_attn_workspace_size")
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(n, dtype=torch.uint8, device=device)


def _check(status: int, what: str):
    if status != LWM_OK:
        raise LwmError(status, what)


def lwm_attn_fwd(q, k, v, segment_ids=None, causal=True, rope_theta=1e4, softmax_scale=0.0,
                 o=None, lse=None, workspace=None, stream=None, check_status=False):
    """O [B,S,H,D] and LSE [B,H,S] fp32 for un-rotated q, k, v (see lwm_attn.h).

    check_status: wait for the stream and raise if a kernel reported a
    device-side error (a bounded wait that ran out) in the status word."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        _cuda(t, name)
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError(f"{name} must match q in shape and dtype")
    desc = make_desc(q, segment_ids, causal, rope_theta, softmax_scale)
    B, S, H, D = q.shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(desc, False, q.device)
    st = _lib.lwm_attn_fwd(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                           o.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                           workspace.numel(), _stream(stream))
    _check(st, "lwm_attn_fwd")
    if check_status:
        _check(lwm_attn_read_status(workspace, stream), "lwm_attn_fwd (device status)")
    return o, lse


def lwm_attn_bwd(q, k, v, o, lse, d_o, segment_ids=None, causal=True, rope_theta=1e4,
                 softmax_scale=0.0, dq=None, dk=None, dv=None, workspace=None, stream=None,
                 check_status=False):
    """dq, dk, dv (gradients w.r.t. the un-rotated inputs) of sum(O * dO)."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("d_o", d_o)):
        _cuda(t, name)
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError(f"{name} must match q in shape and dtype")
    _cuda(lse, "lse")
    desc = make_desc(q, segment_ids, causal, rope_theta, softmax_scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    if workspace is None:
        workspace = alloc_workspace(desc, True, q.device)
    st = _lib.lwm_attn_bwd(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                           o.data_ptr(), lse.data_ptr(), d_o.data_ptr(), dq.data_ptr(),
                           dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(), workspace.numel(),
                           _stream(stream))
    _check(st, "lwm_attn_bwd")
    if check_status:
        _check(lwm_attn_read_status(workspace, stream), "lwm_attn_bwd (device status)")
    return dq, dk, dv


def lwm_attn_decode_workspace_size(desc: LwmAttnDesc, n_new: int) -> int:
    return int(_lib.lwm_attn_decode_workspace_size(ctypes.byref(desc), int(n_new)))


def lwm_attn_decode(q_new, k_cache, v_cache, segment_ids=None, causal=True, rope_theta=1e4,
                    softmax_scale=0.0, o=None, lse=None, workspace=None, stream=None,
                    check_status=False):
    """o [B,T,H,D] and lse [B,H,T] for T new un-rotated queries against a cache
    of S rotated keys and values (the new tokens are its last T entries)."""
    _cuda(q_new, "q_new")
    for name, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        _cuda(t, name)
        if t.shape != k_cache.shape or t.dtype != q_new.dtype:
            raise ValueError(f"{name} must be [B, S, H, D] of q_new's dtype")
    B, T, H, D = q_new.shape
    if k_cache.dim() != 4 or k_cache.shape[0] != B or k_cache.shape[2:] != q_new.shape[2:]:
        raise ValueError("k_cache must be [B, S, H, D] with q_new's B, H, D")
    desc = make_desc(k_cache, segment_ids, causal, rope_theta, softmax_scale)
    if o is None:
        o = torch.empty_like(q_new)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q_new.device)
    if workspace is None:
        n = lwm_attn_decode_workspace_size(desc, T)
        if n == 0:
            raise LwmError(-1, "lwm_attn_decode_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=q_new.device)
    st = _lib.lwm_attn_decode(ctypes.byref(desc), T, q_new.data_ptr(), k_cache.data_ptr(),
                              v_cache.data_ptr(), o.data_ptr(), lse.data_ptr(),
                              workspace.data_ptr(), workspace.numel(), _stream(stream))
    _check(st, "lwm_attn_decode")
    if check_status:
        _check(lwm_attn_read_status(workspace, stream), "lwm_attn_decode (device status)")
    return o, lse


def _kseg_ptr(k_segment_ids, q):
    if k_segment_ids is None:
        return None
    _cuda(k_segment_ids, "k_segment_ids")
    if k_segment_ids.dtype != torch.int32 or tuple(k_segment_ids.shape) != tuple(q.shape[:2]):
        raise ValueError("k_segment_ids must be int32 [B, S]")
    return k_segment_ids.data_ptr()


def lwm_attn_fwd_pair(q, k, v, segment_ids, k_segment_ids, causal=True, rope_theta=1e4,
                      softmax_scale=0.0, o=None, lse=None, workspace=None, stream=None):
    """lwm_attn_fwd for a block pair: query ids ``segment_ids``, key ids
    ``k_segment_ids`` (both or neither)."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        _cuda(t, name)
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError(f"{name} must match q in shape and dtype")
    desc = make_desc(q, segment_ids, causal, rope_theta, softmax_scale)
    B, S, H, D = q.shape
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device) if lse is None else lse
    workspace = alloc_workspace(desc, False, q.device) if workspace is None else workspace
    _check(_lib.lwm_attn_fwd_pair(ctypes.byref(desc), _kseg_ptr(k_segment_ids, q), q.data_ptr(),
                                  k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                  workspace.data_ptr(), workspace.numel(), _stream(stream)),
           "lwm_attn_fwd_pair")
    return o, lse


def lwm_attn_bwd_pair(q, k, v, o, lse, d_o, segment_ids, k_segment_ids, causal=True,
                      rope_theta=1e4, softmax_scale=0.0, dq=None, dk=None, dv=None,
                      workspace=None, stream=None):
    """lwm_attn_bwd for a block pair (see lwm_attn_fwd_pair)."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("d_o", d_o)):
        _cuda(t, name)
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError(f"{name} must match q in shape and dtype")
    _cuda(lse, "lse")
    desc = make_desc(q, segment_ids, causal, rope_theta, softmax_scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    workspace = alloc_workspace(desc, True, q.device) if workspace is None else workspace
    _check(_lib.lwm_attn_bwd_pair(ctypes.byref(desc), _kseg_ptr(k_segment_ids, q), q.data_ptr(),
                                  k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                  d_o.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                  workspace.data_ptr(), workspace.numel(), _stream(stream)),
           "lwm_attn_bwd_pair")
    return dq, dk, dv


def lwm_attn_fwd_pair_f32(q, k, v, segment_ids, k_segment_ids, causal=True, rope_theta=1e4,
                          softmax_scale=0.0, workspace=None, stream=None):
    """lwm_attn_fwd_pair with an fp32 O whatever the input dtype (block
    partials of a ring, merged without a bf16 rounding)."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        _cuda(t, name)
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError(f"{name} must match q in shape and dtype")
    desc = make_desc(q, segment_ids, causal, rope_theta, softmax_scale)
    B, S, H, D = q.shape
    o = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    workspace = alloc_workspace(desc, False, q.device) if workspace is None else workspace
    _check(_lib.lwm_attn_fwd_pair_f32(ctypes.byref(desc), _kseg_ptr(k_segment_ids, q),
                                      q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                      lse.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                      _stream(stream)), "lwm_attn_fwd_pair_f32")
    return o, lse


def lwm_attn_bwd_pair_f32(q, k, v, o, lse, d_o, segment_ids, k_segment_ids, causal=True,
                          rope_theta=1e4, softmax_scale=0.0, workspace=None, stream=None):
    """lwm_attn_bwd_pair with fp32 dq, dk, dv whatever the input dtype."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("d_o", d_o)):
        _cuda(t, name)
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError(f"{name} must match q in shape and dtype")
    _cuda(lse, "lse")
    desc = make_desc(q, segment_ids, causal, rope_theta, softmax_scale)
    dq, dk, dv = (torch.empty(q.shape, dtype=torch.float32, device=q.device) for _ in range(3))
    workspace = alloc_workspace(desc, True, q.device) if workspace is None else workspace
    _check(_lib.lwm_attn_bwd_pair_f32(ctypes.byref(desc), _kseg_ptr(k_segment_ids, q),
                                      q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                      lse.data_ptr(), d_o.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                      dv.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                      _stream(stream)), "lwm_attn_bwd_pair_f32")
    return dq, dk, dv


def lwm_rope_apply(x, theta, inverse=False, out=None, stream=None):
    """y = R(p) x (or R(p)^T x) for x [B,S,H,D]; out may be x (in place)."""
    _cuda(x, "x")
    if x.dim() != 4:
        raise ValueError("x must be [B, S, H, D]")
    out = torch.empty_like(x) if out is None else out
    B, S, H, D = x.shape
    st = _lib.lwm_rope_apply(B, S, H, D, _dtype_code(x), float(theta), x.data_ptr(),
                             out.data_ptr(), 1 if inverse else 0, _stream(stream))
    _check(st, "lwm_rope_apply")
    return out


def lwm_attn_read_status(workspace, stream=None) -> int:
    return int(_lib.lwm_attn_read_status(workspace.data_ptr(), _stream(stream)))


def lwm_attn_set_timing_events(fwd_start=None, fwd_stop=None, bwd_start=None, bwd_stop=None,
                               bwd_split=None):
    """Have the next calls record these torch.cuda.Event objects around their
    main attention kernels, bwd_split between the two backward kernels (None
    leaves that slot empty)."""
    def handle(e):
        if e is None:
            return None
        if not e.cuda_event:  # torch creates the CUDA event on first record
            e.record()
        return ctypes.c_void_p(e.cuda_event)
    _lib.lwm_attn_set_timing_events(handle(fwd_start), handle(fwd_stop), handle(bwd_start),
                                    handle(bwd_stop), handle(bwd_split))


def lwm_attn_selftest_wait(workspace, limit_cycles: int, arrive: bool, stream=None) -> int:
    """Run the bounded-wait self-test; returns the device status it leaves."""
    _check(_lib.lwm_attn_selftest_wait(workspace.data_ptr(), workspace.numel(), int(limit_cycles),
                                       1 if arrive else 0, _stream(stream)),
           "lwm_attn_selftest_wait")
    return lwm_attn_read_status(workspace, stream)


def lwm_attn_kernel_launches() -> int:
    return int(_lib.lwm_attn_kernel_launches())


def lwm_rope_apply_at(x, theta, position_offset, inverse=False, out=None, stream=None):
    """lwm_rope_apply with positions starting at ``position_offset``."""
    _cuda(x, "x")
    if x.dim() != 4:
        raise ValueError("x must be [B, S, H, D]")
    out = torch.empty_like(x) if out is None else out
    B, S, H, D = x.shape
    _check(_lib.lwm_rope_apply_at(B, S, H, D, _dtype_code(x), float(theta), int(position_offset),
                                  x.data_ptr(), out.data_ptr(), 1 if inverse else 0,
                                  _stream(stream)), "lwm_rope_apply_at")
    return out


def lwm_attn_merge(o_acc, lse_acc, o_part, lse_part, stream=None):
    """In place: (o_acc, lse_acc) <- log-sum-exp merge with (o_part, lse_part)."""
    for name, t in (("o_acc", o_acc), ("lse_acc", lse_acc), ("o_part", o_part),
                    ("lse_part", lse_part)):
        _cuda(t, name)
    if o_acc.dtype != torch.float32 or lse_acc.dtype != torch.float32:
        raise TypeError("o_acc and lse_acc must be float32")
    if o_part.shape != o_acc.shape or lse_part.shape != lse_acc.shape:
        raise ValueError("partial result must match the accumulator's shapes")
    B, S, H, D = o_acc.shape
    _check(_lib.lwm_attn_merge(B, S, H, D, _dtype_code(o_part), o_acc.data_ptr(),
                               lse_acc.data_ptr(), o_part.data_ptr(), lse_part.data_ptr(),
                               _stream(stream)), "lwm_attn_merge")


def lwm_accumulate(acc, x, stream=None):
    """In place: acc (float32) += x."""
    _cuda(acc, "acc")
    _cuda(x, "x")
    if acc.dtype != torch.float32 or acc.shape != x.shape:
        raise ValueError("acc must be float32 with x's shape")
    _check(_lib.lwm_accumulate(x.numel(), _dtype_code(x), acc.data_ptr(), x.data_ptr(),
                               _stream(stream)), "lwm_accumulate")


def lwm_convert_f32(x, dtype, out=None, stream=None):
    """x (float32) rounded to ``dtype`` (bfloat16 or float32)."""
    _cuda(x, "x")
    out = torch.empty(x.shape, dtype=dtype, device=x.device) if out is None else out
    _check(_lib.lwm_convert_f32(x.numel(), _dtype_code(out), x.data_ptr(), out.data_ptr(),
                                _stream(stream)), "lwm_convert_f32")
    return out


def lwm_packed_cross_entropy(logits, targets, segment_ids=None, with_grad=True, stream=None,
                             check_status=False):
    """(loss [1] float32 on the device, dlogits or None) of a packed batch with
    per-sample re-weighting; logits [B, S, V], targets / segment_ids int32 [B, S].
    check_status=True reads the kernel's status word after the call (a sync)."""
    _cuda(logits, "logits")
    _cuda(targets, "targets")
    if logits.dim() != 3:
        raise ValueError("logits must be [B, S, V]")
    B, S, V = logits.shape
    if targets.dtype != torch.int32 or tuple(targets.shape) != (B, S):
        raise ValueError("targets must be int32 [B, S]")
    seg_ptr = None
    if segment_ids is not None:
        _cuda(segment_ids, "segment_ids")
        if segment_ids.dtype != torch.int32 or tuple(segment_ids.shape) != (B, S):
            raise ValueError("segment_ids must be int32 [B, S]")
        seg_ptr = segment_ids.data_ptr()
    loss = torch.empty(1, dtype=torch.float32, device=logits.device)
    d = torch.empty_like(logits) if with_grad else None
    ws = torch.empty(int(_lib.lwm_packed_ce_workspace_size(B, S)), dtype=torch.uint8,
                     device=logits.device)
    _check(_lib.lwm_packed_cross_entropy(B, S, V, _dtype_code(logits), logits.data_ptr(),
                                         targets.data_ptr(), seg_ptr, loss.data_ptr(),
                                         d.data_ptr() if d is not None else None, ws.data_ptr(),
                                         ws.numel(), _stream(stream)), "lwm_packed_cross_entropy")
    if check_status:
        _check(lwm_attn_read_status(ws, stream), "lwm_packed_cross_entropy (device status)")
    return loss, d
