"""Ring Attention exact forward (and backward) on NVIDIA B200 (sm_100a).

A thin ctypes binding over the C ABI of ``include/ra.h`` (``libra_b200.so``, built in-tree by
``python -m long_context_exact_forward_b200._build``).  Every step of the computation runs in the
library's CUDA kernels; this module only checks tensor properties and marshals pointers.  PyTorch
provides device memory and streams.  There is no fallback: if the library is missing or the
device is not a CUDA device the calls raise.

Entry points (same names as the C ABI):
    forward(q, k, v, n_ring, causal, layout, ...)   -> (out, lse)      ra_forward_ex
    forward_noalloc(q, k, v, n_ring, causal, layout) -> (out, lse)      ra_forward_noalloc
    forward_varlen(q, k, v, cu_seqlens, n_ring, ...) -> (out, lse)      ra_forward_varlen_ex
    varlen_workspace_size(cu_seqlens, H, D, ...)     -> int             ra_varlen_workspace_size
    backward(q, k, v, out, lse, dout, n_ring, ...)   -> (dq, dk, dv)    ra_backward_ex
    rope(x, pos_offset, base)                        -> tensor          ra_rope
    ring_step(q_i, k_j, v_j, O_acc, lse_acc, ...)                        ra_ring_step
    ring_step_workspace_size(...)                    -> int             ra_ring_step_workspace_size
    ring_finalize(O_acc, lse_acc)                    -> (out, lse)      ra_ring_finalize
    workspace_size(...)                              -> int             ra_workspace_size
    permute(x, n_ring, layout) / unpermute(...)      -> tensor          ra_permute / ra_unpermute
    merge_partials(O_run, lse_run, O_step, lse_step)                     ra_merge_partials
    layout_positions(S, n_ring, layout)              -> np.ndarray      ra_layout_positions
    plan_tiles(S, n_ring, layout, causal, tile)      -> np.ndarray      ra_plan_tiles
    plan_items(B, H, S, n_ring, causal, layout, D)   -> np.ndarray      ra_plan_items
    get_device_status()                              -> int             ra_get_device_status
"""
import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# RA_LIB may name another build of the same library (for example one compiled with different
# tuning constants); by default the in-tree build is used.
LIB_PATH = os.environ.get("RA_LIB") or os.path.join(_HERE, "libra_b200.so")

LAYOUTS = {"contiguous": 0, "striped": 1, "zigzag": 2}
VARIANTS = {"auto": 0, "fused": 1, "per_step": 2}
KERNELS = {"auto": 0, "tc": 1, "simt": 2}
DEBUG_STALL_LOADS = 1
DEBUG_FROZEN_MAX = 2   # score-bound pre-pass and frozen row max at any size (tests)

RA_OK = 0
STATUS = {
    0: "RA_OK", -1: "RA_ERR_INVALID_ARG", -2: "RA_ERR_SHAPE", -3: "RA_ERR_ALIGN",
    -4: "RA_ERR_UNSUPPORTED", -5: "RA_ERR_NO_WORKSPACE", -6: "RA_ERR_CUDA",
    -7: "RA_ERR_DEVICE_TIMEOUT",
}


class RAError(RuntimeError):
    def __init__(self, code, where, detail=""):
        self.code = code
        name = STATUS.get(code, str(code))
        super().__init__(f"{where} failed: {name}" + (f" ({detail})" if detail else ""))


class Options(ctypes.Structure):
    _fields_ = [
        ("variant", ctypes.c_int),
        ("kernel", ctypes.c_int),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("timeout_ns", ctypes.c_uint64),
        ("debug", ctypes.c_int),
        ("attn_events", ctypes.c_void_p * 2),
        ("steps_per_launch", ctypes.c_int),
    ]


_lib = None


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m long_context_exact_forward_b200._build`")
        L = ctypes.CDLL(LIB_PATH)
        i64, vp, ci = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
        L.ra_forward.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, ci, ci, ci, ci, vp]
        L.ra_forward_ex.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, ci, ci, ci, ci, vp,
                                    ctypes.POINTER(Options)]
        L.ra_workspace_size.argtypes = [i64, i64, i64, i64, ci, ci, ci, ci, ci, ci,
                                        ctypes.POINTER(ctypes.c_size_t)]
        L.ra_permute.argtypes = [vp, vp, i64, i64, i64, i64, ci, ci, ci, vp]
        L.ra_unpermute.argtypes = [vp, vp, i64, i64, i64, i64, ci, ci, ci, vp]
        L.ra_merge_partials.argtypes = [vp, vp, vp, vp, i64, i64, vp]
        L.ra_forward_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, ci, ci, ci, vp]
        L.ra_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, ci, ci, ci,
                                  ci, vp]
        L.ra_forward_varlen.argtypes = [vp, vp, vp, vp, vp, vp, ci, i64, i64, ci, ci, ci, ci, vp]
        L.ra_forward_varlen_ex.argtypes = [vp, vp, vp, vp, vp, vp, ci, i64, i64, ci, ci, ci, ci, vp,
                                           ctypes.POINTER(Options)]
        L.ra_varlen_workspace_size.argtypes = [vp, ci, i64, i64, ci, ci, ci, ci, ci,
                                               ctypes.POINTER(ctypes.c_size_t)]
        L.ra_rope.argtypes = [vp, vp, i64, i64, i64, i64, i64, ctypes.c_double, ci, vp]
        L.ra_backward_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, ci, ci, ci,
                                     ci, ci, ctypes.c_uint64, ci, vp]
        L.ra_ring_step.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, ci, ci, ci, ci, ci, ci, ci, vp,
                                   ctypes.c_size_t, vp]
        L.ra_ring_step_workspace_size.argtypes = [i64, i64, i64, i64, ci, ci, ci, ci,
                                                  ctypes.POINTER(ctypes.c_size_t)]
        L.ra_ring_finalize.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, ci, vp]
        L.ra_steps_per_launch.argtypes = [i64, i64, ci, ci, ci, ci, ci, ctypes.POINTER(ctypes.c_int)]
        L.ra_layout_positions.argtypes = [i64, ci, ci, vp]
        L.ra_plan_tiles.argtypes = [i64, ci, ci, ci, ci, vp]
        L.ra_plan_items.argtypes = [i64, i64, i64, i64, ci, ci, ci, vp, i64, ctypes.POINTER(ctypes.c_int64)]
        L.ra_status_string.restype = ctypes.c_char_p
        L.ra_status_string.argtypes = [ci]
        L.ra_last_error_string.restype = ctypes.c_char_p
        L.ra_last_error_string.argtypes = []
        L.ra_get_device_status.argtypes = []
        L.ra_clear_last_error.argtypes = []
        L.ra_clear_last_error.restype = None
        for name in ("ra_forward", "ra_forward_ex", "ra_forward_noalloc", "ra_workspace_size", "ra_permute",
                     "ra_unpermute", "ra_merge_partials", "ra_layout_positions", "ra_plan_tiles",
                     "ra_plan_items", "ra_get_device_status", "ra_backward", "ra_backward_ex", "ra_rope", "ra_forward_varlen",
                     "ra_forward_varlen_ex", "ra_varlen_workspace_size", "ra_ring_step",
                     "ra_ring_step_workspace_size", "ra_ring_finalize", "ra_steps_per_launch"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _last_error():
    return lib().ra_last_error_string().decode()


def _clear_error():
    """Empty the library's per-thread message before a call, so that whatever it holds after a
    failure was recorded by that call."""
    lib().ra_clear_last_error()


def _check(rc, where):
    """Raise RAError for a non-zero status, with the library's message when the call left one."""
    if rc != RA_OK:
        raise RAError(rc, where, _last_error())


def _check_out(t, shape, dtype, name, like=None):
    """A caller-supplied output tensor must match the shape and dtype the kernels write, live on
    the inputs' device and be contiguous; otherwise the kernels would write outside it."""
    _check_cuda(t)
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} {list(shape)}, got {t.dtype} {list(t.shape)}")
    if like is not None and t.device != like.device:
        raise ValueError(f"{name} must be on {like.device}")


def _torch():
    import torch
    return torch


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.float32:
        return 0
    if t.dtype == torch.bfloat16:
        return 1
    raise TypeError(f"dtype {t.dtype} not supported (float32 or bfloat16)")


def _stream_handle(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_cuda(*ts):
    """Every tensor of one call lives on the same CUDA device (the kernels run on that device and
    dereference every pointer there) and is contiguous."""
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if t.device != ts[0].device:
            raise ValueError(f"tensors of one call must share a device ({ts[0].device} and {t.device})")


def workspace_size(B, H, S, D, n_ring, causal, layout, dtype_code, variant="auto", kernel="auto"):
    n = ctypes.c_size_t(0)
    _clear_error()
    _check(lib().ra_workspace_size(B, H, S, D, n_ring, int(bool(causal)), LAYOUTS[layout],
                                   dtype_code, VARIANTS[variant], KERNELS[kernel], ctypes.byref(n)),
           "ra_workspace_size")
    return n.value


def forward(q, k, v, n_ring, causal=True, layout="contiguous", *, variant="auto", kernel="auto",
            out=None, lse=None, workspace=None, stream=None, events=None, timeout_ns=0, debug=0,
            steps_per_launch=0):
    """Exact attention of q, k, v ([B, S, H, D], CUDA, fp32 or bf16) over an n_ring virtual ring.

    Returns (out [B, S, H, D] in q's dtype, lse [B, H, S] fp32).  `workspace` is an optional
    uint8 CUDA tensor of at least workspace_size(...) bytes (otherwise the library allocates
    stream-ordered); `events` an optional pair of torch.cuda.Event recorded around the attention
    kernel launches on `stream`.  `steps_per_launch`: ring steps per attention launch of the
    per_step variant (0 = one).
    """
    torch = _torch()
    _check_cuda(q, k, v)
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must all be [B, S, H, D]")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share a dtype")
    B, S, H, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    _check_out(out, q.shape, q.dtype, "out", q)
    _check_out(lse, (B, H, S), torch.float32, "lse", q)
    opt = Options()
    opt.variant = VARIANTS[variant]
    opt.kernel = KERNELS[kernel]
    opt.steps_per_launch = int(steps_per_launch)
    if workspace is not None:
        _check_cuda(q, workspace)
        opt.workspace = workspace.data_ptr()
        opt.workspace_bytes = workspace.numel() * workspace.element_size()
    opt.timeout_ns = int(timeout_ns)
    opt.debug = int(debug)
    if events is not None:
        for ev in events:  # torch creates the CUDA event lazily, on first record
            if ev.cuda_event == 0:
                ev.record(stream if stream is not None else torch.cuda.current_stream())
        opt.attn_events[0] = events[0].cuda_event
        opt.attn_events[1] = events[1].cuda_event
    _clear_error()
    with torch.cuda.device(q.device):
        rc = lib().ra_forward_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 lse.data_ptr(), B, H, S, D, int(n_ring), int(bool(causal)),
                                 LAYOUTS[layout], _dtype_code(q), _stream_handle(stream),
                                 ctypes.byref(opt))
    _check(rc, "ra_forward_ex")
    return out, lse


def steps_per_launch(S, D, n_ring, layout, dtype_code, variant="auto", steps=0):
    """Ring steps each attention launch of forward() covers for these arguments (ra_steps_per_launch):
    n_ring means one fused launch."""
    n = ctypes.c_int(0)
    _clear_error()
    _check(lib().ra_steps_per_launch(S, D, int(n_ring), LAYOUTS[layout], dtype_code, VARIANTS[variant], int(steps),
                                     ctypes.byref(n)), "ra_steps_per_launch")
    return n.value


def forward_noalloc(q, k, v, n_ring, causal=True, layout="contiguous", *, out=None, lse=None,
                    stream=None):
    """ra_forward_noalloc: like forward() for bf16 inputs, but the library allocates nothing --
    its scratch is a fixed device array shared by all calls on the device (see include/ra.h)."""
    torch = _torch()
    _check_cuda(q, k, v)
    if q.dtype != torch.bfloat16 or k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("forward_noalloc takes bf16 q, k, v")
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must all be [B, S, H, D]")
    B, S, H, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    _check_out(out, q.shape, q.dtype, "out", q)
    _check_out(lse, (B, H, S), torch.float32, "lse", q)
    _clear_error()
    with torch.cuda.device(q.device):
        rc = lib().ra_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                      lse.data_ptr(), B, H, S, D, int(n_ring), int(bool(causal)),
                                      LAYOUTS[layout], _stream_handle(stream))
    _check(rc, "ra_forward_noalloc")
    return out, lse


def backward(q, k, v, out, lse, dout, n_ring, causal=True, layout="contiguous", *, kernel="auto", dq=None,
             dk=None, dv=None, stream=None, timeout_ns=0, debug=0):
    """ra_backward_ex: gradients (dq, dk, dv) of forward(q, k, v, n_ring, causal, layout) for the
    upstream gradient dout, recomputed block by block in ring order from the saved out and lse.
    kernel: "auto" (tensor cores for bf16 with D in {64, 128} and 16-byte aligned tensors, any layout --
    zigzag through shard-major copies -- else CUDA cores), "tc" or "simt".  All tensors [B, S, H, D] in
    q's dtype except lse."""
    torch = _torch()
    _check_cuda(q, k, v, out, lse, dout)
    if not (q.shape == k.shape == v.shape == out.shape == dout.shape) or q.dim() != 4:
        raise ValueError("q, k, v, out, dout must all be [B, S, H, D]")
    if not (q.dtype == k.dtype == v.dtype == out.dtype == dout.dtype):
        raise TypeError("q, k, v, out, dout must share a dtype")
    B, S, H, D = q.shape
    if lse.shape != (B, H, S) or lse.dtype != torch.float32:
        raise ValueError("lse must be float32 [B, H, S]")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        _check_out(g, q.shape, q.dtype, name, q)
    _clear_error()
    with torch.cuda.device(q.device):
        rc = lib().ra_backward_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                  dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, S, D,
                                  int(n_ring), int(bool(causal)), LAYOUTS[layout], _dtype_code(q),
                                  KERNELS[kernel], int(timeout_ns), int(debug), _stream_handle(stream))
    _check(rc, "ra_backward_ex")
    return dq, dk, dv


def _cu_array(cu_seqlens):
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    if cu.ndim != 1 or cu.size < 2:
        raise ValueError("cu_seqlens must hold n_seqs + 1 offsets")
    return cu


def varlen_workspace_size(cu_seqlens, H, D, n_ring, layout="contiguous", dtype_code=1, variant="auto",
                          kernel="auto"):
    """Bytes of scratch forward_varlen needs for these packed sequences (ra_varlen_workspace_size)."""
    cu = _cu_array(cu_seqlens)
    n = ctypes.c_size_t(0)
    _clear_error()
    _check(lib().ra_varlen_workspace_size(cu.ctypes.data, int(cu.size - 1), H, D, int(n_ring), LAYOUTS[layout],
                                          int(dtype_code), VARIANTS[variant], KERNELS[kernel], ctypes.byref(n)),
           "ra_varlen_workspace_size")
    return n.value


def forward_varlen(q, k, v, cu_seqlens, n_ring, causal=True, layout="contiguous", *, variant="auto",
                   kernel="auto", steps_per_launch=0, out=None, lse=None, workspace=None, stream=None,
                   events=None, timeout_ns=0, debug=0):
    """ra_forward_varlen_ex: attention over sequences packed on the token axis of q, k, v [S_total, H, D]
    (fp32 or bf16); cu_seqlens: n_seqs + 1 offsets (a host sequence of ints); layout "contiguous",
    "striped" or "zigzag" inside each sequence; variant "auto", "fused" or "per_step" (with
    `steps_per_launch` ring steps per launch); kernel "auto", "tc" or "simt".  Returns
    (out [S_total, H, D] in q's dtype, lse [H, S_total]).

    `workspace` is an optional uint8 CUDA tensor of at least varlen_workspace_size(...) bytes; without
    it the scratch comes from torch's caching allocator on the call's stream, so repeated calls do
    not allocate device memory anew.  `events`: an optional pair of torch.cuda.Event recorded around
    the attention launches."""
    torch = _torch()
    _check_cuda(q, k, v)
    if q.dim() != 3 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must all be [S_total, H, D]")
    dtype_code = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    S, H, D = q.shape
    cu = _cu_array(cu_seqlens)
    if cu[-1] != S:
        raise ValueError("cu_seqlens must end at S_total")
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((H, S), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_out(out, q.shape, q.dtype, "out", q)
    _check_out(lse, (H, S), torch.float32, "lse", q)
    if workspace is None:
        n = varlen_workspace_size(cu, H, D, n_ring, layout, dtype_code, variant, kernel)
        with torch.cuda.device(q.device):
            workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
        if stream is not None:  # the scratch must outlive the work enqueued on `stream`
            workspace.record_stream(stream)
    _check_cuda(q, workspace)
    opt = Options()
    opt.variant = VARIANTS[variant]
    opt.kernel = KERNELS[kernel]
    opt.steps_per_launch = int(steps_per_launch)
    opt.workspace = workspace.data_ptr()
    opt.workspace_bytes = workspace.numel() * workspace.element_size()
    opt.timeout_ns = int(timeout_ns)
    opt.debug = int(debug)
    if events is not None:
        for ev in events:  # torch creates the CUDA event lazily, on first record
            if ev.cuda_event == 0:
                ev.record(stream if stream is not None else torch.cuda.current_stream())
        opt.attn_events[0] = events[0].cuda_event
        opt.attn_events[1] = events[1].cuda_event
    _clear_error()
    with torch.cuda.device(q.device):
        rc = lib().ra_forward_varlen_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                        cu.ctypes.data, int(cu.size - 1), H, D, int(n_ring), int(bool(causal)),
                                        LAYOUTS[layout], dtype_code, _stream_handle(stream), ctypes.byref(opt))
    _check(rc, "ra_forward_varlen_ex")
    return out, lse


def rope(x, pos_offset=0, base=10000.0, out=None, stream=None):
    """ra_rope: rotary embedding of x [B, S, H, D] with global positions (token g at g + pos_offset);
    out may be x itself (in place)."""
    torch = _torch()
    _check_cuda(x)
    if x.dim() != 4:
        raise ValueError("x must be [B, S, H, D]")
    out = torch.empty_like(x) if out is None else out
    _check_out(out, x.shape, x.dtype, "out", x)
    B, S, H, D = x.shape
    _clear_error()
    with torch.cuda.device(x.device):
        rc = lib().ra_rope(x.data_ptr(), out.data_ptr(), B, S, H, D, int(pos_offset), float(base),
                           _dtype_code(x), _stream_handle(stream))
    _check(rc, "ra_rope")
    return out


def ring_step_workspace_size(B, H, S, D, n_ring, causal, layout, dtype_code):
    """Scratch bytes that suffice for ring_step at every (shard, step) of these arguments."""
    n = ctypes.c_size_t(0)
    _clear_error()
    _check(lib().ra_ring_step_workspace_size(B, H, S, D, int(n_ring), int(bool(causal)), LAYOUTS[layout],
                                             dtype_code, ctypes.byref(n)), "ra_ring_step_workspace_size")
    return n.value


def ring_step(q_i, k_j, v_j, O_acc, lse_acc, n_ring, shard, step, causal=True, layout="contiguous", *,
              sms_reserved=0, workspace=None, stream=None):
    """ra_ring_step: one ring step of query shard `shard` against the key/value block
    j = (shard - step) mod n_ring held in this device's own buffers.

    q_i, k_j, v_j: [B, S_loc, H, D] (fp32 or bf16) in the layout's local token order; O_acc fp32
    [B, S_loc, H, D] and lse_acc fp32 [B, S_loc, H] hold the running result (written at step 0,
    merged into afterwards).  `workspace`: an optional uint8 CUDA tensor of at least
    ring_step_workspace_size(...) bytes; without it the scratch comes from torch's caching
    allocator.  `sms_reserved`: SMs the tensor-core kernel leaves free for a concurrent transfer."""
    torch = _torch()
    _check_cuda(q_i, k_j, v_j, O_acc, lse_acc)
    if q_i.dim() != 4 or q_i.shape != k_j.shape or q_i.shape != v_j.shape:
        raise ValueError("q_i, k_j, v_j must all be [B, S_loc, H, D]")
    if not (q_i.dtype == k_j.dtype == v_j.dtype):
        raise TypeError("q_i, k_j, v_j must share a dtype")
    B, S_loc, H, D = q_i.shape
    _check_out(O_acc, q_i.shape, torch.float32, "O_acc", q_i)
    _check_out(lse_acc, (B, S_loc, H), torch.float32, "lse_acc", q_i)
    S = S_loc * int(n_ring)
    if workspace is None:
        n = ring_step_workspace_size(B, H, S, D, n_ring, causal, layout, _dtype_code(q_i))
        with torch.cuda.device(q_i.device):
            workspace = torch.empty(n, dtype=torch.uint8, device=q_i.device)
        if stream is not None:  # the scratch must outlive the work enqueued on `stream`
            workspace.record_stream(stream)
    _check_cuda(q_i, workspace)
    _clear_error()
    with torch.cuda.device(q_i.device):
        rc = lib().ra_ring_step(q_i.data_ptr(), k_j.data_ptr(), v_j.data_ptr(), O_acc.data_ptr(),
                                lse_acc.data_ptr(), B, H, S, D, int(n_ring), int(bool(causal)), LAYOUTS[layout],
                                _dtype_code(q_i), int(shard), int(step), int(sms_reserved), workspace.data_ptr(),
                                workspace.numel(), _stream_handle(stream))
    _check(rc, "ra_ring_step")
    return O_acc, lse_acc


def ring_finalize(O_acc, lse_acc, out=None, lse=None, dtype=None, stream=None):
    """ra_ring_finalize: the shard's result after its last ring step, out [B, S_loc, H, D] in `dtype`
    (default bf16) and lse [B, H, S_loc] fp32, in the shard's local token order."""
    torch = _torch()
    _check_cuda(O_acc, lse_acc)
    if O_acc.dim() != 4 or O_acc.dtype != torch.float32:
        raise ValueError("O_acc must be fp32 [B, S_loc, H, D]")
    B, S_loc, H, D = O_acc.shape
    _check_out(lse_acc, (B, S_loc, H), torch.float32, "lse_acc", O_acc)
    dtype = dtype or (out.dtype if out is not None else torch.bfloat16)
    out = torch.empty(O_acc.shape, dtype=dtype, device=O_acc.device) if out is None else out
    lse = torch.empty((B, H, S_loc), dtype=torch.float32, device=O_acc.device) if lse is None else lse
    _check_out(out, O_acc.shape, dtype, "out", O_acc)
    _check_out(lse, (B, H, S_loc), torch.float32, "lse", O_acc)
    _clear_error()
    with torch.cuda.device(O_acc.device):
        rc = lib().ra_ring_finalize(O_acc.data_ptr(), lse_acc.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H,
                                    S_loc, D, _dtype_code(out), _stream_handle(stream))
    _check(rc, "ra_ring_finalize")
    return out, lse


def permute(x, n_ring, layout, out=None, stream=None, inverse=False):
    """Natural order [B, S, H, D] -> shard-major [B, n_ring, S/n_ring, H, D] (or back)."""
    torch = _torch()
    _check_cuda(x)
    if x.dim() != (5 if inverse else 4) or int(n_ring) < 1:
        raise ValueError("permute takes x [B, S, H, D], unpermute [B, n_ring, S_loc, H, D]; n_ring >= 1")
    if inverse and x.shape[1] != n_ring:
        raise ValueError("unpermute: x.shape[1] must equal n_ring")
    B, S, H, D = (x.shape[0], x.shape[1] * x.shape[2], x.shape[3], x.shape[4]) if inverse else x.shape
    shape = (B, S, H, D) if inverse else (B, n_ring, S // n_ring, H, D)
    if out is None:
        out = torch.empty(shape, dtype=x.dtype, device=x.device)
    _check_out(out, shape, x.dtype, "out", x)
    fn = lib().ra_unpermute if inverse else lib().ra_permute
    _clear_error()
    with torch.cuda.device(x.device):
        rc = fn(x.data_ptr(), out.data_ptr(), B, S, H, D, int(n_ring), LAYOUTS[layout],
                _dtype_code(x), _stream_handle(stream))
    _check(rc, "ra_unpermute" if inverse else "ra_permute")
    return out


def unpermute(x, n_ring, layout, out=None, stream=None):
    return permute(x, n_ring, layout, out=out, stream=stream, inverse=True)


def merge_partials(O_run, lse_run, O_step, lse_step, stream=None):
    """In-place merge of a step's normalised partial (O_step, lse_step) into (O_run, lse_run)."""
    torch = _torch()
    _check_cuda(O_run, lse_run, O_step, lse_step)
    for t in (O_run, lse_run, O_step, lse_step):
        if t.dtype != torch.float32:
            raise TypeError("merge_partials works on fp32 tensors")
    D = O_run.shape[-1]
    rows = O_run.numel() // D
    if O_step.shape != O_run.shape or lse_run.numel() != rows or lse_step.numel() != rows:
        raise ValueError("O_step must match O_run, and lse_run, lse_step hold one value per row of O_run")
    _clear_error()
    with torch.cuda.device(O_run.device):
        rc = lib().ra_merge_partials(O_run.data_ptr(), lse_run.data_ptr(), O_step.data_ptr(),
                                     lse_step.data_ptr(), rows, D, _stream_handle(stream))
    _check(rc, "ra_merge_partials")
    return O_run, lse_run


def layout_positions(S, n_ring, layout):
    pos = np.empty(S, dtype=np.int64)
    _clear_error()
    _check(lib().ra_layout_positions(S, n_ring, LAYOUTS[layout], pos.ctypes.data),
           "ra_layout_positions")
    return pos.reshape(n_ring, S // n_ring)


def plan_tiles(S, n_ring, layout, causal, tile):
    if n_ring < 1 or tile < 1:
        raise ValueError("n_ring and tile must be >= 1")
    nt = -(-(S // n_ring) // tile)
    cls = np.empty((n_ring, n_ring, nt, nt), dtype=np.int8)
    _clear_error()
    _check(lib().ra_plan_tiles(S, n_ring, LAYOUTS[layout], int(bool(causal)), tile,
                               cls.ctypes.data), "ra_plan_tiles")
    return cls


def plan_items(B, H, S, n_ring, causal, layout, D=128):
    n = ctypes.c_int64(0)
    _clear_error()
    _check(lib().ra_plan_items(B, H, S, D, n_ring, int(bool(causal)), LAYOUTS[layout], None, 0,
                               ctypes.byref(n)), "ra_plan_items")
    items = np.empty((n.value, 5), dtype=np.int32)
    _check(lib().ra_plan_items(B, H, S, D, n_ring, int(bool(causal)), LAYOUTS[layout],
                               items.ctypes.data, n.value, ctypes.byref(n)), "ra_plan_items")
    return items


def get_device_status():
    return lib().ra_get_device_status()


def status_string(code):
    return lib().ra_status_string(code).decode()
