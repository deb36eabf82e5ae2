"""ctypes binding of the C ABI in ``include/xlstm_mlstm.h``.

The functions named ``xlstm_*`` mirror the C entry points one to one: they take
plain integers (device addresses) or objects with ``data_ptr()`` (torch tensors)
and return the status code.  ``fwd``/``step`` below only allocate outputs with
torch and marshal arguments; every arithmetic step runs in the CUDA library.
A missing library raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libxlstm_mlstm.so")

XLSTM_OK, XLSTM_ERR_INVALID_ARG, XLSTM_ERR_UNSUPPORTED = 0, 1, 2
XLSTM_ERR_CUDA, XLSTM_ERR_TIMEOUT, XLSTM_ERR_WORKSPACE = 3, 4, 5
XLSTM_F32, XLSTM_BF16 = 0, 1

EXPORTED = ("xlstm_mlstm_fwd_chunkwise", "xlstm_mlstm_fwd_recurrent", "xlstm_mlstm_step",
            "xlstm_mlstm_workspace_size", "xlstm_mlstm_workspace_status", "xlstm_status_string",
            "xlstm_mlstm_version", "xlstm_mlstm_chunkwise_kernel", "xlstm_mlstm_test_timeout_next",
            "xlstm_mlstm_fwd_chunkwise_noalloc", "xlstm_mlstm_workspace_size_parallel",
            "xlstm_mlstm_fwd_chunkwise_out", "xlstm_mlstm_noalloc_status", "xlstm_mlstm_segment_summary",
            "xlstm_mlstm_combine_states", "xlstm_mlstm_bwd_chunkwise", "xlstm_mlstm_bwd_workspace_size")


class xlstm_mlstm_desc_t(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("T", ctypes.c_int32),
                ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32), ("qkv_dtype", ctypes.c_int32),
                ("qk_scale", ctypes.c_float), ("chunk", ctypes.c_int32)]


class xlstm_mlstm_output_t(ctypes.Structure):
    _fields_ = [("o_pre", ctypes.c_void_p), ("o_dtype", ctypes.c_int32), ("h_dtype", ctypes.c_int32)]


class XlstmError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})" if what else status_string(status))


_lib = None


def load(path: str = LIB_PATH):
    """Open the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} (run python -m xlstm_mlstm_matrix_b200.build)")
    lib = ctypes.CDLL(path)
    vp, sz, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    dp = ctypes.POINTER(xlstm_mlstm_desc_t)
    seq = [dp] + [vp] * 12 + [vp, sz, vp]
    for name in ("xlstm_mlstm_fwd_chunkwise", "xlstm_mlstm_fwd_recurrent"):
        getattr(lib, name).argtypes = seq
        getattr(lib, name).restype = st
    lib.xlstm_mlstm_fwd_chunkwise_out.argtypes = [dp, ctypes.POINTER(xlstm_mlstm_output_t)] + [vp] * 12 + [vp, sz, vp]
    lib.xlstm_mlstm_fwd_chunkwise_out.restype = st
    lib.xlstm_mlstm_fwd_chunkwise_noalloc.argtypes = [dp] + [vp] * 12 + [vp]
    lib.xlstm_mlstm_fwd_chunkwise_noalloc.restype = st
    lib.xlstm_mlstm_step.argtypes = [dp] + [vp] * 12 + [vp]
    lib.xlstm_mlstm_step.restype = st
    lib.xlstm_mlstm_workspace_size.argtypes = [dp]
    lib.xlstm_mlstm_workspace_size.restype = sz
    lib.xlstm_mlstm_workspace_size_parallel.argtypes = [dp]
    lib.xlstm_mlstm_workspace_size_parallel.restype = sz
    lib.xlstm_mlstm_workspace_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int32), vp]
    lib.xlstm_mlstm_workspace_status.restype = st
    lib.xlstm_mlstm_noalloc_status.argtypes = [ctypes.POINTER(ctypes.c_int32), vp]
    lib.xlstm_mlstm_noalloc_status.restype = st
    lib.xlstm_mlstm_segment_summary.argtypes = [dp] + [vp] * 7 + [vp, sz, vp]
    lib.xlstm_mlstm_segment_summary.restype = st
    lib.xlstm_mlstm_combine_states.argtypes = [dp, ctypes.c_int32] + [vp] * 9 + [vp]
    lib.xlstm_mlstm_combine_states.restype = st
    lib.xlstm_mlstm_bwd_chunkwise.argtypes = [dp] + [vp] * 19 + [vp, sz, vp]
    lib.xlstm_mlstm_bwd_chunkwise.restype = st
    lib.xlstm_mlstm_bwd_workspace_size.argtypes = [dp]
    lib.xlstm_mlstm_bwd_workspace_size.restype = sz
    lib.xlstm_status_string.argtypes = [st]
    lib.xlstm_status_string.restype = ctypes.c_char_p
    lib.xlstm_mlstm_version.argtypes = []
    lib.xlstm_mlstm_version.restype = ctypes.c_char_p
    lib.xlstm_mlstm_chunkwise_kernel.argtypes = [dp]
    lib.xlstm_mlstm_chunkwise_kernel.restype = ctypes.c_char_p
    lib.xlstm_mlstm_test_timeout_next.argtypes = [ctypes.c_int32]
    lib.xlstm_mlstm_test_timeout_next.restype = None
    if path == LIB_PATH:
        _lib = lib
    return lib


def _p(x):
    if x is None:
        return None
    if isinstance(x, int):
        return ctypes.c_void_p(x)
    if hasattr(x, "data_ptr"):
        return ctypes.c_void_p(x.data_ptr())
    raise TypeError(f"expected a device address or tensor, got {type(x)}")


def _s(stream):
    if stream is None:
        return None
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def make_desc(B, H, T, d_qk, d_v, dtype=XLSTM_BF16, qk_scale=1.0, chunk=0) -> xlstm_mlstm_desc_t:
    return xlstm_mlstm_desc_t(B, H, T, d_qk, d_v, dtype, qk_scale, chunk)


# ---- one-to-one C entry points -----------------------------------------------
def xlstm_mlstm_fwd_chunkwise(desc, q, k, v, i_pre, f_pre, C_in, n_in, m_in, h_out, C_out,
                              n_out, m_out, workspace, workspace_bytes, stream=None) -> int:
    return load().xlstm_mlstm_fwd_chunkwise(
        ctypes.byref(desc), _p(q), _p(k), _p(v), _p(i_pre), _p(f_pre), _p(C_in), _p(n_in),
        _p(m_in), _p(h_out), _p(C_out), _p(n_out), _p(m_out), _p(workspace), workspace_bytes,
        _s(stream))


def xlstm_mlstm_fwd_chunkwise_noalloc(desc, q, k, v, i_pre, f_pre, C_in, n_in, m_in, h_out, C_out,
                                      n_out, m_out, stream=None) -> int:
    """Chunkwise forward using the library's fixed scratch array instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    return load().xlstm_mlstm_fwd_chunkwise_noalloc(
        ctypes.byref(desc), _p(q), _p(k), _p(v), _p(i_pre), _p(f_pre), _p(C_in), _p(n_in),
        _p(m_in), _p(h_out), _p(C_out), _p(n_out), _p(m_out), _s(stream))


def xlstm_mlstm_fwd_recurrent(desc, q, k, v, i_pre, f_pre, C_in, n_in, m_in, h_out, C_out,
                              n_out, m_out, workspace=None, workspace_bytes=0, stream=None) -> int:
    return load().xlstm_mlstm_fwd_recurrent(
        ctypes.byref(desc), _p(q), _p(k), _p(v), _p(i_pre), _p(f_pre), _p(C_in), _p(n_in),
        _p(m_in), _p(h_out), _p(C_out), _p(n_out), _p(m_out), _p(workspace), workspace_bytes,
        _s(stream))


def xlstm_mlstm_fwd_chunkwise_out(desc, out, q, k, v, i_pre, f_pre, C_in, n_in, m_in, h_out, C_out,
                                  n_out, m_out, workspace, workspace_bytes, stream=None) -> int:
    """out: an xlstm_mlstm_output_t or None."""
    return load().xlstm_mlstm_fwd_chunkwise_out(
        ctypes.byref(desc), None if out is None else ctypes.byref(out), _p(q), _p(k), _p(v), _p(i_pre),
        _p(f_pre), _p(C_in), _p(n_in), _p(m_in), _p(h_out), _p(C_out), _p(n_out), _p(m_out), _p(workspace),
        int(workspace_bytes), _s(stream))


def xlstm_mlstm_step(desc, q, k, v, i_pre, f_pre, C, n, m, h_out, C_new, n_new, m_new,
                     stream=None) -> int:
    return load().xlstm_mlstm_step(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(i_pre), _p(f_pre),
                                   _p(C), _p(n), _p(m), _p(h_out), _p(C_new), _p(n_new),
                                   _p(m_new), _s(stream))


def xlstm_mlstm_segment_summary(desc, k, v, i_pre, f_pre, C_seg, n_seg, F_m, workspace, workspace_bytes,
                                stream=None) -> int:
    return load().xlstm_mlstm_segment_summary(ctypes.byref(desc), _p(k), _p(v), _p(i_pre), _p(f_pre), _p(C_seg),
                                               _p(n_seg), _p(F_m), _p(workspace), int(workspace_bytes), _s(stream))


def xlstm_mlstm_combine_states(desc, nsum, C_in, n_in, m_in, C_seg, n_seg, F_m, C_out, n_out, m_out,
                               stream=None) -> int:
    return load().xlstm_mlstm_combine_states(ctypes.byref(desc), int(nsum), _p(C_in), _p(n_in), _p(m_in),
                                              _p(C_seg), _p(n_seg), _p(F_m), _p(C_out), _p(n_out), _p(m_out),
                                              _s(stream))


def xlstm_mlstm_bwd_chunkwise(desc, q, k, v, i_pre, f_pre, C_in, n_in, m_in, dh, dC_out, dn_out, dq, dk, dv,
                              di_pre, df_pre, dC_in, dn_in, dm_in, workspace, workspace_bytes, stream=None) -> int:
    return load().xlstm_mlstm_bwd_chunkwise(
        ctypes.byref(desc), *(_p(x) for x in (q, k, v, i_pre, f_pre, C_in, n_in, m_in, dh, dC_out, dn_out,
                                              dq, dk, dv, di_pre, df_pre, dC_in, dn_in, dm_in, workspace)),
        int(workspace_bytes), _s(stream))


def xlstm_mlstm_bwd_workspace_size(desc) -> int:
    return int(load().xlstm_mlstm_bwd_workspace_size(ctypes.byref(desc)))


def xlstm_mlstm_workspace_size(desc) -> int:
    return int(load().xlstm_mlstm_workspace_size(ctypes.byref(desc)))


def xlstm_mlstm_workspace_size_parallel(desc) -> int:
    return int(load().xlstm_mlstm_workspace_size_parallel(ctypes.byref(desc)))


def xlstm_mlstm_workspace_status(workspace, stream=None):
    where = ctypes.c_int32(0)
    st = load().xlstm_mlstm_workspace_status(_p(workspace), ctypes.byref(where), _s(stream))
    return int(st), int(where.value)


def xlstm_mlstm_noalloc_status(stream=None):
    """(code, where) of the status block used by the last allocation-free call."""
    where = ctypes.c_int32(0)
    st = load().xlstm_mlstm_noalloc_status(ctypes.byref(where), _s(stream))
    return int(st), int(where.value)


def xlstm_status_string(status: int) -> str:
    return load().xlstm_status_string(int(status)).decode()


def xlstm_mlstm_version() -> str:
    return load().xlstm_mlstm_version().decode()


def xlstm_mlstm_chunkwise_kernel(desc) -> str:
    return load().xlstm_mlstm_chunkwise_kernel(ctypes.byref(desc)).decode()


def xlstm_mlstm_test_timeout_next(enable: int = 1) -> None:
    load().xlstm_mlstm_test_timeout_next(int(enable))


def status_string(status: int) -> str:
    try:
        return xlstm_status_string(status)
    except Exception:
        return f"status {status}"


def check(status: int, what: str = "") -> None:
    if status != XLSTM_OK:
        raise XlstmError(status, what)


# ---- torch conveniences (allocation + marshalling only) -------------------------
def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return XLSTM_BF16
    if t.dtype == torch.float32:
        return XLSTM_F32
    raise TypeError(f"q/k/v must be bf16 or fp32, got {t.dtype}")


def fwd(q, k, v, i_pre, f_pre, state=None, qk_scale=None, chunk=0, kind="chunkwise",
        stream=None, workspace=None, out=None, parallel=True, o_pre=None, h_dtype=None):
    """Sequence forward through the C ABI.  q, k [B,H,T,dqk], v [B,H,T,dv]
    (bf16 or fp32, CUDA, contiguous), i_pre/f_pre [B,H,T] fp32; state is None
    or (C [B,H,dv,dqk], n [B,H,dqk], m [B,H]).  Returns (h, (C, n, m)).
    Without a given workspace, the chunkwise call gets one large enough for the
    segment-parallel evaluation of long sequences (parallel=False: the minimum).
    o_pre [B,H,T,dv] (bf16 or fp32) applies the output gate, h = sigmoid(o_pre) h~,
    and h_dtype (torch.bfloat16 or torch.float32) picks h's type: both through
    xlstm_mlstm_fwd_chunkwise_out (chunkwise only)."""
    import torch
    B, H, T, dqk = q.shape
    dv = v.shape[-1]
    scale = (dqk ** -0.5) if qk_scale is None else float(qk_scale)
    desc = make_desc(B, H, T, dqk, dv, _dtype_code(q), scale, chunk)
    dev = q.device
    staged = o_pre is not None or h_dtype is not None
    if staged and kind != "chunkwise":
        raise ValueError("the output stage is fused into the chunkwise call only")
    hdt = torch.float32 if h_dtype is None else h_dtype
    if out is None:
        h = torch.empty(B, H, T, dv, device=dev, dtype=hdt)
        C1 = torch.empty(B, H, dv, dqk, device=dev, dtype=torch.float32)
        n1 = torch.empty(B, H, dqk, device=dev, dtype=torch.float32)
        m1 = torch.empty(B, H, device=dev, dtype=torch.float32)
    else:
        h, C1, n1, m1 = out
    C0, n0, m0 = state if state is not None else (None, None, None)
    stream = stream if stream is not None else torch.cuda.current_stream(dev)
    if kind == "chunkwise":
        if workspace is None:
            need = (xlstm_mlstm_workspace_size_parallel if parallel else xlstm_mlstm_workspace_size)(desc)
            workspace = torch.empty(max(256, need), device=dev, dtype=torch.uint8)
        if staged:
            ostage = xlstm_mlstm_output_t(None if o_pre is None else o_pre.data_ptr(),
                                          XLSTM_F32 if o_pre is None else _dtype_code(o_pre),
                                          XLSTM_BF16 if hdt == torch.bfloat16 else XLSTM_F32)
            st = xlstm_mlstm_fwd_chunkwise_out(desc, ostage, q, k, v, i_pre, f_pre, C0, n0, m0, h, C1, n1,
                                               m1, workspace, workspace.numel(), stream)
        else:
            st = xlstm_mlstm_fwd_chunkwise(desc, q, k, v, i_pre, f_pre, C0, n0, m0, h, C1, n1, m1,
                                           workspace, workspace.numel(), stream)
    elif kind == "recurrent":
        st = xlstm_mlstm_fwd_recurrent(desc, q, k, v, i_pre, f_pre, C0, n0, m0, h, C1, n1, m1,
                                       None, 0, stream)
    else:
        raise ValueError(kind)
    check(st, f"xlstm_mlstm_fwd_{kind}")
    return h, (C1, n1, m1)


def step(q, k, v, i_pre, f_pre, state, qk_scale=None, stream=None, out=None, inplace=False):
    """One decode step.  q, k [B,H,dqk], v [B,H,dv], i_pre/f_pre [B,H]; state
    (C, n, m).  Returns (h, (C', n', m')); inplace=True updates state's tensors."""
    import torch
    B, H, dqk = q.shape
    dv = v.shape[-1]
    scale = (dqk ** -0.5) if qk_scale is None else float(qk_scale)
    desc = make_desc(B, H, 1, dqk, dv, _dtype_code(q), scale, 0)
    C, n, m = state
    if inplace:
        C1, n1, m1 = C, n, m
        h = torch.empty(B, H, dv, device=q.device, dtype=torch.float32) if out is None else out[0]
    elif out is None:
        h = torch.empty(B, H, dv, device=q.device, dtype=torch.float32)
        C1, n1, m1 = torch.empty_like(C), torch.empty_like(n), torch.empty_like(m)
    else:
        h, C1, n1, m1 = out
    stream = stream if stream is not None else torch.cuda.current_stream(q.device)
    check(xlstm_mlstm_step(desc, q, k, v, i_pre, f_pre, C, n, m, h, C1, n1, m1, stream),
          "xlstm_mlstm_step")
    return h, (C1, n1, m1)


def summary(k, v, i_pre, f_pre, stream=None, workspace=None):
    """Summary of each (b, h) stretch through xlstm_mlstm_segment_summary:
    (C_seg [B,H,dv,dqk] fp32, n_seg [B,H,dqk] fp32, F_m [B,H,2] float64)."""
    import torch
    B, H, T, dqk = k.shape
    dv = v.shape[-1]
    desc = make_desc(B, H, T, dqk, dv, _dtype_code(k), 1.0, 0)
    dev = k.device
    C = torch.empty(B, H, dv, dqk, device=dev, dtype=torch.float32)
    n = torch.empty(B, H, dqk, device=dev, dtype=torch.float32)
    Fm = torch.empty(B, H, 2, device=dev, dtype=torch.float64)
    if workspace is None:
        workspace = torch.empty(256, device=dev, dtype=torch.uint8)
    stream = stream if stream is not None else torch.cuda.current_stream(dev)
    check(xlstm_mlstm_segment_summary(desc, k, v, i_pre, f_pre, C, n, Fm, workspace, workspace.numel(), stream),
          "xlstm_mlstm_segment_summary")
    return C, n, Fm


def combine(C_seg, n_seg, F_m, state=None, stream=None):
    """State after the stacked summaries (leading axis = stretch, in order)
    chained onto state (or the zero state), through xlstm_mlstm_combine_states."""
    import torch
    S, B, H, dv, dqk = C_seg.shape
    desc = make_desc(B, H, 1, dqk, dv, XLSTM_F32, 1.0, 0)
    dev = C_seg.device
    C1 = torch.empty(B, H, dv, dqk, device=dev, dtype=torch.float32)
    n1 = torch.empty(B, H, dqk, device=dev, dtype=torch.float32)
    m1 = torch.empty(B, H, device=dev, dtype=torch.float32)
    C0, n0, m0 = state if state is not None else (None, None, None)
    stream = stream if stream is not None else torch.cuda.current_stream(dev)
    check(xlstm_mlstm_combine_states(desc, S, C0, n0, m0, C_seg, n_seg, F_m, C1, n1, m1, stream),
          "xlstm_mlstm_combine_states")
    return C1, n1, m1


def bwd(q, k, v, i_pre, f_pre, dh, state=None, dstate=None, qk_scale=None, stream=None, workspace=None):
    """Backward through xlstm_mlstm_bwd_chunkwise.  Same inputs as ``fwd`` plus the
    upstream gradients dh of h~ (and dstate = (dC, dn) of the final state, or
    None).  Returns dict(dq, dk, dv, di, df, dC0, dn0, dm0), fp32."""
    import torch
    B, H, T, dqk = q.shape
    dv = v.shape[-1]
    scale = (dqk ** -0.5) if qk_scale is None else float(qk_scale)
    desc = make_desc(B, H, T, dqk, dv, _dtype_code(q), scale, 0)
    dev = q.device
    f32 = dict(device=dev, dtype=torch.float32)
    g = dict(dq=torch.empty(B, H, T, dqk, **f32), dk=torch.empty(B, H, T, dqk, **f32),
             dv=torch.empty(B, H, T, dv, **f32), di=torch.empty(B, H, T, **f32), df=torch.empty(B, H, T, **f32),
             dC0=torch.empty(B, H, dv, dqk, **f32), dn0=torch.empty(B, H, dqk, **f32), dm0=torch.empty(B, H, **f32))
    C0, n0, m0 = state if state is not None else (None, None, None)
    dC, dn = dstate if dstate is not None else (None, None)
    if workspace is None:
        workspace = torch.empty(max(256, xlstm_mlstm_bwd_workspace_size(desc)), device=dev, dtype=torch.uint8)
    stream = stream if stream is not None else torch.cuda.current_stream(dev)
    check(xlstm_mlstm_bwd_chunkwise(desc, q, k, v, i_pre, f_pre, C0, n0, m0, dh, dC, dn, g["dq"], g["dk"],
                                    g["dv"], g["di"], g["df"], g["dC0"], g["dn0"], g["dm0"], workspace,
                                    workspace.numel(), stream), "xlstm_mlstm_bwd_chunkwise")
    return g
