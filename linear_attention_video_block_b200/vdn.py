"""ctypes binding of libvdn (the C ABI declared in include/vdn.h).

Argument marshalling only: every step of the operation runs in libvdn's CUDA
kernels. PyTorch provides device memory and the current stream. There is no
CPU fallback: the functions raise if the library or a CUDA device is missing.

Public calls (same names as the C ABI, without the ``vdn_`` prefix):
  window_softmax_fwd, vda_scan_fwd, hybrid_attn_fwd, workspace_bytes,
  device_status, vda_scan_fwd_noalloc, joint_softmax_fwd, joint_attn_fwd.
vda_scan_fwd and hybrid_attn_fwd take an optional ``alpha`` [B, F, H, d]
float32 (KDA channel decay); when given they call the ``_decay`` entry points.
The joint_* calls add the audio keys and the dense text/audio query rows of a
joint text-video-audio layer (the C ABI's vdn_context_t).
Tensors follow the C ABI's layout: q/k/v/gates/outputs [B, L, H, d],
text k/v [B, T, H, d], beta [B, L, H] and beta_text [B, T, H] in float32.
"""

from __future__ import annotations

import ctypes
import os

import torch

from .synth import Layout

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvdn.so")
_lib = None

VDN_F32, VDN_BF16 = 0, 1
STATUS = {0: "VDN_OK", 1: "VDN_ERR_INVALID", 2: "VDN_ERR_UNSUPPORTED",
          3: "VDN_ERR_WORKSPACE", 4: "VDN_ERR_CUDA", 5: "VDN_ERR_TIMEOUT",
          6: "VDN_ERR_BOUNDS"}
EXPORTS = ("vdn_workspace_bytes", "vdn_window_softmax_fwd", "vdn_vda_scan_fwd",
           "vdn_vda_scan_fwd_decay", "vdn_hybrid_attn_fwd", "vdn_hybrid_attn_fwd_decay",
           "vdn_vda_scan_fwd_noalloc", "vdn_joint_softmax_fwd", "vdn_joint_attn_fwd",
           "vdn_window_softmax_fwd_fp8", "vdn_hybrid_attn_fwd_host",
           "vdn_hybrid_host_workspace_bytes", "vdn_gated_combine_fwd",
           "vdn_window_softmax_fwd_f32out", "vdn_vda_scan_fwd_f32out", "vdn_set_wait_limit_ns",
           "vdn_device_status",
           "vdn_status_string", "vdn_last_cuda_error")


class VdnError(RuntimeError):
    def __init__(self, code, where):
        msg = lib().vdn_status_string(code).decode() if _lib is not None else ""
        if code == 4 and _lib is not None:
            msg += ": " + lib().vdn_last_cuda_error().decode()
        super().__init__(f"{where}: {STATUS.get(code, code)} ({msg})")
        self.code = code


class _CLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "F", "N", "T", "c", "H", "d")]


class _CContext(ctypes.Structure):
    _fields_ = [("A", ctypes.c_int)] + [(n, ctypes.c_void_p) for n in (
        "k_audio", "v_audio", "q_text", "q_audio", "o_text", "o_audio", "lse_text", "lse_audio")]


def lib():
    """Loads libvdn.so (built in-tree by ``build.py``); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"libvdn.so not built ({_LIB_PATH}); run "
                               "python -m linear_attention_video_block_b200.build")
        L = ctypes.CDLL(_LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        LP = ctypes.POINTER(_CLayout)
        L.vdn_workspace_bytes.argtypes = [LP, I]
        L.vdn_workspace_bytes.restype = S
        L.vdn_window_softmax_fwd.argtypes = [LP, I] + [P] * 8
        L.vdn_window_softmax_fwd.restype = I
        L.vdn_vda_scan_fwd.argtypes = [LP, I] + [P] * 9 + [P, S, P]
        L.vdn_vda_scan_fwd.restype = I
        L.vdn_hybrid_attn_fwd.argtypes = [LP, I] + [P] * 9 + [P, ctypes.c_float] + [P] * 3 + [P, S, P]
        L.vdn_hybrid_attn_fwd.restype = I
        L.vdn_vda_scan_fwd_decay.argtypes = [LP, I] + [P] * 10 + [P, S, P]
        L.vdn_vda_scan_fwd_decay.restype = I
        L.vdn_hybrid_attn_fwd_decay.argtypes = ([LP, I] + [P] * 10 + [P, ctypes.c_float]
                                                + [P] * 3 + [P, S, P])
        L.vdn_hybrid_attn_fwd_decay.restype = I
        F = ctypes.c_float
        L.vdn_hybrid_host_workspace_bytes.argtypes = [LP, I, I]
        L.vdn_hybrid_host_workspace_bytes.restype = S
        L.vdn_hybrid_attn_fwd_host.argtypes = [LP, I, I] + [P] * 10 + [F, P, P, S]
        L.vdn_hybrid_attn_fwd_host.restype = I
        L.vdn_window_softmax_fwd_fp8.argtypes = [LP] + [P] * 5 + [F, F, F] + [P, P, P]
        L.vdn_window_softmax_fwd_fp8.restype = I
        CP = ctypes.POINTER(_CContext)
        L.vdn_joint_softmax_fwd.argtypes = [LP, I, CP] + [P] * 8
        L.vdn_joint_softmax_fwd.restype = I
        L.vdn_joint_attn_fwd.argtypes = ([LP, I, CP] + [P] * 10 + [P, ctypes.c_float]
                                         + [P] * 3 + [P, S, P])
        L.vdn_joint_attn_fwd.restype = I
        L.vdn_vda_scan_fwd_noalloc.argtypes = [LP, I] + [P] * 10
        L.vdn_vda_scan_fwd_noalloc.restype = I
        L.vdn_window_softmax_fwd_f32out.argtypes = [LP, I] + [P] * 8
        L.vdn_window_softmax_fwd_f32out.restype = I
        L.vdn_vda_scan_fwd_f32out.argtypes = [LP, I] + [P] * 9 + [P, S, P]
        L.vdn_vda_scan_fwd_f32out.restype = I
        L.vdn_gated_combine_fwd.argtypes = [ctypes.c_longlong, I, I, I] + [P] * 5 + [F, P, P]
        L.vdn_gated_combine_fwd.restype = I
        L.vdn_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
        L.vdn_set_wait_limit_ns.restype = I
        L.vdn_device_status.argtypes = []
        L.vdn_device_status.restype = I
        L.vdn_status_string.argtypes = [I]
        L.vdn_status_string.restype = ctypes.c_char_p
        L.vdn_last_cuda_error.argtypes = []
        L.vdn_last_cuda_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _clayout(layout: Layout):
    return _CLayout(layout.B, layout.F, layout.N, layout.T, layout.c, layout.H, layout.d)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return VDN_F32
    if t.dtype == torch.bfloat16:
        return VDN_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _expect(name, t, shape, dtype=None, required=True):
    """Checks one tensor argument against the layout before anything reaches
    the library: the kernels build their TMA tensor maps and index arithmetic
    from the layout alone, so a tensor of another shape would be read or
    written out of bounds on the device."""
    if t is None:
        if required:
            raise ValueError(f"{name} is required")
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}; the layout needs {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}; expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _same_device(*ts):
    devs = {t.device for t in ts if t is not None}
    if len(devs) > 1:
        raise ValueError(f"tensors on several devices: {sorted(str(d) for d in devs)}")


def _io_dtype(q):
    if q is None:
        raise ValueError("q is required")
    if q.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"unsupported dtype {q.dtype}; float32 or bfloat16")
    return q.dtype


def _validate(layout: Layout, q=None, io=(), text=(), beta=None, beta_text=None, alpha=None,
              rms_weight=None, lse=None, chunk_states=None, io_dtype=None, optional_io=(),
              text_dtype=None):
    """Shape, dtype and device checks of the common arguments. io / optional_io:
    (name, tensor) pairs of [B, L, H, d] tensors in the io dtype (required /
    nullable); text: (name, tensor) pairs of [B, T, H, d] tensors (required
    when T > 0)."""
    B, F, N, T, c, H, d = layout.B, layout.F, layout.N, layout.T, layout.c, layout.H, layout.d
    L = F * N
    dt = io_dtype if io_dtype is not None else _io_dtype(q)
    video = (B, L, H, d)
    _expect("q", q, video, dt)
    for name, t in io:
        _expect(name, t, video, dt)
    for name, t in optional_io:
        _expect(name, t, video, dt, required=False)
    for name, t in text:
        _expect(name, t, (B, T, H, d), text_dtype or dt, required=T > 0)
    _expect("beta", beta, (B, L, H), torch.float32, required=False)
    _expect("beta_text", beta_text, (B, T, H), torch.float32, required=False)
    _expect("alpha", alpha, (B, F, H, d), torch.float32, required=False)
    _expect("rms_weight", rms_weight, (d,), torch.float32, required=False)
    _expect("lse", lse, (B, L, H), torch.float32, required=False)
    J = -(-F // c) if c > 0 else 0
    _expect("chunk_states", chunk_states, (B, H, 2, J, d, d), torch.float32, required=False)
    _same_device(q, *(t for _, t in io), *(t for _, t in optional_io), *(t for _, t in text), beta,
                 beta_text, alpha, rms_weight, lse, chunk_states)


def _validate_workspace(workspace, q):
    if workspace is None:
        return
    if workspace.dtype != torch.uint8 or workspace.dim() != 1 or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous 1-D torch.uint8 tensor")
    _same_device(q, workspace)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(code, where):
    if code != 0:
        raise VdnError(code, where)


def _require_cuda():
    if not torch.cuda.is_available():
        raise RuntimeError("libvdn needs a CUDA device; there is no CPU path")


def workspace_bytes(layout: Layout, dtype: torch.dtype) -> int:
    code = VDN_BF16 if dtype == torch.bfloat16 else VDN_F32
    return int(lib().vdn_workspace_bytes(ctypes.byref(_clayout(layout)), code))


def window_softmax_fwd(layout: Layout, q, k, v, k_text, v_text, o_soft=None, lse=None,
                       want_lse=False, out_f32=False):
    """Softmax branch: returns o_soft (and lse [B, L, H] if want_lse); o_soft in
    the io dtype, or float32 with out_f32 (vdn_window_softmax_fwd_f32out)."""
    _validate(layout, q, io=[("k", k), ("v", v)], text=[("k_text", k_text), ("v_text", v_text)],
              lse=lse)
    _expect("o_soft", o_soft, tuple(q.shape), torch.float32 if out_f32 else q.dtype, required=False)
    _same_device(q, o_soft)
    _require_cuda()
    if o_soft is None:
        o_soft = torch.empty(q.shape, dtype=torch.float32 if out_f32 else q.dtype, device=q.device)
    if want_lse and lse is None:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    fn = lib().vdn_window_softmax_fwd_f32out if out_f32 else lib().vdn_window_softmax_fwd
    code = fn(ctypes.byref(_clayout(layout)), _dtype_code(q), _ptr(q), _ptr(k), _ptr(v),
              _ptr(k_text), _ptr(v_text), _ptr(o_soft), _ptr(lse), _stream(q.device))
    _check(code, "vdn_window_softmax_fwd" + ("_f32out" if out_f32 else ""))
    return (o_soft, lse) if want_lse else o_soft


def vda_scan_fwd(layout: Layout, q, k, v, k_text, v_text, beta, beta_text, o_lin=None,
                 chunk_states=None, want_states=False, workspace=None, alpha=None, out_f32=False):
    """Linear branch: returns o_lin (ungated, pre-norm) and, if want_states, the
    chunk table [B, H, 2, J, d, d] float32. alpha (optional, [B, F, H, d]
    float32) decays the state per key channel before each frame's write.
    out_f32: o_lin in float32 (vdn_vda_scan_fwd_f32out; not with alpha)."""
    _validate(layout, q, io=[("k", k), ("v", v)], text=[("k_text", k_text), ("v_text", v_text)],
              beta=beta, beta_text=beta_text, alpha=alpha, chunk_states=chunk_states)
    _expect("o_lin", o_lin, tuple(q.shape), torch.float32 if out_f32 else q.dtype, required=False)
    _same_device(q, o_lin)
    if out_f32 and alpha is not None:
        raise ValueError("out_f32 is not offered with alpha")
    _expect("beta", beta, (layout.B, layout.F * layout.N, layout.H), torch.float32)
    _expect("beta_text", beta_text, (layout.B, layout.T, layout.H), torch.float32,
            required=layout.T > 0)
    _validate_workspace(workspace, q)
    _require_cuda()
    if o_lin is None:
        o_lin = torch.empty(q.shape, dtype=torch.float32 if out_f32 else q.dtype, device=q.device)
    if want_states and chunk_states is None:
        J = -(-layout.F // layout.c)
        chunk_states = torch.empty((layout.B, layout.H, 2, J, layout.d, layout.d),
                                   dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(workspace_bytes(layout, q.dtype), dtype=torch.uint8, device=q.device)
    head = [ctypes.byref(_clayout(layout)), _dtype_code(q), _ptr(q), _ptr(k), _ptr(v),
            _ptr(k_text), _ptr(v_text), _ptr(beta), _ptr(beta_text)]
    tail = [_ptr(o_lin), _ptr(chunk_states), _ptr(workspace), workspace.numel(), _stream(q.device)]
    if out_f32:
        code, name = lib().vdn_vda_scan_fwd_f32out(*head, *tail), "vdn_vda_scan_fwd_f32out"
    elif alpha is None:
        code, name = lib().vdn_vda_scan_fwd(*head, *tail), "vdn_vda_scan_fwd"
    else:
        code = lib().vdn_vda_scan_fwd_decay(*head, _ptr(alpha), *tail)
        name = "vdn_vda_scan_fwd_decay"
    _check(code, name)
    return (o_lin, chunk_states) if want_states else o_lin


def hybrid_attn_fwd(layout: Layout, q, k, v, k_text, v_text, beta, beta_text, g_soft, g_lin,
                    rms_weight=None, rms_eps=1e-6, out=None, out_soft=None, out_lin=None,
                    workspace=None, device=None, alpha=None):
    """The hybrid forward: out = sigmoid(g_soft) o_soft + sigmoid(g_lin) RMSNorm(o_lin).
    alpha (optional, [B, F, H, d] float32): KDA decay of the linear branch.

    Device tensors: launched asynchronously on the current stream; returns out.
    Host tensors: vdn_hybrid_attn_fwd_host on ``device`` (default cuda:0), which
    copies in, computes and copies out in pipelined head chunks; returns the
    host output (pinned inputs let the copies overlap the kernels).
    """
    _validate(layout, q, io=[("k", k), ("v", v), ("g_soft", g_soft), ("g_lin", g_lin)],
              optional_io=[("out", out), ("out_soft", out_soft), ("out_lin", out_lin)],
              text=[("k_text", k_text), ("v_text", v_text)], beta=beta, beta_text=beta_text,
              alpha=alpha, rms_weight=rms_weight)
    _expect("beta", beta, (layout.B, layout.F * layout.N, layout.H), torch.float32)
    _expect("beta_text", beta_text, (layout.B, layout.T, layout.H), torch.float32,
            required=layout.T > 0)
    _validate_workspace(workspace, q)
    _require_cuda()
    if not q.is_cuda:
        if out_soft is not None or out_lin is not None or alpha is not None:
            raise ValueError("out_soft, out_lin and alpha need device tensors")
        return hybrid_attn_fwd_host(layout, q, k, v, k_text, v_text, beta, beta_text, g_soft, g_lin,
                                    rms_weight=rms_weight, rms_eps=rms_eps, out=out,
                                    workspace=workspace, device=device)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = torch.empty(workspace_bytes(layout, q.dtype), dtype=torch.uint8, device=q.device)
    head = [ctypes.byref(_clayout(layout)), _dtype_code(q), _ptr(q), _ptr(k), _ptr(v),
            _ptr(k_text), _ptr(v_text), _ptr(beta), _ptr(beta_text)]
    tail = [_ptr(g_soft), _ptr(g_lin), _ptr(rms_weight), ctypes.c_float(rms_eps), _ptr(out),
            _ptr(out_soft), _ptr(out_lin), _ptr(workspace), workspace.numel(), _stream(q.device)]
    if alpha is None:
        code, name = lib().vdn_hybrid_attn_fwd(*head, *tail), "vdn_hybrid_attn_fwd"
    else:
        code = lib().vdn_hybrid_attn_fwd_decay(*head, _ptr(alpha), *tail)
        name = "vdn_hybrid_attn_fwd_decay"
    _check(code, name)
    return out


def host_workspace_bytes(layout: Layout, dtype: torch.dtype, head_chunk: int = 0) -> int:
    code = VDN_BF16 if dtype == torch.bfloat16 else VDN_F32
    return int(lib().vdn_hybrid_host_workspace_bytes(ctypes.byref(_clayout(layout)), code, head_chunk))


def _host_ptr(t):
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError("tensor must live in host memory")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def hybrid_attn_fwd_host(layout: Layout, q, k, v, k_text, v_text, beta, beta_text, g_soft, g_lin,
                         rms_weight=None, rms_eps=1e-6, out=None, head_chunk=0, workspace=None,
                         device=None):
    """The hybrid forward on host tensors (vdn_hybrid_attn_fwd_host): copies in,
    computes and copies out in pipelined chunks of head_chunk heads (0: about
    ten chunks). workspace: device uint8 tensor of host_workspace_bytes (made
    here if None). Returns out, a host tensor (pinned when made here)."""
    _validate(layout, q, io=[("k", k), ("v", v), ("g_soft", g_soft), ("g_lin", g_lin)],
              optional_io=[("out", out)], text=[("k_text", k_text), ("v_text", v_text)],
              beta=beta, beta_text=beta_text, rms_weight=rms_weight)
    _expect("beta", beta, (layout.B, layout.F * layout.N, layout.H), torch.float32)
    _expect("beta_text", beta_text, (layout.B, layout.T, layout.H), torch.float32,
            required=layout.T > 0)
    _require_cuda()
    dev = torch.device(device or "cuda:0")
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    with torch.cuda.device(dev):
        if workspace is None:
            workspace = torch.empty(host_workspace_bytes(layout, q.dtype, head_chunk), dtype=torch.uint8,
                                    device=dev)
        code = lib().vdn_hybrid_attn_fwd_host(
            ctypes.byref(_clayout(layout)), _dtype_code(q), head_chunk, _host_ptr(q), _host_ptr(k),
            _host_ptr(v), _host_ptr(k_text), _host_ptr(v_text), _host_ptr(beta), _host_ptr(beta_text),
            _host_ptr(g_soft), _host_ptr(g_lin), _host_ptr(rms_weight), ctypes.c_float(rms_eps),
            _host_ptr(out), _ptr(workspace), workspace.numel())
    _check(code, "vdn_hybrid_attn_fwd_host")
    return out


NOALLOC_SCRATCH_BYTES = 64 << 20


def vda_scan_fwd_noalloc(layout: Layout, q, k, v, k_text, v_text, beta, beta_text, o_lin,
                         chunk_states=None):
    """Linear branch without a workspace and without allocating: for callers
    that cannot allocate device memory where they run the op. Scratch comes
    from a static 64 MiB device array inside the library (shared by all calls;
    overlapping calls race). o_lin (and chunk_states, if wanted) are
    caller-provided device tensors."""
    _validate(layout, q, io=[("k", k), ("v", v), ("o_lin", o_lin)],
              text=[("k_text", k_text), ("v_text", v_text)], beta=beta, beta_text=beta_text,
              chunk_states=chunk_states)
    _expect("beta", beta, (layout.B, layout.F * layout.N, layout.H), torch.float32)
    _expect("beta_text", beta_text, (layout.B, layout.T, layout.H), torch.float32,
            required=layout.T > 0)
    _require_cuda()
    code = lib().vdn_vda_scan_fwd_noalloc(ctypes.byref(_clayout(layout)), _dtype_code(q), _ptr(q), _ptr(k), _ptr(v),
             _ptr(k_text), _ptr(v_text), _ptr(beta), _ptr(beta_text), _ptr(o_lin),
             _ptr(chunk_states), _stream(q.device))
    _check(code, "vdn_vda_scan_fwd_noalloc")
    return o_lin


def gated_combine_fwd(o_soft, o_lin, g_soft, g_lin, rms_weight=None, rms_eps=1e-6, out=None):
    """out = sigmoid(g_soft) o_soft + sigmoid(g_lin) RMSNorm(o_lin) over the last
    dimension (vdn_gated_combine_fwd). o_soft, o_lin: float32 [..., H, d] (the
    _f32out branch outputs); g_soft, g_lin (and out) of the same shape in the io
    dtype; rms_weight [d] float32; one device. Returns out."""
    if g_soft is None:
        raise ValueError("g_soft is required")
    dt = _io_dtype(g_soft)
    shape = tuple(g_soft.shape)
    if len(shape) < 2:
        raise ValueError("tensors must be [..., H, d]")
    _expect("o_soft", o_soft, shape, torch.float32)
    _expect("o_lin", o_lin, shape, torch.float32)
    _expect("g_lin", g_lin, shape, dt)
    _expect("out", out, shape, dt, required=False)
    _expect("rms_weight", rms_weight, (shape[-1],), torch.float32, required=False)
    _same_device(o_soft, o_lin, g_soft, g_lin, rms_weight, out)
    _require_cuda()
    if out is None:
        out = torch.empty_like(g_soft)
    H, d = shape[-2], shape[-1]
    tokens = g_soft.numel() // (H * d) if H * d else 0
    code = lib().vdn_gated_combine_fwd(tokens, H, d, _dtype_code(g_soft), _ptr(o_soft), _ptr(o_lin),
                                       _ptr(g_soft), _ptr(g_lin), _ptr(rms_weight),
                                       ctypes.c_float(rms_eps), _ptr(out), _stream(g_soft.device))
    _check(code, "vdn_gated_combine_fwd")
    return out


def set_wait_limit_ns(ns: int) -> None:
    """Limit of the tensor-core kernels' role waits (vdn_set_wait_limit_ns; 0:
    the 4 s default). For tests of the timeout path only."""
    _require_cuda()
    _check(lib().vdn_set_wait_limit_ns(int(ns)), "vdn_set_wait_limit_ns")


def device_status() -> int:
    """Reads and clears libvdn's device status word (synchronises the device)."""
    return int(lib().vdn_device_status())


def _validate_context(layout, q, k_audio, v_audio, q_text, q_audio, o_text, o_audio):
    """Joint-layer tensors: audio keys/values [B, A, H, d] (both or neither),
    text query rows and their output [B, T, H, d], audio query rows and their
    output [B, A, H, d], all in the io dtype on q's device."""
    B, T, H, d = layout.B, layout.T, layout.H, layout.d
    dt = _io_dtype(q)
    if (k_audio is None) != (v_audio is None):
        raise ValueError("k_audio and v_audio go together")
    A = 0 if k_audio is None else int(k_audio.shape[1]) if k_audio.dim() == 4 else -1
    if A < 0:
        raise ValueError(f"k_audio has shape {tuple(k_audio.shape)}; expected [B, A, H, d]")
    _expect("k_audio", k_audio, (B, A, H, d), dt, required=False)
    _expect("v_audio", v_audio, (B, A, H, d), dt, required=False)
    _expect("q_text", q_text, (B, T, H, d), dt, required=False)
    _expect("o_text", o_text, (B, T, H, d), dt, required=False)
    _expect("q_audio", q_audio, (B, A, H, d), dt, required=False)
    _expect("o_audio", o_audio, (B, A, H, d), dt, required=False)
    if q_audio is not None and A == 0:
        raise ValueError("q_audio needs k_audio and v_audio")
    _same_device(q, k_audio, v_audio, q_text, o_text, q_audio, o_audio)


def _context(k_audio, v_audio, q_text, q_audio, o_text, o_audio, lse_text=None, lse_audio=None):
    A = 0 if k_audio is None else int(k_audio.shape[1])
    return _CContext(A, _ptr(k_audio), _ptr(v_audio), _ptr(q_text), _ptr(q_audio), _ptr(o_text),
                     _ptr(o_audio), _ptr(lse_text), _ptr(lse_audio))


def _context_outputs(q_text, q_audio, o_text, o_audio, want_lse):
    if q_text is not None and o_text is None:
        o_text = torch.empty_like(q_text)
    if q_audio is not None and o_audio is None:
        o_audio = torch.empty_like(q_audio)
    lt = la = None
    if want_lse:
        if q_text is not None:
            lt = torch.empty(q_text.shape[:3], dtype=torch.float32, device=q_text.device)
        if q_audio is not None:
            la = torch.empty(q_audio.shape[:3], dtype=torch.float32, device=q_audio.device)
    return o_text, o_audio, lt, la


def joint_softmax_fwd(layout: Layout, q, k, v, k_text, v_text, k_audio=None, v_audio=None,
                      q_text=None, q_audio=None, o_soft=None, o_text=None, o_audio=None,
                      want_lse=False):
    """Softmax part of a joint text-video-audio layer. Returns a dict with
    o_soft (video rows; their key sets include the audio keys), o_text and
    o_audio (dense context query rows, None when not asked for) and, with
    want_lse, lse / lse_text / lse_audio."""
    _validate(layout, q, io=[("k", k), ("v", v)], optional_io=[("o_soft", o_soft)],
              text=[("k_text", k_text), ("v_text", v_text)])
    _validate_context(layout, q, k_audio, v_audio, q_text, q_audio, o_text, o_audio)
    _require_cuda()
    if o_soft is None:
        o_soft = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if want_lse else None
    o_text, o_audio, lt, la = _context_outputs(q_text, q_audio, o_text, o_audio, want_lse)
    cx = _context(k_audio, v_audio, q_text, q_audio, o_text, o_audio, lt, la)
    code = lib().vdn_joint_softmax_fwd(
        ctypes.byref(_clayout(layout)), _dtype_code(q), ctypes.byref(cx), _ptr(q), _ptr(k), _ptr(v),
        _ptr(k_text), _ptr(v_text), _ptr(o_soft), _ptr(lse), _stream(q.device))
    _check(code, "vdn_joint_softmax_fwd")
    return {"o_soft": o_soft, "o_text": o_text, "o_audio": o_audio, "lse": lse,
            "lse_text": lt, "lse_audio": la}


def joint_attn_fwd(layout: Layout, q, k, v, k_text, v_text, beta, beta_text, g_soft, g_lin,
                   k_audio=None, v_audio=None, q_text=None, q_audio=None, alpha=None,
                   rms_weight=None, rms_eps=1e-6, out=None, o_text=None, o_audio=None,
                   out_soft=None, out_lin=None, workspace=None):
    """The attention of a joint text-video-audio layer: video rows get the
    hybrid (softmax branch with the audio keys; KDA decay when alpha is given),
    text/audio query rows the dense softmax. Returns (out, o_text, o_audio)."""
    _validate(layout, q, io=[("k", k), ("v", v), ("g_soft", g_soft), ("g_lin", g_lin)],
              optional_io=[("out", out), ("out_soft", out_soft), ("out_lin", out_lin)],
              text=[("k_text", k_text), ("v_text", v_text)], beta=beta, beta_text=beta_text,
              alpha=alpha, rms_weight=rms_weight)
    _expect("beta", beta, (layout.B, layout.F * layout.N, layout.H), torch.float32)
    _expect("beta_text", beta_text, (layout.B, layout.T, layout.H), torch.float32,
            required=layout.T > 0)
    _validate_context(layout, q, k_audio, v_audio, q_text, q_audio, o_text, o_audio)
    _validate_workspace(workspace, q)
    _require_cuda()
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = torch.empty(workspace_bytes(layout, q.dtype), dtype=torch.uint8, device=q.device)
    o_text, o_audio, _, _ = _context_outputs(q_text, q_audio, o_text, o_audio, False)
    cx = _context(k_audio, v_audio, q_text, q_audio, o_text, o_audio)
    code = lib().vdn_joint_attn_fwd(
        ctypes.byref(_clayout(layout)), _dtype_code(q), ctypes.byref(cx), _ptr(q), _ptr(k), _ptr(v),
        _ptr(k_text), _ptr(v_text), _ptr(beta), _ptr(beta_text), _ptr(alpha), _ptr(g_soft),
        _ptr(g_lin), _ptr(rms_weight), ctypes.c_float(rms_eps), _ptr(out), _ptr(out_soft),
        _ptr(out_lin), _ptr(workspace), workspace.numel(), _stream(q.device))
    _check(code, "vdn_joint_attn_fwd")
    return out, o_text, o_audio


def window_softmax_fwd_fp8(layout: Layout, q, k, v, k_text, v_text, q_scale, k_scale, v_scale,
                           o_soft=None, want_lse=False):
    """Softmax branch with float8 e4m3 operands (torch.float8_e4m3fn tensors,
    one scale per tensor; text shares k / v scales). Returns o_soft (bf16) and,
    with want_lse, the natural-log normaliser."""
    e4 = torch.float8_e4m3fn
    _validate(layout, q, io=[("k", k), ("v", v)], text=[("k_text", k_text), ("v_text", v_text)],
              io_dtype=e4)
    _expect("o_soft", o_soft, (layout.B, layout.F * layout.N, layout.H, layout.d), torch.bfloat16,
            required=False)
    _same_device(q, o_soft)
    _require_cuda()
    if o_soft is None:
        o_soft = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if want_lse else None
    code = lib().vdn_window_softmax_fwd_fp8(
        ctypes.byref(_clayout(layout)), _ptr(q), _ptr(k), _ptr(v), _ptr(k_text), _ptr(v_text),
        ctypes.c_float(q_scale), ctypes.c_float(k_scale), ctypes.c_float(v_scale), _ptr(o_soft),
        _ptr(lse), _stream(q.device))
    _check(code, "vdn_window_softmax_fwd_fp8")
    return (o_soft, lse) if want_lse else o_soft
