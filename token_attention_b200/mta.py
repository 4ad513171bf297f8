"""ctypes binding of libmta.so (include/mta.h).

Argument marshalling only: shapes and pointers are taken from torch tensors and
handed to the C ABI; every step of the computation runs in the library's CUDA
kernels.  There is no fallback: if libmta.so is missing or a call fails, this
module raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# MTA_LIB selects another build of the library (for comparing builds); default:
# the in-tree libmta.so next to this file.
LIB_PATH = os.environ.get("MTA_LIB") or os.path.join(HERE, "libmta.so")

OFF, PRE, POST, PRE_EXACT = 0, 1, 2, 3   # PRE_EXACT: key-query convolution with the exact causal indicator
F32, BF16 = 0, 1
PATH_AUTO, PATH_SIMT, PATH_TC, PATH_KQ = 0, 1, 2, 3

STATUS = {0: "MTA_OK", 1: "MTA_ERR_INVALID", 2: "MTA_ERR_UNSUPPORTED", 3: "MTA_ERR_WORKSPACE",
          4: "MTA_ERR_CUDA", 5: "MTA_ERR_TIMEOUT"}

# Every function include/mta.h declares.
EXPORTS = ["mta_attn_workspace_bytes", "mta_attn_fwd", "mta_layer_workspace_bytes",
           "mta_layer_fwd", "mta_gemm_bf16_nt", "mta_group_norm_scale", "mta_sync_status",
           "mta_status_string", "mta_abi_version", "mta_layer_fwd_static",
           "mta_attn_bwd_workspace_bytes", "mta_attn_bwd", "mta_attn_kernel",
           "mta_selftest_wait_timeout", "mta_layer_bwd_workspace_bytes", "mta_layer_bwd",
           "mta_gemm_bf16", "mta_group_norm_scale_bwd"]


class MtaCfg(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("L", ctypes.c_int), ("d", ctypes.c_int),
                ("c_q", ctypes.c_int), ("c_k", ctypes.c_int), ("c_h", ctypes.c_int),
                ("kq_place", ctypes.c_int), ("head_place", ctypes.c_int),
                ("kq_post", ctypes.c_int), ("dtype", ctypes.c_int), ("path", ctypes.c_int), ("scale", ctypes.c_float),
                ("qkv_row_stride", ctypes.c_longlong), ("stream", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("events", ctypes.POINTER(ctypes.c_void_p)), ("n_events", ctypes.c_int)]


class MtaGn(ctypes.Structure):
    _fields_ = [("gamma", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("eps", ctypes.c_float),
                ("layer", ctypes.c_int), ("depth_scale", ctypes.c_float), ("gate", ctypes.c_void_p)]


class MtaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libmta.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m token_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        cfgp = ctypes.POINTER(MtaCfg)
        L.mta_attn_workspace_bytes.argtypes = [cfgp]
        L.mta_attn_workspace_bytes.restype = S
        L.mta_layer_workspace_bytes.argtypes = [cfgp]
        L.mta_layer_workspace_bytes.restype = S
        L.mta_attn_fwd.argtypes = [P, P, P, P, P, cfgp, P]
        L.mta_attn_fwd.restype = I
        L.mta_layer_fwd.argtypes = [P, P, P, P, ctypes.POINTER(MtaGn), P, cfgp, P]
        L.mta_layer_fwd.restype = I
        L.mta_gemm_bf16_nt.argtypes = [P, P, P, I, I, I, P]
        L.mta_gemm_bf16_nt.restype = I
        L.mta_group_norm_scale.argtypes = [P, ctypes.POINTER(MtaGn), I, I, I, P, P]
        L.mta_group_norm_scale.restype = I
        L.mta_attn_bwd_workspace_bytes.argtypes = [cfgp]
        L.mta_attn_bwd_workspace_bytes.restype = S
        L.mta_attn_bwd.argtypes = [P, P, P, P, P, P, cfgp, P, P, P, P, P]
        L.mta_attn_bwd.restype = I
        L.mta_layer_bwd_workspace_bytes.argtypes = [cfgp]
        L.mta_layer_bwd_workspace_bytes.restype = S
        L.mta_layer_bwd.argtypes = [P, P, P, P, ctypes.POINTER(MtaGn), P, P, cfgp] + [P] * 8
        L.mta_layer_bwd.restype = I
        L.mta_gemm_bf16.argtypes = [P, P, P, I, I, I, I, I, I, P]
        L.mta_gemm_bf16.restype = I
        L.mta_group_norm_scale_bwd.argtypes = [P, P, ctypes.POINTER(MtaGn), I, I, I, P, P, P, P, P, P]
        L.mta_group_norm_scale_bwd.restype = I
        L.mta_attn_kernel.argtypes = [cfgp]
        L.mta_attn_kernel.restype = I
        L.mta_selftest_wait_timeout.argtypes = [cfgp, ctypes.c_uint]
        L.mta_selftest_wait_timeout.restype = I
        L.mta_sync_status.argtypes = [cfgp]
        L.mta_sync_status.restype = I
        L.mta_status_string.argtypes = [I]
        L.mta_status_string.restype = ctypes.c_char_p
        L.mta_abi_version.argtypes = []
        L.mta_abi_version.restype = I
        _lib = L
    return _lib


def _check(fn: str, code: int) -> None:
    if code != 0:
        raise MtaError(fn, code)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(name, t, device, dtype=None, shape=None, contiguous=True):
    """Rejects, before the library sees it, a tensor the C ABI cannot take.  The
    library reads raw device pointers, so a host tensor, a tensor on another GPU,
    another dtype or a strided view would be read as something else.  None passes
    (an optional argument)."""
    if t is None:
        return
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}, not on {t.device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, not {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _stream_handle(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _set_events(cfg: MtaCfg, events, n_events=None) -> None:
    """events: CUDA event handles (ints or objects with a cuda_event handle, such
    as torch.cuda.Event after its first record) the call records; n_events
    overrides the count (to test the library's checks)."""
    if events:
        hs = [e.cuda_event if hasattr(e, "cuda_event") else int(e) for e in events]
        arr = (ctypes.c_void_p * len(hs))(*hs)
        cfg._events_keep = arr          # keeps the array alive with the struct
        cfg.events = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    cfg.n_events = len(events or ()) if n_events is None else n_events


def make_cfg(B, H, L, d, c_q, c_k, c_h, kq_place, head_place, dtype, path=PATH_AUTO, scale=0.0,
             qkv_row_stride=0, stream=None, workspace=None, kq_post=0, events=None,
             n_events=None) -> MtaCfg:
    cfg = MtaCfg()
    cfg.B, cfg.H, cfg.L, cfg.d = B, H, L, d
    cfg.c_q, cfg.c_k, cfg.c_h = c_q, c_k, c_h
    cfg.kq_place, cfg.head_place, cfg.dtype, cfg.path = kq_place, head_place, dtype, path
    cfg.kq_post = kq_post
    cfg.scale = scale
    cfg.qkv_row_stride = qkv_row_stride
    cfg.stream = stream
    if workspace is not None:
        cfg.workspace = workspace.data_ptr()
        cfg.workspace_bytes = workspace.numel() * workspace.element_size()
    _set_events(cfg, events, n_events)
    return cfg


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def workspace(nbytes: int, device="cuda"):
    """A 256-byte aligned device buffer of at least nbytes (torch allocations are)."""
    import torch
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def kq_kernels(theta, theta_post, kq_place=PRE):
    """The library's key-query kernel array for a convolution after the softmax:
    the pre-softmax kernels [H, c_q, c_k] (when kq_place is on) stacked on the
    post-softmax ones, as one [n, H, c_q, c_k] tensor.  Build it once and pass it
    as `theta` to skip the per-call copy."""
    import torch
    if kq_place == OFF:
        return theta_post.contiguous()[None]
    return torch.stack([theta, theta_post])


def _kernels(theta, theta_post, kq_place):
    """(kernel array, kq_post) for the C ABI: a stacked [n, H, c_q, c_k] theta means
    the post-softmax kernels are its last entry."""
    if theta_post is not None:
        return kq_kernels(theta, theta_post, kq_place), 1
    if theta is not None and theta.dim() == 4:
        if theta.shape[0] != (1 if kq_place == OFF else 2) or not theta.is_contiguous():
            raise ValueError("a stacked theta holds the pre-softmax kernels (if on), then the post-softmax ones")
        return theta, 1
    return theta, 0


KERNEL_NAMES = {PATH_SIMT: "attn_simt_kernel", PATH_TC: "attn_tc_kernel", PATH_KQ: "attn_kq_kernel"}


def attn_kernel(cfg: MtaCfg) -> int:
    """The kernel mta_attn_fwd picks for cfg (PATH_SIMT, PATH_TC or PATH_KQ), asked
    of the library on the host; raises MtaError with the status the call would
    return instead of launching."""
    r = lib().mta_attn_kernel(ctypes.byref(cfg))
    if r < 0:
        raise MtaError("mta_attn_kernel", -r)
    return r


def attn_fwd(q, k, v, theta, w, c_q, c_k, c_h, kq_place=PRE, head_place=POST, *, out=None,
             ws=None, path=PATH_AUTO, scale=0.0, stream=None, check=False, theta_post=None,
             events=None):
    """MTA attention.  q, k, v: [B, L, H, d] CUDA tensors (fp32 or bf16), dense in
    (H, d) with a common token stride; theta [H, c_q, c_k] fp32; w [H/c_h, c_h, c_h]
    fp32; theta_post: optional [H, c_q, c_k] fp32 kernels of the key-query
    convolution after the softmax.  Returns out [B, L, H, d] (dtype of q)."""
    import torch
    B, L, H, d = q.shape
    for t in (k, v):
        if t.shape != q.shape or t.stride() != q.stride() or t.dtype != q.dtype:
            raise ValueError("q, k, v must share shape, strides and dtype")
    if q.stride(3) != 1 or q.stride(2) != d or q.stride(0) != L * q.stride(1):
        raise ValueError("q, k, v must be [B, L, H, d] with dense heads and a token stride")
    dv = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(name, t, dv, contiguous=False)
    for name, t in (("theta", theta), ("w", w), ("theta_post", theta_post)):
        _need(name, t, dv, torch.float32)
    _need("out", out, dv, q.dtype, (B, L, H, d))
    _need("ws", ws, dv)
    if out is None:
        out = torch.empty((B, L, H, d), dtype=q.dtype, device=q.device)
    theta, kq_post = _kernels(theta, theta_post, kq_place)
    cfg = make_cfg(B, H, L, d, c_q, c_k, c_h, kq_place, head_place, _dtype_code(q), path, scale,
                   q.stride(1), _stream_handle(stream), kq_post=kq_post, events=events)
    if ws is None:
        ws = workspace(lib().mta_attn_workspace_bytes(ctypes.byref(cfg)), q.device)
    cfg.workspace, cfg.workspace_bytes = ws.data_ptr(), _nbytes(ws)
    _check("mta_attn_fwd", lib().mta_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(theta), _ptr(w),
                                             ctypes.byref(cfg), _ptr(out)))
    if check:
        _check("mta_sync_status", lib().mta_sync_status(ctypes.byref(cfg)))
    return out


def attn_bwd(q, k, v, theta, w, dout, c_q, c_k, c_h, kq_place=PRE, head_place=POST, *, ws=None,
             path=PATH_AUTO, scale=0.0, stream=None, check=False, grads=None, theta_post=None,
             events=None):
    """Gradients of attn_fwd.  dout: [B, L, H, d] dense, dtype of q.  theta,
    theta_post: as for attn_fwd (a stacked [n, H, c_q, c_k] theta included).
    Returns a dict of fp32 tensors: dq, dk, dv [B, L, H, d]; dtheta [H, c_q, c_k]
    (kq_place on) and dtheta_post [H, c_q, c_k] (post-softmax convolution), views of
    one dtheta_all [n, H, c_q, c_k] laid out as the kernel array; dw
    [H/c_h, c_h, c_h] (head_place on).  `grads` may pass that dict to reuse."""
    import torch
    B, L, H, d = q.shape
    if dout.shape != q.shape or dout.dtype != q.dtype or not dout.is_contiguous():
        raise ValueError("dout must be a dense [B, L, H, d] tensor of q's dtype")
    if q.stride(3) != 1 or q.stride(2) != d or q.stride(0) != L * q.stride(1):
        raise ValueError("q, k, v must be [B, L, H, d] with dense heads and a token stride")
    dv = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(name, t, dv, q.dtype, q.shape, contiguous=False)
        if t.stride() != q.stride():
            raise ValueError("q, k, v must share strides")
    _need("dout", dout, dv)
    for name, t in (("theta", theta), ("w", w), ("theta_post", theta_post)):
        _need(name, t, dv, torch.float32)
    _need("ws", ws, dv)
    theta, kq_post = _kernels(theta, theta_post, kq_place)
    n_th = (1 if kq_place != OFF else 0) + kq_post
    if grads is None:
        z = lambda *shape: torch.empty(shape, dtype=torch.float32, device=q.device)
        dth = z(n_th, H, c_q, c_k) if n_th else None
        grads = {"dq": z(B, L, H, d), "dk": z(B, L, H, d), "dv": z(B, L, H, d), "dtheta_all": dth,
                 "dtheta": dth[0] if kq_place != OFF else None,
                 "dtheta_post": dth[n_th - 1] if kq_post else None,
                 "dw": z(H // c_h, c_h, c_h) if head_place != OFF else None}
    else:
        want = {"dq": (B, L, H, d), "dk": (B, L, H, d), "dv": (B, L, H, d),
                "dtheta_all": (n_th, H, c_q, c_k) if n_th else None,
                "dw": (H // c_h, c_h, c_h) if head_place != OFF else None}
        for name, shape in want.items():
            if shape is None:
                continue
            if grads.get(name) is None:
                raise ValueError(f"grads[{name!r}] is missing")
            _need(f"grads[{name!r}]", grads[name], dv, torch.float32, shape)
    cfg = make_cfg(B, H, L, d, c_q, c_k, c_h, kq_place, head_place, _dtype_code(q), path, scale,
                   q.stride(1), _stream_handle(stream), kq_post=kq_post, events=events)
    if ws is None:
        ws = workspace(lib().mta_attn_bwd_workspace_bytes(ctypes.byref(cfg)), q.device)
    cfg.workspace, cfg.workspace_bytes = ws.data_ptr(), _nbytes(ws)
    _check("mta_attn_bwd", lib().mta_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(theta), _ptr(w),
                                             _ptr(dout), ctypes.byref(cfg), _ptr(grads["dq"]),
                                             _ptr(grads["dk"]), _ptr(grads["dv"]),
                                             _ptr(grads["dtheta_all"]), _ptr(grads["dw"])))
    if check:
        _check("mta_sync_status", lib().mta_sync_status(ctypes.byref(cfg)))
    return grads


def _attention_function():
    """torch.autograd.Function over mta_attn_fwd / mta_attn_bwd (built on first use,
    so that importing this module needs no torch)."""
    import torch

    class _MtaAttention(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q, k, v, theta, w, c_q, c_k, c_h, kq_place, head_place, theta_post):
            out = attn_fwd(q, k, v, theta, w, c_q, c_k, c_h, kq_place, head_place, theta_post=theta_post)
            ctx.save_for_backward(q, k, v, theta, w, theta_post)
            ctx.shape = (c_q, c_k, c_h, kq_place, head_place)
            return out

        @staticmethod
        def backward(ctx, dout):
            q, k, v, theta, w, theta_post = ctx.saved_tensors
            c_q, c_k, c_h, kq_place, head_place = ctx.shape
            g = attn_bwd(q, k, v, theta, w, dout.contiguous().to(q.dtype), c_q, c_k, c_h, kq_place,
                         head_place, theta_post=theta_post)
            cast = lambda x, like: None if x is None or like is None else x.to(like.dtype)
            return (cast(g["dq"], q), cast(g["dk"], k), cast(g["dv"], v), cast(g["dtheta"], theta),
                    cast(g["dw"], w), None, None, None, None, None, cast(g["dtheta_post"], theta_post))

    return _MtaAttention


_MTA_FN = None


def mta_attention(q, k, v, theta, w, c_q, c_k, c_h, kq_place=PRE, head_place=POST, theta_post=None):
    """MTA attention as a differentiable torch op: the forward runs mta_attn_fwd, the
    backward mta_attn_bwd (gradients of q, k, v, theta, w and theta_post, cast to
    their dtypes).  Arguments as for attn_fwd; theta and theta_post are separate
    [H, c_q, c_k] tensors here."""
    global _MTA_FN
    if _MTA_FN is None:
        _MTA_FN = _attention_function()
    return _MTA_FN.apply(q, k, v, theta, w, c_q, c_k, c_h, kq_place, head_place, theta_post)


def layer_fwd(x, wqkv, theta, w, gamma, beta, wo, H, c_q, c_k, c_h, kq_place=PRE,
              head_place=POST, *, eps=1e-5, layer=12, lam=-1.0, gate=None, out=None, ws=None,
              path=PATH_AUTO, stream=None, check=False, theta_post=None, events=None):
    """Full MTA layer, bf16.  x [B, L, D]; wqkv [3D, D]; wo [D, D]; gamma, beta [D]
    fp32; gate: optional [H] fp32 sigmoid-gate logits replacing the depth scale;
    theta_post: optional [H, c_q, c_k] post-softmax key-query kernels.
    Returns out [B, L, D] bf16."""
    import torch
    B, L, D = x.shape
    if D % H:
        raise ValueError(f"D = {D} is not a multiple of H = {H}")
    d = D // H
    dv = x.device
    _need("x", x, dv)
    _need("wqkv", wqkv, dv, x.dtype, (3 * D, D))
    _need("wo", wo, dv, x.dtype, (D, D))
    for name, t in (("theta", theta), ("w", w), ("theta_post", theta_post)):
        _need(name, t, dv, torch.float32)
    _need("gamma", gamma, dv, torch.float32, (D,))
    _need("beta", beta, dv, torch.float32, (D,))
    _need("gate", gate, dv, torch.float32, (H,))
    _need("out", out, dv, x.dtype, (B, L, D))
    _need("ws", ws, dv)
    if out is None:
        out = torch.empty((B, L, D), dtype=x.dtype, device=x.device)
    theta, kq_post = _kernels(theta, theta_post, kq_place)
    cfg = make_cfg(B, H, L, d, c_q, c_k, c_h, kq_place, head_place, _dtype_code(x), path, 0.0, 0,
                   _stream_handle(stream), kq_post=kq_post, events=events)
    if ws is None:
        ws = workspace(lib().mta_layer_workspace_bytes(ctypes.byref(cfg)), x.device)
    cfg.workspace, cfg.workspace_bytes = ws.data_ptr(), _nbytes(ws)
    gn = MtaGn(gamma.data_ptr(), beta.data_ptr(), eps, layer, lam,
               gate.data_ptr() if gate is not None else None)
    _check("mta_layer_fwd", lib().mta_layer_fwd(_ptr(x), _ptr(wqkv), _ptr(theta), _ptr(w),
                                               ctypes.byref(gn), _ptr(wo), ctypes.byref(cfg),
                                               _ptr(out)))
    if check:
        _check("mta_sync_status", lib().mta_sync_status(ctypes.byref(cfg)))
    return out


def layer_bwd(x, wqkv, theta, w, gamma, beta, wo, dout, H, c_q, c_k, c_h, kq_place=PRE,
              head_place=POST, *, eps=1e-5, layer=12, lam=-1.0, gate=None, ws=None,
              path=PATH_AUTO, stream=None, check=False, theta_post=None, events=None):
    """Gradients of layer_fwd for dout [B, L, D] bf16.  Returns a dict of fp32
    tensors: dx [B, L, D], dwqkv [3D, D], dwo [D, D], dgamma, dbeta [D], dgate [H]
    (with a gate), dtheta / dtheta_post [H, c_q, c_k] (views of dtheta_all, laid
    out as the kernel array) and dw [H/c_h, c_h, c_h] as for attn_bwd."""
    import torch
    B, L, D = x.shape
    if D % H:
        raise ValueError(f"D = {D} is not a multiple of H = {H}")
    d = D // H
    dv = x.device
    _need("x", x, dv)
    _need("wqkv", wqkv, dv, x.dtype, (3 * D, D))
    _need("wo", wo, dv, x.dtype, (D, D))
    _need("dout", dout, dv, x.dtype, (B, L, D))
    for name, t in (("theta", theta), ("w", w), ("theta_post", theta_post)):
        _need(name, t, dv, torch.float32)
    _need("gamma", gamma, dv, torch.float32, (D,))
    _need("beta", beta, dv, torch.float32, (D,))
    _need("gate", gate, dv, torch.float32, (H,))
    _need("ws", ws, dv)
    theta, kq_post = _kernels(theta, theta_post, kq_place)
    n_th = (1 if kq_place != OFF else 0) + kq_post
    z = lambda *shape: torch.empty(shape, dtype=torch.float32, device=dv)
    dth = z(n_th, H, c_q, c_k) if n_th else None
    g = {"dx": z(B, L, D), "dwqkv": z(3 * D, D), "dwo": z(D, D), "dgamma": z(D), "dbeta": z(D),
         "dgate": z(H) if gate is not None else None, "dtheta_all": dth,
         "dtheta": dth[0] if kq_place != OFF else None,
         "dtheta_post": dth[n_th - 1] if kq_post else None,
         "dw": z(H // c_h, c_h, c_h) if head_place != OFF else None}
    cfg = make_cfg(B, H, L, d, c_q, c_k, c_h, kq_place, head_place, _dtype_code(x), path, 0.0, 0,
                   _stream_handle(stream), kq_post=kq_post, events=events)
    if ws is None:
        ws = workspace(lib().mta_layer_bwd_workspace_bytes(ctypes.byref(cfg)), x.device)
    cfg.workspace, cfg.workspace_bytes = ws.data_ptr(), _nbytes(ws)
    gn = MtaGn(gamma.data_ptr(), beta.data_ptr(), eps, layer, lam,
               gate.data_ptr() if gate is not None else None)
    _check("mta_layer_bwd", lib().mta_layer_bwd(
        _ptr(x), _ptr(wqkv), _ptr(theta), _ptr(w), ctypes.byref(gn), _ptr(wo), _ptr(dout),
        ctypes.byref(cfg), _ptr(g["dx"]), _ptr(g["dwqkv"]), _ptr(g["dwo"]), _ptr(g["dtheta_all"]),
        _ptr(g["dw"]), _ptr(g["dgamma"]), _ptr(g["dbeta"]), _ptr(g["dgate"])))
    if check:
        _check("mta_sync_status", lib().mta_sync_status(ctypes.byref(cfg)))
    return g


def layer_bwd_workspace_bytes(B, L, H, d, c_q, c_k, c_h, kq_place=PRE, head_place=POST,
                              kq_post=0) -> int:
    cfg = make_cfg(B, H, L, d, c_q, c_k, c_h, kq_place, head_place, BF16, kq_post=kq_post)
    return lib().mta_layer_bwd_workspace_bytes(ctypes.byref(cfg))


def layer_workspace_bytes(B, L, H, d, c_q, c_k, c_h, kq_place=PRE, head_place=POST,
                          kq_post=0) -> int:
    cfg = make_cfg(B, H, L, d, c_q, c_k, c_h, kq_place, head_place, BF16, kq_post=kq_post)
    return lib().mta_layer_workspace_bytes(ctypes.byref(cfg))


def gemm_bf16_nt(a, b, out=None, stream=None):
    """C = a b^T for bf16 a [M, K], b [N, K] (contiguous)."""
    import torch
    M, K = a.shape
    N = b.shape[0]
    _need("a", a, a.device, torch.bfloat16)
    _need("b", b, a.device, torch.bfloat16, (N, K))
    _need("out", out, a.device, torch.bfloat16, (M, N))
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    _check("mta_gemm_bf16_nt", lib().mta_gemm_bf16_nt(_ptr(a), _ptr(b), _ptr(out), M, N, K,
                                                     _stream_handle(stream)))
    return out


def gemm_bf16(a, b, M, N, K, a_mn=False, b_mn=False, f32_out=False, out=None, stream=None):
    """C [M, N] = A B^T with A given as a [M, K] (a_mn: as [K, M]) and B as b [N, K]
    (b_mn: as [K, N]), bf16 contiguous; C bf16, or fp32 with f32_out."""
    import torch
    _need("a", a, a.device, torch.bfloat16, (K, M) if a_mn else (M, K))
    _need("b", b, a.device, torch.bfloat16, (K, N) if b_mn else (N, K))
    odt = torch.float32 if f32_out else torch.bfloat16
    _need("out", out, a.device, odt, (M, N))
    if out is None:
        out = torch.empty((M, N), dtype=odt, device=a.device)
    _check("mta_gemm_bf16", lib().mta_gemm_bf16(_ptr(a), _ptr(b), _ptr(out), M, N, K, int(a_mn), int(b_mn),
                                               int(f32_out), _stream_handle(stream)))
    return out


def group_norm_scale_bwd(o, dy, gamma, beta, eps=1e-5, lam=1.0, gate=None, stream=None):
    """Backward of group_norm_scale: o [..., H, d] bf16, dy the same shape fp32.
    Returns (y bf16, do bf16, dgamma, dbeta [H*d] fp32, dgate [H] fp32 or None)."""
    import torch
    H, d = o.shape[-2], o.shape[-1]
    tokens = o.numel() // (H * d)
    dv = o.device
    _need("o", o, dv, torch.bfloat16)
    _need("dy", dy, dv, torch.float32, tuple(o.shape))
    _need("gamma", gamma, dv, torch.float32, (H * d,))
    _need("beta", beta, dv, torch.float32, (H * d,))
    _need("gate", gate, dv, torch.float32, (H,))
    y = torch.empty_like(o)
    do = torch.empty_like(o)
    z = lambda *shape: torch.empty(shape, dtype=torch.float32, device=dv)
    dgamma, dbeta = z(H * d), z(H * d)
    dgate = z(H) if gate is not None else None
    gn = MtaGn(gamma.data_ptr(), beta.data_ptr(), eps, 0, lam, gate.data_ptr() if gate is not None else None)
    _check("mta_group_norm_scale_bwd", lib().mta_group_norm_scale_bwd(
        _ptr(o), _ptr(dy), ctypes.byref(gn), tokens, H, d, _ptr(y), _ptr(do), _ptr(dgamma), _ptr(dbeta),
        _ptr(dgate), _stream_handle(stream)))
    return y, do, dgamma, dbeta, dgate


def group_norm_scale(o, gamma, beta, eps=1e-5, lam=1.0, out=None, stream=None, gate=None):
    """Depth-scaled group norm of o [..., H, d] bf16 (dense)."""
    import torch
    H, d = o.shape[-2], o.shape[-1]
    tokens = o.numel() // (H * d)
    _need("o", o, o.device, torch.bfloat16)
    for name, t in (("gamma", gamma), ("beta", beta)):
        _need(name, t, o.device, torch.float32)
        if t.numel() != H * d:
            raise ValueError(f"{name} must hold H*d = {H * d} values, not {t.numel()}")
    _need("gate", gate, o.device, torch.float32, (H,))
    _need("out", out, o.device, torch.bfloat16, tuple(o.shape))
    if out is None:
        out = torch.empty_like(o)
    gn = MtaGn(gamma.data_ptr(), beta.data_ptr(), eps, 0, lam,
               gate.data_ptr() if gate is not None else None)
    _check("mta_group_norm_scale", lib().mta_group_norm_scale(_ptr(o), ctypes.byref(gn), tokens, H,
                                                             d, _ptr(out), _stream_handle(stream)))
    return out
