"""Python binding of the SQuad-Attention C ABI, with the C names.

Argument marshalling only: every step of the computation runs in the CUDA library. Tensors are torch
CUDA tensors (PyTorch provides device memory and streams); shapes are [B, h, n, d] contiguous with
n = T*H*W in (t, y, x) row-major order.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib

ORDERS = {"local_then_global": _lib.SQUAD_LOCAL_THEN_GLOBAL, "global_then_local": _lib.SQUAD_GLOBAL_THEN_LOCAL,
          "local_only": _lib.SQUAD_LOCAL_ONLY, "global_only": _lib.SQUAD_GLOBAL_ONLY}
_DTYPES = {torch.bfloat16: _lib.SQUAD_BF16, torch.float32: _lib.SQUAD_FP32}


class SquadError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = _lib.load().squad_status_string(status).decode()
        super().__init__(f"{what}: {msg} (status {status})")


def make_params(B, h, d, grid, window=(1, 1, 1), order="local_then_global", dtype=torch.bfloat16, scale=None):
    T, H, W = grid
    tw, hw, ww = window
    o = ORDERS[order] if isinstance(order, str) else int(order)
    dt = _DTYPES[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    return _lib.SquadParams(B, h, d, T, H, W, tw, hw, ww, o, dt, 0.0 if scale is None else float(scale))


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check_qkv(*ts):
    """Every tensor handed to the library (q, k, v, o, dout, dq, dk, dv; None = not given) must be a
    contiguous CUDA tensor of q's dtype, shape and device: the kernels address them with q's layout on
    the device the call runs on."""
    q = ts[0]
    for t in ts:
        if t is None:
            continue
        if (not t.is_cuda or not t.is_contiguous() or t.dtype != q.dtype or t.shape != q.shape
                or t.device != q.device):
            raise ValueError("q, k, v and the outputs must be contiguous CUDA tensors of one dtype, shape "
                             "[B,h,n,d] and device")
    if q.dim() != 4:
        raise ValueError("expected [B, h, n, d]")


def _check_workspace(ws, q, nbytes):
    if not ws.is_cuda or ws.device != q.device or not ws.is_contiguous():
        raise ValueError("the workspace must be a contiguous CUDA tensor on q's device")
    if ws.numel() * ws.element_size() < nbytes:
        raise ValueError(f"workspace needs {nbytes} bytes")


def _params_for(q, grid, window, order, scale):
    B, h, n, d = q.shape
    if n != grid[0] * grid[1] * grid[2]:
        raise ValueError(f"n = {n} but T*H*W = {grid[0] * grid[1] * grid[2]}")
    return make_params(B, h, d, grid, window, order, q.dtype, scale)


def squad_attn_fwd_workspace_bytes(params) -> int:
    return int(_lib.load().squad_attn_fwd_workspace_bytes(ctypes.byref(params)))


def squad_attn_bwd_workspace_bytes(params) -> int:
    return int(_lib.load().squad_attn_bwd_workspace_bytes(ctypes.byref(params)))


def squad_attn_fwd(q, k, v, grid, window, order="local_then_global", scale=None, out=None, workspace=None,
                   stream=None):
    """SQuad-Attention forward. Returns (out, workspace); keep the workspace for squad_attn_bwd."""
    _check_qkv(q, k, v, out)
    prm = _params_for(q, grid, window, order, scale)
    lib = _lib.load()
    nbytes = lib.squad_attn_fwd_workspace_bytes(ctypes.byref(prm))
    if nbytes == 0:
        raise SquadError(_lib.SQUAD_ERR_INVALID_ARG, "squad_attn_fwd_workspace_bytes")
    out = torch.empty_like(q) if out is None else out
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    else:
        _check_workspace(workspace, q, nbytes)
    with torch.cuda.device(q.device):
        st = lib.squad_attn_fwd(ctypes.byref(prm), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(workspace),
                                _stream(stream))
    if st != _lib.SQUAD_OK:
        raise SquadError(st, "squad_attn_fwd")
    return out, workspace


def squad_attn_fwd_noalloc(q, k, v, grid, window, order="local_then_global", scale=None, out=None, stream=None):
    """SQuad-Attention forward with the library's fixed device scratch instead of a workspace (for
    callers that cannot allocate device memory; calls that overlap on the GPU race on the scratch)."""
    _check_qkv(q, k, v, out)
    prm = _params_for(q, grid, window, order, scale)
    out = torch.empty_like(q) if out is None else out
    with torch.cuda.device(q.device):
        st = _lib.load().squad_attn_fwd_noalloc(ctypes.byref(prm), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                                _stream(stream))
    if st != _lib.SQUAD_OK:
        raise SquadError(st, "squad_attn_fwd_noalloc")
    return out


def squad_attn_fwd_status(workspace, q, grid, window, order="local_then_global", scale=None, stream=None) -> int:
    """Device status of the last call on `workspace` (synchronises the stream): 0 ok, 4 timeout."""
    prm = _params_for(q, grid, window, order, scale)
    with torch.cuda.device(q.device):
        return int(_lib.load().squad_attn_fwd_status(ctypes.byref(prm), _ptr(workspace), _stream(stream)))


def squad_attn_bwd(q, k, v, o, dout, fwd_workspace, grid, window, order="local_then_global", scale=None,
                   dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients (dq, dk, dv) of <dout, o>; `fwd_workspace` as left by squad_attn_fwd."""
    _check_qkv(q, k, v, o, dout, dq, dk, dv)
    prm = _params_for(q, grid, window, order, scale)
    lib = _lib.load()
    nbytes = lib.squad_attn_bwd_workspace_bytes(ctypes.byref(prm))
    if nbytes == 0:
        raise SquadError(_lib.SQUAD_ERR_INVALID_ARG, "squad_attn_bwd_workspace_bytes")
    _check_workspace(fwd_workspace, q, lib.squad_attn_fwd_workspace_bytes(ctypes.byref(prm)))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    else:
        _check_workspace(workspace, q, nbytes)
    with torch.cuda.device(q.device):
        st = lib.squad_attn_bwd(ctypes.byref(prm), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout),
                                _ptr(fwd_workspace), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), _stream(stream))
    if st != _lib.SQUAD_OK:
        raise SquadError(st, "squad_attn_bwd")
    return dq, dk, dv


BWD_KERNEL_NAMES = {0: None, _lib.SQUAD_BWD_TC_WHOLE: "tc_whole", _lib.SQUAD_BWD_TC_CHUNKED: "tc_chunked",
                    _lib.SQUAD_BWD_CUDA_CORE: "cuda_core"}


def squad_attn_bwd_kernels(B, h, d, grid, window, order="local_then_global", dtype=torch.bfloat16):
    """The backward kernel of each pass, in forward execution order: ("tc_whole" | "tc_chunked" |
    "cuda_core", second pass or None)."""
    ks = (ctypes.c_int * 2)()
    st = _lib.load().squad_attn_bwd_kernels(ctypes.byref(make_params(B, h, d, grid, window, order, dtype)), ks)
    if st != _lib.SQUAD_OK:
        raise SquadError(st, "squad_attn_bwd_kernels")
    return BWD_KERNEL_NAMES[ks[0]], BWD_KERNEL_NAMES[ks[1]]


def full_attn_fwd(q, k, v, grid=None, scale=None, out=None, lse=None, stream=None):
    """softmax(q k^T * scale) v over all n tokens per head. Returns out (and fills `lse` if given)."""
    _check_qkv(q, k, v, out)
    B, h, n, d = q.shape
    if lse is not None and (not lse.is_cuda or lse.device != q.device or lse.dtype != torch.float32
                            or not lse.is_contiguous() or lse.numel() < B * h * n):
        raise ValueError("lse must be a contiguous float32 CUDA tensor of B*h*n elements on q's device")
    grid = (1, 1, n) if grid is None else grid
    prm = _params_for(q, grid, (1, 1, 1), "local_then_global", scale)
    out = torch.empty_like(q) if out is None else out
    with torch.cuda.device(q.device):
        st = _lib.load().full_attn_fwd(ctypes.byref(prm), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                       _ptr(lse), _stream(stream))
    if st != _lib.SQUAD_OK:
        raise SquadError(st, "full_attn_fwd")
    return out


SP_LAYOUTS = {"band": _lib.SQUAD_SP_BAND, "frames": _lib.SQUAD_SP_FRAMES, "chunks": _lib.SQUAD_SP_CHUNKS}


def squad_seqpar_reorder(x, grid, R, src, dst, add=None, out=None, stream=None):
    """The sequence split's block reordering (squad_seqpar_reorder): x in layout `src` ("band",
    "frames" or "chunks") -> a new tensor in layout `dst`, plus `add` (layout `dst`) if given.
    band and frames tensors are [B, h, n/R, d]; chunks tensors are [R, B, h, n/R^2, d] (the all-to-all
    splits their first dimension). With one rank, or src == dst, and neither add nor out given, the
    layouts order the blocks alike and x itself is returned, reshaped."""
    T, H, W = grid
    if x.dim() not in (4, 5) or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA tensor [B, h, n/R, d] or [R, B, h, n/R^2, d]")
    B, h = (x.shape[1], x.shape[2]) if x.dim() == 5 else (x.shape[0], x.shape[1])
    d = x.shape[-1]
    if R < 1 or T % R or H % R or x.numel() * R != B * h * T * H * W * d or (x.dim() == 5) != (src == "chunks"):
        raise ValueError(f"x does not hold one rank's {src} tensor of the {T}x{H}x{W} grid split {R} ways")
    shape = (R, B, h, T * H * W // (R * R), d) if dst == "chunks" else (B, h, T * H * W // R, d)
    if add is None and out is None and (R == 1 or src == dst):
        return x.view(shape)   # the two layouts order the blocks alike: nothing moves
    out = torch.empty(shape, dtype=x.dtype, device=x.device) if out is None else out
    for t in (add, out):
        if t is not None and (not t.is_cuda or not t.is_contiguous() or t.dtype != x.dtype or t.device != x.device
                              or tuple(t.shape) != shape):
            raise ValueError(f"add and out must be contiguous CUDA tensors of x's dtype and device, shape {shape}")
    prm = make_params(B, h, d, grid, (T, 1, 1), "local_then_global", x.dtype)
    with torch.cuda.device(x.device):
        st = _lib.load().squad_seqpar_reorder(ctypes.byref(prm), int(R), SP_LAYOUTS[src], SP_LAYOUTS[dst], _ptr(x),
                                              _ptr(add), _ptr(out), _stream(stream))
    if st != _lib.SQUAD_OK:
        raise SquadError(st, "squad_seqpar_reorder")
    return out


def squad_attn_flops(B, h, d, grid, window, order="local_then_global") -> float:
    return float(_lib.load().squad_attn_flops(ctypes.byref(make_params(B, h, d, grid, window, order))))


def squad_window_solve(grid):
    """The window (tw, hw, ww) for a (T, H, W) grid (w_t = T, aspect-following, least padded cost)."""
    tw, hw, ww = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    st = _lib.load().squad_window_solve(int(grid[0]), int(grid[1]), int(grid[2]), ctypes.byref(tw), ctypes.byref(hw),
                                        ctypes.byref(ww))
    if st != _lib.SQUAD_OK:
        raise SquadError(st, "squad_window_solve")
    return tw.value, hw.value, ww.value


def full_attn_flops(B, h, d, grid) -> float:
    return float(_lib.load().full_attn_flops(ctypes.byref(make_params(B, h, d, grid))))


KPASS_ORDERS = {"forward": _lib.SQUAD_KPASS_FORWARD, "reverse": _lib.SQUAD_KPASS_REVERSE}


def make_kpass_params(B, h, d, grid, levels, order="forward", dtype=torch.bfloat16, scale=None):
    """squad_kpass_params_t for k = len(levels) nested-window passes; levels = [(h_1, w_1), ...]."""
    T, H, W = grid
    levels = [(int(a), int(b)) for a, b in levels]
    m = _lib.SQUAD_KPASS_MAX_LEVELS
    if not 1 <= len(levels) <= m:
        raise ValueError(f"1 to {m} levels")
    pad = [0] * (m - len(levels))
    lh = (ctypes.c_int * m)(*([a for a, _ in levels] + pad))
    lw = (ctypes.c_int * m)(*([b for _, b in levels] + pad))
    o = KPASS_ORDERS[order] if isinstance(order, str) else int(order)
    dt = _DTYPES[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    return _lib.SquadKpassParams(B, h, d, T, H, W, len(levels), lh, lw, o, dt, 0.0 if scale is None else float(scale))


def _kpass_params_for(q, grid, levels, order, scale):
    B, h, n, d = q.shape
    if n != grid[0] * grid[1] * grid[2]:
        raise ValueError(f"n = {n} but T*H*W = {grid[0] * grid[1] * grid[2]}")
    return make_kpass_params(B, h, d, grid, levels, order, q.dtype, scale)


def squad_kpass_pass_params(params, level):
    """The single-pass problem (SquadParams) that `level` (0-based) of a k-pass call runs."""
    out = _lib.SquadParams()
    st = _lib.load().squad_kpass_pass_params(ctypes.byref(params), int(level), ctypes.byref(out))
    if st != _lib.SQUAD_OK:
        raise SquadError(st, "squad_kpass_pass_params")
    return out


def squad_kpass_fwd(q, k, v, grid, levels, order="forward", scale=None, out=None, workspace=None, stream=None):
    """k nested-window passes composed. Returns (out, workspace); keep the workspace for the backward."""
    _check_qkv(q, k, v, out)
    prm = _kpass_params_for(q, grid, levels, order, scale)
    lib = _lib.load()
    nbytes = lib.squad_kpass_fwd_workspace_bytes(ctypes.byref(prm))
    if nbytes == 0:
        raise SquadError(_lib.SQUAD_ERR_INVALID_ARG, "squad_kpass_fwd_workspace_bytes")
    out = torch.empty_like(q) if out is None else out
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    else:
        _check_workspace(workspace, q, nbytes)
    with torch.cuda.device(q.device):
        st = lib.squad_kpass_fwd(ctypes.byref(prm), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(workspace),
                                 _stream(stream))
    if st != _lib.SQUAD_OK:
        raise SquadError(st, "squad_kpass_fwd")
    return out, workspace


def squad_kpass_bwd(q, k, v, o, dout, fwd_workspace, grid, levels, order="forward", scale=None, dq=None, dk=None,
                    dv=None, workspace=None, stream=None):
    """Gradients (dq, dk, dv) of <dout, o> for squad_kpass_fwd; `fwd_workspace` as it left it."""
    _check_qkv(q, k, v, o, dout, dq, dk, dv)
    prm = _kpass_params_for(q, grid, levels, order, scale)
    lib = _lib.load()
    nbytes = lib.squad_kpass_bwd_workspace_bytes(ctypes.byref(prm))
    if nbytes == 0:
        raise SquadError(_lib.SQUAD_ERR_INVALID_ARG, "squad_kpass_bwd_workspace_bytes")
    _check_workspace(fwd_workspace, q, lib.squad_kpass_fwd_workspace_bytes(ctypes.byref(prm)))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    else:
        _check_workspace(workspace, q, nbytes)
    with torch.cuda.device(q.device):
        st = lib.squad_kpass_bwd(ctypes.byref(prm), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout),
                                 _ptr(fwd_workspace), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), _stream(stream))
    if st != _lib.SQUAD_OK:
        raise SquadError(st, "squad_kpass_bwd")
    return dq, dk, dv


def squad_kpass_status(workspace, q, grid, levels, order="forward", scale=None, stream=None) -> int:
    """Device status of the last k-pass call on `workspace` (synchronises the stream): 0 ok, 4 timeout."""
    prm = _kpass_params_for(q, grid, levels, order, scale)
    with torch.cuda.device(q.device):
        return int(_lib.load().squad_kpass_status(ctypes.byref(prm), _ptr(workspace), _stream(stream)))


def squad_kpass_flops(B, h, d, grid, levels) -> float:
    return float(_lib.load().squad_kpass_flops(ctypes.byref(make_kpass_params(B, h, d, grid, levels))))


class _SquadAttention(torch.autograd.Function):
    """squad_attn_fwd / squad_attn_bwd as one autograd node; the workspace is saved for the backward."""

    @staticmethod
    def forward(ctx, q, k, v, grid, window, order, scale):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, ws = squad_attn_fwd(q, k, v, grid, window, order, scale)
        ctx.save_for_backward(q, k, v, o, ws)
        ctx.cfg = (grid, window, order, scale)
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, ws = ctx.saved_tensors
        grid, window, order, scale = ctx.cfg
        dq, dk, dv = squad_attn_bwd(q, k, v, o, do.contiguous(), ws, grid, window, order, scale)
        return dq, dk, dv, None, None, None, None


def squad_attention(q, k, v, grid, window, order="local_then_global", scale=None):
    """SQuad-Attention as a differentiable torch op (the library's forward and backward kernels)."""
    return _SquadAttention.apply(q, k, v, tuple(grid), tuple(window), order, scale)


class _KpassAttention(torch.autograd.Function):
    """squad_kpass_fwd / squad_kpass_bwd as one autograd node."""

    @staticmethod
    def forward(ctx, q, k, v, grid, levels, order, scale):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, ws = squad_kpass_fwd(q, k, v, grid, levels, order, scale)
        ctx.save_for_backward(q, k, v, o, ws)
        ctx.cfg = (grid, levels, order, scale)
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, ws = ctx.saved_tensors
        grid, levels, order, scale = ctx.cfg
        dq, dk, dv = squad_kpass_bwd(q, k, v, o, do.contiguous(), ws, grid, levels, order, scale)
        return dq, dk, dv, None, None, None, None


def squad_kpass_attention(q, k, v, grid, levels, order="forward", scale=None):
    """k composed nested-window passes as a differentiable torch op."""
    return _KpassAttention.apply(q, k, v, tuple(grid), tuple(tuple(l) for l in levels), order, scale)


def squad_attn_fwd_host_workspace_bytes(params, groups) -> int:
    return int(_lib.load().squad_attn_fwd_host_workspace_bytes(ctypes.byref(params), int(groups)))


def squad_attn_fwd_host(q_host, k_host, v_host, o_host, q_dev, k_dev, v_dev, o_dev, workspace, grid, window,
                        order="local_then_global", scale=None, groups=4, copy_in=None, compute=None, copy_out=None):
    """The C forward from host memory (squad_attn_fwd_host): q, k, v host tensors -> device buffers ->
    forward -> o_host, in `groups` runs of heads whose copies overlap the forwards on three streams."""
    for t in (q_host, k_host, v_host, o_host):
        if t.is_cuda or not t.is_contiguous() or t.shape != q_dev.shape or t.dtype != q_dev.dtype:
            raise ValueError("host tensors must be contiguous CPU tensors of the device buffers' shape and dtype")
    _check_qkv(q_dev, k_dev, v_dev, o_dev)
    prm = _params_for(q_dev, grid, window, order, scale)
    lib = _lib.load()
    nbytes = lib.squad_attn_fwd_host_workspace_bytes(ctypes.byref(prm), int(groups))
    if nbytes == 0:
        raise SquadError(_lib.SQUAD_ERR_INVALID_ARG, "squad_attn_fwd_host_workspace_bytes")
    _check_workspace(workspace, q_dev, nbytes)
    with torch.cuda.device(q_dev.device):
        st = lib.squad_attn_fwd_host(ctypes.byref(prm), _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(o_host),
                                     _ptr(q_dev), _ptr(k_dev), _ptr(v_dev), _ptr(o_dev), _ptr(workspace), int(groups),
                                     _stream(copy_in), _stream(compute), _stream(copy_out))
    if st != _lib.SQUAD_OK:
        raise SquadError(st, "squad_attn_fwd_host")
    return o_host


class HostRunner:
    """End-to-end forward from pinned host buffers through the C entry point squad_attn_fwd_host.

    Device buffers, the workspace and three streams (input copies, forwards, output copies) are made
    once; every call() enqueues the copies in, the forwards and the copies out for `groups` runs of
    heads, overlapping each run's copies with the neighbouring runs' forwards. `start` and `end` record
    CUDA events that bracket any number of calls (end: after the last output copy).
    """

    def __init__(self, B, h, d, grid, window, order="local_then_global", dtype=torch.bfloat16, device="cuda",
                 groups=4):
        n = grid[0] * grid[1] * grid[2]
        self.shape = (B, h, n, d)
        self.grid, self.window, self.order = grid, window, order
        self.groups = max(1, min(int(groups), B * h, 64))
        self.dev = [torch.empty(self.shape, dtype=dtype, device=device) for _ in range(4)]
        prm = make_params(B, h, d, grid, window, order, dtype)
        self.ws = torch.empty(squad_attn_fwd_host_workspace_bytes(prm, self.groups), dtype=torch.uint8, device=device)
        self.s_in, self.s_comp, self.s_out = (torch.cuda.Stream(device=device) for _ in range(3))

    def h2d_bytes(self):
        return 3 * self.dev[0].numel() * self.dev[0].element_size()

    def d2h_bytes(self):
        return self.dev[3].numel() * self.dev[3].element_size()

    def start(self, event):
        """Record `event` before the next call's first copy."""
        event.record(self.s_in)

    def end(self, event):
        """Record `event` after everything issued so far (the last output copy comes last)."""
        event.record(self.s_out)

    def __call__(self, q_host, k_host, v_host, o_host):
        q, k, v, o = self.dev
        return squad_attn_fwd_host(q_host, k_host, v_host, o_host, q, k, v, o, self.ws, self.grid, self.window,
                                   self.order, groups=self.groups, copy_in=self.s_in, compute=self.s_comp,
                                   copy_out=self.s_out)
