"""Python binding of the ISA (In-context Sparse Attention) library: forward and backward.

Thin ctypes layer over ``libisa.so`` (entry points in include/isa.h): it
marshals torch tensor pointers, sizes and the current CUDA stream and turns
status codes into exceptions.  Every step of the computation runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback -- importing
works without a GPU, but any call fails loudly if the library or a CUDA
device is missing.

The method is the sparse attention of "LIVEditor-14B: Lightning Unified
Video Editing via In-Context Sparse Attention" (paper.rainbus.top summary,
"Method steps in detail"):
  plan(...)    steps (1)-(3) + the exact-block choice of step (5)
  forward(...) steps (4)-(6), sharp and flat query blocks in one launch
  backward(...) gradients of steps (4)-(6) with the plan held fixed
  dense(...)   the full attention that ISA replaces
  coarse_residual(...) step (6)'s gamma * O_coarse residual (and its backward)
  IsaAttention torch.autograd.Function over plan + forward (+ residual) / backward
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libisa.so")

ISA_OK = 0
ISA_ERR_INVALID_ARG = 1
ISA_ERR_UNSUPPORTED = 2
ISA_ERR_WORKSPACE = 3
ISA_ERR_CUDA = 4
ISA_ERR_DEVICE_TIMEOUT = 5

# every entry point declared in include/isa.h
EXPORTS = (
    "isa_plan_workspace_size", "isa_plan", "isa_plan_rope", "isa_plan_view_get", "isa_forward", "isa_dense",
    "isa_last_error", "isa_version", "isa_set_wait_timeout_ns", "isa_set_fault_injection",
    "isa_forward_static", "isa_forward_static_status", "isa_rope_workspace_size", "isa_rope", "isa_backward_workspace_size", "isa_backward",
    "isa_coarse_residual", "isa_coarse_residual_backward_workspace_size", "isa_coarse_residual_backward",
)


class IsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"isa status {status}: {message}")
        self.status = status


class Params(ctypes.Structure):
    """isa_params: shapes, the three ratios and the softmax scale (<= 0: 1/sqrt(D))."""
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("D", ctypes.c_int32),
                ("L_src", ctypes.c_int32), ("L_ctx", ctypes.c_int32), ("block", ctypes.c_int32),
                ("alpha_s", ctypes.c_float), ("alpha_f", ctypes.c_float), ("alpha_ns", ctypes.c_float),
                ("scale", ctypes.c_float)]

    def __repr__(self) -> str:
        return ("Params(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")")


class _PlanView(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("T_src", "T_ctx", "T", "K_sel", "T_kv", "n_flat", "n_sharp", "n_exact", "T_kv_pad",
                 "bitmap_words")] + \
               [(n, ctypes.c_void_p) for n in
                ("Qc", "Kc", "Vc", "imp", "ctx_sel", "kept", "energy", "sharp_ids", "flat_ids", "exact",
                 "exact_bits", "Kp", "Vp", "status")]


_lib: Optional[ctypes.CDLL] = None


def load_library() -> ctypes.CDLL:
    """Loads libisa.so once.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise IsaError(ISA_ERR_CUDA, f"{LIB_PATH} is missing; build it with "
                                     "`python -m block_sparse_attention_coarse_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(Params)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.isa_plan_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
    lib.isa_plan.argtypes = [P, vp, vp, vp, vp, sz, vp]
    lib.isa_plan_rope.argtypes = [P, ctypes.c_float, vp, vp, vp, vp, vp, vp, sz, vp, sz, vp]
    lib.isa_plan_view_get.argtypes = [P, vp, sz, ctypes.POINTER(_PlanView)]
    lib.isa_forward.argtypes = [P, vp, vp, vp, vp, sz, vp, vp, vp]
    lib.isa_dense.argtypes = [P, vp, vp, vp, vp, vp, vp, vp]
    lib.isa_last_error.restype = ctypes.c_char_p
    lib.isa_version.restype = ctypes.c_char_p
    lib.isa_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.isa_set_fault_injection.argtypes = [ctypes.c_int32]
    lib.isa_forward_static.argtypes = [P, vp, vp, vp, vp, vp, vp]
    lib.isa_forward_static.restype = ctypes.c_int
    lib.isa_forward_static_status.argtypes = [ctypes.c_int32, vp, vp]
    lib.isa_forward_static_status.restype = ctypes.c_int
    lib.isa_rope_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
    lib.isa_rope.argtypes = [P, ctypes.c_float, vp, vp, vp, vp, vp, sz, vp]
    lib.isa_backward_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
    lib.isa_backward.argtypes = [P, vp, vp, vp, vp, sz, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.isa_coarse_residual.argtypes = [P, ctypes.c_float, vp, sz, vp, vp]
    lib.isa_coarse_residual_backward_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
    lib.isa_coarse_residual_backward.argtypes = [P, ctypes.c_float, vp, sz, vp, vp, vp, vp, vp, vp, sz, vp]
    for name in ("isa_plan_workspace_size", "isa_plan", "isa_plan_rope", "isa_plan_view_get", "isa_forward",
                 "isa_dense",
                 "isa_set_wait_timeout_ns", "isa_set_fault_injection", "isa_rope_workspace_size", "isa_rope",
                 "isa_backward_workspace_size", "isa_backward", "isa_coarse_residual",
                 "isa_coarse_residual_backward_workspace_size", "isa_coarse_residual_backward"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != ISA_OK:
        raise IsaError(status, load_library().isa_last_error().decode())


def make_params(B: int, H: int, D: int, L_src: int, L_ctx: int, block: int = 64, alpha_s: float = 0.125,
                alpha_f: float = 0.5, alpha_ns: float = 0.0625, scale: float = 0.0) -> Params:
    return Params(B, H, D, L_src, L_ctx, block, alpha_s, alpha_f, alpha_ns, scale)


def version() -> str:
    return load_library().isa_version().decode()


def workspace_size(p: Params) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().isa_plan_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return n.value


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check_qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, p: Params) -> None:
    shape = (p.B, p.H, p.L_src + p.L_ctx, p.D)
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda:
            raise IsaError(ISA_ERR_INVALID_ARG, f"{name} must be a CUDA tensor")
        if t.dtype != torch.bfloat16 or tuple(t.shape) != shape or not t.is_contiguous():
            raise IsaError(ISA_ERR_INVALID_ARG, f"{name} must be contiguous bfloat16 {shape}, "
                                                f"got {t.dtype} {tuple(t.shape)}")


def alloc_workspace(p: Params, device=None) -> torch.Tensor:
    return torch.empty(workspace_size(p), dtype=torch.uint8, device=device or "cuda")


def plan(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, p: Params, ws: Optional[torch.Tensor] = None,
         stream=None) -> torch.Tensor:
    """Runs the planning kernels; returns the workspace holding the plan."""
    _check_qkv(q, k, v, p)
    if ws is None:
        ws = alloc_workspace(p, q.device)
    _check(load_library().isa_plan(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), ws.data_ptr(),
                                   ws.numel(), _stream(stream)))
    return ws


def plan_rope(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, p: Params, base: float = 10000.0,
              ws: Optional[torch.Tensor] = None, inplace: bool = False, rope_ws: Optional[torch.Tensor] = None,
              stream=None, q_rot: Optional[torch.Tensor] = None, k_rot: Optional[torch.Tensor] = None):
    """Decoupled RoPE of q and k folded into the planning pass (isa_plan_rope);
    returns (ws, q_rot, k_rot): the plan and the rotated q and k that
    `forward` takes with v.  q_rot, k_rot are the given tensors, q / k when
    `inplace`, else new tensors."""
    _check_qkv(q, k, v, p)
    if ws is None:
        ws = alloc_workspace(p, q.device)
    if inplace:
        qo, ko = q, k
    else:
        qo = torch.empty_like(q) if q_rot is None else q_rot
        ko = torch.empty_like(k) if k_rot is None else k_rot
        _check_qkv(qo, ko, ko, p)
    if rope_ws is None:
        rope_ws = torch.empty(rope_workspace_size(p), dtype=torch.uint8, device=q.device)
    _check(load_library().isa_plan_rope(ctypes.byref(p), float(base), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                        qo.data_ptr(), ko.data_ptr(), ws.data_ptr(), ws.numel(), rope_ws.data_ptr(),
                                        rope_ws.numel(), _stream(stream)))
    return ws, qo, ko


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, ws: torch.Tensor, p: Params,
            out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Sparse attention with a plan from `plan`; returns out [B,H,L,D] bf16."""
    _check_qkv(q, k, v, p)
    if out is None:
        out = torch.empty_like(q)
    _check(load_library().isa_forward(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), ws.data_ptr(),
                                      ws.numel(), out.data_ptr(), lse.data_ptr() if lse is not None else None,
                                      _stream(stream)))
    return out


def dense(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, p: Params, out: Optional[torch.Tensor] = None,
          lse: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Dense softmax attention over all L tokens with the same kernel machinery."""
    _check_qkv(q, k, v, p)
    if out is None:
        out = torch.empty_like(q)
    _check(load_library().isa_dense(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                    lse.data_ptr() if lse is not None else None,
                                    status.data_ptr() if status is not None else None, _stream(stream)))
    return out


def plan_view(p: Params, ws: torch.Tensor) -> Dict[str, object]:
    """Sizes of the plan and CUDA tensor views of every plan array in `ws`."""
    view = _PlanView()
    _check(load_library().isa_plan_view_get(ctypes.byref(p), ws.data_ptr(), ws.numel(), ctypes.byref(view)))
    BH = p.B * p.H
    base = ws.data_ptr()

    def arr(ptr, dtype, shape):
        n = 1
        for s in shape:
            n *= s
        off = ptr - base
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return ws[off:off + nbytes].view(dtype).view(*shape)

    v = view
    out: Dict[str, object] = {f: getattr(v, f) for f in
                              ("T_src", "T_ctx", "T", "K_sel", "T_kv", "n_flat", "n_sharp", "n_exact", "T_kv_pad",
                               "bitmap_words")}
    out.update(
        Qc=arr(v.Qc, torch.float32, (BH, v.T, p.D)), Kc=arr(v.Kc, torch.float32, (BH, v.T, p.D)),
        Vc=arr(v.Vc, torch.float32, (BH, v.T, p.D)), imp=arr(v.imp, torch.float32, (BH, v.T_ctx)),
        ctx_sel=arr(v.ctx_sel, torch.int32, (BH, v.K_sel)), kept=arr(v.kept, torch.int32, (BH, v.T_kv)),
        energy=arr(v.energy, torch.float32, (BH, v.T)),
        sharp_ids=arr(v.sharp_ids, torch.int32, (BH, v.n_sharp)),
        flat_ids=arr(v.flat_ids, torch.int32, (BH, v.n_flat)),
        exact=arr(v.exact, torch.int32, (BH, v.n_flat, v.n_exact)),
        exact_bits=arr(v.exact_bits, torch.int32, (BH, v.n_flat, v.bitmap_words)),
        Kp=arr(v.Kp, torch.bfloat16, (BH, v.T_kv_pad, p.D)), Vp=arr(v.Vp, torch.bfloat16, (BH, v.T_kv_pad, p.D)),
        status=arr(v.status, torch.int32, (1,)),
    )
    return out


def rope_workspace_size(p: Params) -> int:
    n = ctypes.c_size_t()
    _check(load_library().isa_rope_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return n.value


def rope(q: torch.Tensor, k: torch.Tensor, p: Params, base: float = 10000.0, inplace: bool = False,
         ws: Optional[torch.Tensor] = None, stream=None, q_out: Optional[torch.Tensor] = None,
         k_out: Optional[torch.Tensor] = None):
    """Decoupled rotary position embedding of q and k (positions restart at 0
    in the context segment); returns the rotated (q, k): q_out / k_out when
    given, q / k when `inplace`, else new tensors."""
    _check_qkv(q, k, k, p)
    if inplace:
        qo, ko = q, k
    else:
        qo = torch.empty_like(q) if q_out is None else q_out
        ko = torch.empty_like(k) if k_out is None else k_out
        _check_qkv(qo, ko, ko, p)
    if ws is None:
        ws = torch.empty(rope_workspace_size(p), dtype=torch.uint8, device=q.device)
    _check(load_library().isa_rope(ctypes.byref(p), float(base), q.data_ptr(), k.data_ptr(), qo.data_ptr(),
                                   ko.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)))
    return qo, ko


def backward_workspace_size(p: Params) -> int:
    n = ctypes.c_size_t()
    _check(load_library().isa_backward_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return n.value


def backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, ws: torch.Tensor, p: Params, out: torch.Tensor,
             lse: torch.Tensor, dout: torch.Tensor, dq: Optional[torch.Tensor] = None,
             dk: Optional[torch.Tensor] = None, dv: Optional[torch.Tensor] = None,
             bws: Optional[torch.Tensor] = None, stream=None):
    """Gradients (dq, dk, dv) of sum(dout * out) for the forward that produced
    `out` and `lse` from (q, k, v) with the plan in `ws`."""
    _check_qkv(q, k, v, p)
    _check_qkv(out, dout, out, p)
    L = p.L_src + p.L_ctx
    if not lse.is_cuda or lse.dtype != torch.float32 or tuple(lse.shape) != (p.B, p.H, L) or not lse.is_contiguous():
        raise IsaError(ISA_ERR_INVALID_ARG, f"lse must be contiguous float32 {(p.B, p.H, L)}")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_qkv(dq, dk, dv, p)
    if bws is None:
        bws = torch.empty(backward_workspace_size(p), dtype=torch.uint8, device=q.device)
    _check(load_library().isa_backward(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), ws.data_ptr(),
                                       ws.numel(), out.data_ptr(), lse.data_ptr(), dout.data_ptr(), dq.data_ptr(),
                                       dk.data_ptr(), dv.data_ptr(), bws.data_ptr(), bws.numel(), _stream(stream)))
    return dq, dk, dv


def coarse_residual(out: torch.Tensor, ws: torch.Tensor, p: Params, gamma: float, stream=None) -> torch.Tensor:
    """out += gamma * O_coarse in place (step (6)'s low-frequency residual:
    block-level softmax(Qc Kc^T s) Vc of the plan in `ws`, broadcast to each
    token of its query block); returns out."""
    _check_qkv(out, out, out, p)
    _check(load_library().isa_coarse_residual(ctypes.byref(p), float(gamma), ws.data_ptr(), ws.numel(),
                                              out.data_ptr(), _stream(stream)))
    return out


def coarse_residual_backward_workspace_size(p: Params) -> int:
    n = ctypes.c_size_t()
    _check(load_library().isa_coarse_residual_backward_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return n.value


def coarse_residual_backward(ws: torch.Tensor, p: Params, gamma: float, dout: torch.Tensor, dq: torch.Tensor,
                             dk: torch.Tensor, dv: torch.Tensor, dgamma: Optional[torch.Tensor] = None,
                             cws: Optional[torch.Tensor] = None, stream=None):
    """Adds the residual's gradients to dq, dk, dv in place and writes the
    per-head gradient of gamma to `dgamma` (fp32 [B, H], if given)."""
    _check_qkv(dq, dk, dv, p)
    _check_qkv(dout, dout, dout, p)
    if cws is None:
        cws = torch.empty(coarse_residual_backward_workspace_size(p), dtype=torch.uint8, device=dq.device)
    if dgamma is not None and (dgamma.dtype != torch.float32 or dgamma.numel() != p.B * p.H or not dgamma.is_cuda):
        raise IsaError(ISA_ERR_INVALID_ARG, "dgamma must be a CUDA float32 tensor of B*H elements")
    _check(load_library().isa_coarse_residual_backward(
        ctypes.byref(p), float(gamma), ws.data_ptr(), ws.numel(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
        dv.data_ptr(), dgamma.data_ptr() if dgamma is not None else None, cws.data_ptr(), cws.numel(),
        _stream(stream)))
    return dq, dk, dv, dgamma


class IsaAttention(torch.autograd.Function):
    """ISA as a differentiable op: forward = plan + sparse attention (keeping
    the plan, output and lse), plus gamma * O_coarse when gamma != 0;
    backward = the library's backward with that plan (and the residual's).
    Call as IsaAttention.apply(q, k, v, p, gamma); inputs are contiguous
    bf16 CUDA tensors [B, H, L, D]; gamma is a constant (0.0: no residual;
    its gradient is available from coarse_residual_backward)."""

    @staticmethod
    def forward(ctx, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, p: Params, gamma: float):
        ws = plan(q, k, v, p)
        lse = torch.empty(p.B, p.H, p.L_src + p.L_ctx, dtype=torch.float32, device=q.device)
        out = forward(q, k, v, ws, p, lse=lse)
        ctx.save_for_backward(q, k, v, ws, out, lse)
        ctx.p, ctx.gamma = p, float(gamma)
        if gamma != 0.0:
            return coarse_residual(out.clone(), ws, p, gamma)
        return out

    @staticmethod
    def backward(ctx, dout: torch.Tensor):
        q, k, v, ws, out, lse = ctx.saved_tensors
        dout = dout.contiguous()
        dq, dk, dv = backward(q, k, v, ws, ctx.p, out, lse, dout)
        if ctx.gamma != 0.0:
            coarse_residual_backward(ws, ctx.p, ctx.gamma, dout, dq, dk, dv)
        return dq, dk, dv, None, None


_COPY_STREAMS: Dict[int, tuple] = {}


def _copy_streams(dev: torch.device):
    """Host-to-device and device-to-host copy streams of a device (created once)."""
    if dev.index not in _COPY_STREAMS:
        _COPY_STREAMS[dev.index] = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    return _COPY_STREAMS[dev.index]


def isa_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, p: Params, ws: Optional[torch.Tensor] = None,
                  device=None, rope_base: Optional[float] = None, out: Optional[torch.Tensor] = None,
                  chunks: int = 8) -> torch.Tensor:
    """The user-level call: plan + forward, with the decoupled RoPE of q and
    k folded into the planning pass when `rope_base` is given.

    CUDA inputs stay on the device (returns a new device tensor).  CPU
    inputs (pinned, [B, H, L, D] bf16) are processed in `chunks` contiguous
    slices of the B*H heads -- heads are independent -- so that the copies
    of one slice overlap the kernels of the others: host-to-device copies
    on one stream, planning and attention on the current stream,
    device-to-host copies into `out` (a pinned CPU tensor, allocated if not
    given) on a third.  The current stream waits for the last copy, so
    synchronising it makes `out` complete."""
    if q.is_cuda:
        if rope_base is not None:
            ws, q, k = plan_rope(q, k, v, p, rope_base, ws)
        else:
            ws = plan(q, k, v, p, ws)
        return forward(q, k, v, ws, p)
    dev = torch.device(device or "cuda")
    if dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    BH, L, D = p.B * p.H, p.L_src + p.L_ctx, p.D
    shape = (p.B, p.H, L, D)
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.is_cuda or t.dtype != torch.bfloat16 or tuple(t.shape) != shape or not t.is_contiguous():
            raise IsaError(ISA_ERR_INVALID_ARG, f"{name} must be a contiguous CPU bfloat16 {shape} tensor")
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
    elif out.is_cuda or out.dtype != torch.bfloat16 or tuple(out.shape) != shape or not out.is_contiguous():
        raise IsaError(ISA_ERR_INVALID_ARG, f"out must be a contiguous CPU bfloat16 {shape} tensor")
    n = max(1, min(BH, int(chunks)))
    bounds = [BH * c // n for c in range(n + 1)]
    sub = lambda h: make_params(1, h, D, p.L_src, p.L_ctx, p.block, p.alpha_s, p.alpha_f, p.alpha_ns, p.scale)
    hmax = max(bounds[c + 1] - bounds[c] for c in range(n))
    if ws is None or ws.numel() < workspace_size(sub(hmax)):
        ws = alloc_workspace(sub(hmax), dev)
    h2d, d2h = _copy_streams(dev)
    compute = torch.cuda.current_stream(dev)
    q3, k3, v3, o3 = (t.view(BH, L, D) for t in (q, k, v, out))
    for c in range(n):
        lo, hi = bounds[c], bounds[c + 1]
        if hi == lo:
            continue
        pc = sub(hi - lo)
        with torch.cuda.stream(h2d):
            qd, kd, vd = (t[lo:hi].unsqueeze(0).to(dev, non_blocking=True) for t in (q3, k3, v3))
            ready = torch.cuda.Event()
            ready.record(h2d)
        compute.wait_event(ready)
        for t in (qd, kd, vd):
            t.record_stream(compute)
        with torch.cuda.stream(compute):
            if rope_base is not None:
                plan_rope(qd, kd, vd, pc, rope_base, ws, inplace=True)
            else:
                plan(qd, kd, vd, pc, ws)
            od = forward(qd, kd, vd, ws, pc)
            done = torch.cuda.Event()
            done.record(compute)
        d2h.wait_event(done)
        od.record_stream(d2h)
        with torch.cuda.stream(d2h):
            o3[lo:hi].copy_(od[0], non_blocking=True)
    copied = torch.cuda.Event()
    copied.record(d2h)
    compute.wait_event(copied)
    return out


def set_wait_timeout_ns(ns: int) -> None:
    _check(load_library().isa_set_wait_timeout_ns(int(ns)))


def set_fault_injection(mode: int) -> None:
    _check(load_library().isa_set_fault_injection(int(mode)))
