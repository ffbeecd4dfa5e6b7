"""Python binding of the B200 DECO MoE FFN library (libdeco_moe.so).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  Importing
this package loads the in-tree shared library and fails loudly if it is
missing; there is no fallback implementation.

The C ABI and the layer's definition are documented in include/deco_moe.h.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdeco_moe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python sparse_moe_ffn_relu_b200/build.py` "
        "(the DECO MoE layer has no non-CUDA implementation)")
_lib = ctypes.CDLL(LIB_PATH)

DECO_F32, DECO_BF16 = 0, 1
_DT = {torch.float32: DECO_F32, torch.bfloat16: DECO_BF16}
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "workspace", 4: "cuda", 5: "device"}


class DecoError(RuntimeError):
    def __init__(self, code: int, what: str):
        msg = f"{what}: {_lib.deco_status_string(code).decode()} (status {code})"
        if code == 4:
            msg += f" -- {_lib.deco_last_cuda_error().decode()}"
        super().__init__(msg)
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("d_model", ctypes.c_int), ("E", ctypes.c_int),
                ("d_e", ctypes.c_int), ("d_s", ctypes.c_int), ("dtype", ctypes.c_int),
                ("rms_eps", ctypes.c_float), ("residual", ctypes.c_int), ("topk", ctypes.c_int),
                ("gated", ctypes.c_int), ("experts_on_host", ctypes.c_int)]


WEIGHT_NAMES = ("W_r", "b_r", "W_up", "W_bar_up", "W_down", "s", "W_s_up", "W_s_down", "W_val")


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_NAMES]


GRAD_NAMES = ("dx", "dW_r", "db_r", "dW_up", "dW_down", "ds", "dW_s_up", "dW_s_down", "dW_val")


class Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in GRAD_NAMES]


class Routing(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("r", "active", "counts", "offsets", "perm", "n_tok")]


_vp, _sz = ctypes.c_void_p, ctypes.c_size_t
_sig = {
    "deco_moe_workspace_size": [ctypes.POINTER(Shape), ctypes.POINTER(_sz)],
    "deco_moe_forward": [ctypes.POINTER(Shape), _vp, ctypes.POINTER(Weights), _vp, _vp, _sz, _vp],
    "deco_moe_routing": [ctypes.POINTER(Shape), _vp, ctypes.POINTER(Weights),
                         ctypes.POINTER(Routing), _vp, _sz, _vp],
    "deco_moe_mean_up": [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp],
    "deco_dense_ffn_workspace_size": [ctypes.c_int] * 4 + [ctypes.POINTER(_sz)],
    "deco_dense_ffn_forward": [ctypes.c_int] * 4 + [_vp] * 4 + [_vp, _sz, _vp],
    "deco_moe_device_error": [_vp, ctypes.POINTER(ctypes.c_int), _vp],
    "deco_moe_set_profiling": [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int],
    "deco_moe_forward_static": [ctypes.POINTER(Shape), _vp, ctypes.POINTER(Weights), _vp, _vp],
    "deco_moe_static_device_error": [ctypes.POINTER(ctypes.c_int), _vp],
    "deco_set_wait_limit": [ctypes.c_longlong],
    "deco_moe_backward_workspace_size": [ctypes.POINTER(Shape), ctypes.POINTER(_sz)],
    "deco_moe_backward": [ctypes.POINTER(Shape), _vp, ctypes.POINTER(Weights), _vp, _vp,
                          ctypes.POINTER(Grads), _vp, _sz, _vp],
    "deco_moe_router_entropy": [ctypes.c_int, ctypes.c_int, _vp, _vp, ctypes.c_float, _vp, _vp, _vp],
    "deco_sparsity_controller": [ctypes.POINTER(ctypes.c_double), ctypes.c_double, ctypes.c_double,
                                 ctypes.c_double],
}
for _name, _args in _sig.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = ctypes.c_int
_lib.deco_status_string.argtypes = [ctypes.c_int]
_lib.deco_status_string.restype = ctypes.c_char_p
_lib.deco_last_cuda_error.argtypes = []
_lib.deco_last_cuda_error.restype = ctypes.c_char_p

# every symbol include/deco_moe.h declares
EXPORTS = tuple(_sig) + ("deco_status_string", "deco_last_cuda_error")


def _check(code: int, what: str):
    if code != 0:
        raise DecoError(code, what)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_shape(T, D, E, d_e, d_s, dtype, eps=1e-6, residual=False, topk=0, gated=False,
               experts_on_host=False) -> Shape:
    return Shape(T, D, E, d_e, d_s, _DT[dtype] if isinstance(dtype, torch.dtype) else dtype,
                 eps, int(bool(residual)), int(topk), int(bool(gated)), int(bool(experts_on_host)))


def _weights(L: dict) -> Weights:
    return Weights(*[_ptr(L.get(n)) for n in WEIGHT_NAMES])


def layer_shape(x: torch.Tensor, L: dict, eps=1e-6, residual=False, topk=0) -> Shape:
    """The shape of a call; routed experts held in pinned host tensors (W_up,
    W_down, W_val on the CPU, pin_memory) select experts_on_host."""
    E, d_e, D = L["W_up"].shape if "W_up" in L else (L["W_r"].shape[0], 64, x.shape[1])
    d_s = L["W_s_up"].shape[0] if "W_s_up" in L else 64
    on_host = "W_up" in L and L["W_up"].device.type == "cpu"
    return make_shape(x.shape[0], x.shape[1], L["W_r"].shape[0], d_e, d_s, x.dtype, eps, residual,
                      topk, "W_val" in L, on_host)


def workspace_size(shape: Shape) -> int:
    n = _sz(0)
    _check(_lib.deco_moe_workspace_size(ctypes.byref(shape), ctypes.byref(n)), "workspace_size")
    return n.value


def alloc_workspace(shape: Shape, device="cuda") -> torch.Tensor:
    return torch.empty(max(workspace_size(shape), 256), dtype=torch.uint8, device=device)


def forward(x: torch.Tensor, L: dict, out=None, workspace=None, eps=1e-6, residual=False,
            stream=None, topk=0) -> torch.Tensor:
    """out = DECO MoE layer(x) (+ x if residual).  L: dict of device tensors.
    topk > 0 replaces ReLU routing by the TopK baseline with k = topk."""
    shape = layer_shape(x, L, eps, residual, topk)
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        workspace = alloc_workspace(shape, x.device)
    w = _weights(L)
    _check(_lib.deco_moe_forward(ctypes.byref(shape), _ptr(x), ctypes.byref(w), _ptr(out),
                                 _ptr(workspace), workspace.numel(), _stream(stream)), "forward")
    return out


STATIC_SCRATCH_BYTES = 64 << 20


def forward_static(x: torch.Tensor, L: dict, out=None, eps=1e-6, residual=False,
                   stream=None) -> torch.Tensor:
    """forward() on the library's built-in 64 MiB device scratch instead of a
    workspace, for callers that cannot allocate device memory while running
    layers.  Calls on one device share that scratch: do not let them overlap
    on the GPU.  The first call on a device should come before any stream
    capture.  Raises DecoError (status 3) if the shape needs more scratch."""
    shape = layer_shape(x, L, eps, residual)
    if out is None:
        out = torch.empty_like(x)
    w = _weights(L)
    _check(_lib.deco_moe_forward_static(ctypes.byref(shape), _ptr(x), ctypes.byref(w), _ptr(out),
                                        _stream(stream)), "forward_static")
    return out


def routing(x: torch.Tensor, L: dict, workspace=None, stream=None, topk=0) -> dict:
    """Router + token->expert tables; returns r, active, counts, offsets, perm, n_tok."""
    T, E = x.shape[0], L["W_r"].shape[0]
    shape = layer_shape(x, L, topk=topk)
    if workspace is None:
        workspace = alloc_workspace(shape, x.device)
    dev = x.device
    res = dict(r=torch.empty(T, E, dtype=torch.float32, device=dev),
               active=torch.empty(T, E, dtype=torch.uint8, device=dev),
               counts=torch.empty(E, dtype=torch.int32, device=dev),
               offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               perm=torch.empty(max(T * E, 1), dtype=torch.int32, device=dev),
               n_tok=torch.empty(max(T, 1), dtype=torch.int32, device=dev))
    out = Routing(*[_ptr(res[n]) for n in ("r", "active", "counts", "offsets", "perm", "n_tok")])
    w = _weights(L)
    _check(_lib.deco_moe_routing(ctypes.byref(shape), _ptr(x), ctypes.byref(w), ctypes.byref(out),
                                 _ptr(workspace), workspace.numel(), _stream(stream)), "routing")
    return res


def mean_up(W_up: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """W_bar_up = mean over experts of W_up [E, d_e, D] (fp64 sum, one rounding)."""
    E, d_e, D = W_up.shape
    if out is None:
        out = torch.empty(d_e, D, dtype=W_up.dtype, device=W_up.device)
    _check(_lib.deco_moe_mean_up(E, d_e, D, _DT[W_up.dtype], _ptr(W_up), _ptr(out),
                                 _stream(stream)), "mean_up")
    return out


def dense_workspace_size(T, D, d_ff, dtype) -> int:
    n = _sz(0)
    _check(_lib.deco_dense_ffn_workspace_size(T, D, d_ff, _DT[dtype], ctypes.byref(n)),
           "dense_ffn_workspace_size")
    return n.value


def dense_ffn(x, W1, W2, out=None, workspace=None, stream=None) -> torch.Tensor:
    """out = W2 SiLU(W1 x), the equal-parameter dense FFN baseline."""
    T, D = x.shape
    d_ff = W1.shape[0]
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        workspace = torch.empty(dense_workspace_size(T, D, d_ff, x.dtype), dtype=torch.uint8,
                                device=x.device)
    _check(_lib.deco_dense_ffn_forward(T, D, d_ff, _DT[x.dtype], _ptr(x), _ptr(W1), _ptr(W2),
                                       _ptr(out), _ptr(workspace), workspace.numel(),
                                       _stream(stream)), "dense_ffn")
    return out


# timing slots of deco_moe_set_profiling: slot i is bracketed by events 2i and
# 2i+1.  The general path fills route..down, the prefill path (bf16, T > 16)
# route..combine, the decode path (bf16, T <= 16) only "layer" (one kernel).
KERNELS = ("route", "count", "scatter", "up", "down")
PREFILL_KERNELS = KERNELS + ("proj", "shared", "combine")
ALL_SLOTS = PREFILL_KERNELS + ("layer",)


def set_profiling(events):
    """Record events[2i] / events[2i+1] around the i-th kernel of every later
    forward call (a list of torch.cuda.Event, len 2*len(KERNELS)); None stops."""
    global _prof_keep
    if events is None:
        _prof_keep = None
        _check(_lib.deco_moe_set_profiling(None, 0), "set_profiling")
        return
    handles = [e.cuda_event for e in events]
    if not all(handles):
        raise ValueError("set_profiling: every event must exist (record it once first)")
    arr = (ctypes.c_void_p * len(events))(*handles)
    _prof_keep = (arr, events)
    _check(_lib.deco_moe_set_profiling(arr, len(events)), "set_profiling")


_prof_keep = None


def device_error(workspace, stream=None) -> int:
    code = ctypes.c_int(0)
    _check(_lib.deco_moe_device_error(_ptr(workspace), ctypes.byref(code), _stream(stream)),
           "device_error")
    return code.value


def static_device_error(stream=None) -> int:
    """The device error word of the last forward_static call on this device (cleared)."""
    code = ctypes.c_int(0)
    _check(_lib.deco_moe_static_device_error(ctypes.byref(code), _stream(stream)),
           "static_device_error")
    return code.value


def set_wait_limit(cycles: int):
    """Test hook: kernels give up waits for data after `cycles` SM cycles (0: default)."""
    _check(_lib.deco_set_wait_limit(int(cycles)), "set_wait_limit")


# --------------------------------------------------------------------------
# training side

def backward(x: torch.Tensor, L: dict, dy: torch.Tensor, dz_extra=None, workspace=None, eps=1e-6,
             residual=False, stream=None) -> dict:
    """Gradients of the loss through the layer given dy = dLoss/dout: a dict
    of fp32 tensors dx, dW_r, db_r, dW_up (with the mean up-projection's
    share), dW_down, ds, dW_s_up, dW_s_down (and dW_val for gated experts).
    dz_extra [T][E] fp32: an extra gradient on the router logits (see
    router_entropy)."""
    shape = layer_shape(x, L, eps, residual)
    n = _sz(0)
    _check(_lib.deco_moe_backward_workspace_size(ctypes.byref(shape), ctypes.byref(n)), "backward_workspace_size")
    if workspace is None:
        workspace = torch.empty(max(n.value, 256), dtype=torch.uint8, device=x.device)
    f32 = dict(dtype=torch.float32, device=x.device)
    g = {"dx": torch.empty(x.shape, **f32)}
    for name, src in (("dW_r", "W_r"), ("db_r", "b_r"), ("dW_up", "W_up"), ("dW_down", "W_down"),
                      ("ds", "s"), ("dW_s_up", "W_s_up"), ("dW_s_down", "W_s_down"), ("dW_val", "W_val")):
        if src in L:
            g[name] = torch.empty(L[src].shape, **f32)
    gs = Grads(*[_ptr(g.get(n)) for n in GRAD_NAMES])
    w = _weights(L)
    _check(_lib.deco_moe_backward(ctypes.byref(shape), _ptr(x), ctypes.byref(w), _ptr(dy), _ptr(dz_extra),
                                  ctypes.byref(gs), _ptr(workspace), workspace.numel(), _stream(stream)),
           "backward")
    return g


def router_entropy(r: torch.Tensor, active: torch.Tensor, lam: float, stream=None):
    """(H [T+1] with the per-token router entropies and their mean last,
    dz [T][E] = lam * d(mean entropy)/dz) from deco_moe_routing's r and
    active."""
    T, E = r.shape
    H = torch.empty(T + 1, dtype=torch.float32, device=r.device)
    dz = torch.empty(T, E, dtype=torch.float32, device=r.device)
    _check(_lib.deco_moe_router_entropy(T, E, _ptr(r), _ptr(active), float(lam), _ptr(H), _ptr(dz),
                                        _stream(stream)), "router_entropy")
    return H, dz


def sparsity_controller(lam: float, ratio: float, target: float, factor: float = 1.002) -> float:
    """One step of the adaptive sparsity coefficient (x factor above the
    target activation ratio, / factor below)."""
    v = ctypes.c_double(lam)
    _check(_lib.deco_sparsity_controller(ctypes.byref(v), float(ratio), float(target), float(factor)),
           "sparsity_controller")
    return v.value
