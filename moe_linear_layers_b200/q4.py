"""Thin Python binding of the C ABI in include/q4.h (argument marshalling only).

Every step of the computation runs in the CUDA library ``libq4.so``; this module only passes device
pointers (``tensor.data_ptr()``), sizes and the current CUDA stream.  PyTorch provides device memory
and streams.  There is no fallback: if the library is missing, importing this module fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# Q4_DEBUG_LIBRARY=1 loads the debug build (bounds-checked kernels, Q4_ERR_BOUNDS) instead of the release one
LIB_PATH = os.path.join(_HERE, "libq4_debug.so" if os.environ.get("Q4_DEBUG_LIBRARY") == "1" else "libq4.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m moe_linear_layers_b200.build_lib`")

_lib = ctypes.CDLL(LIB_PATH)

Q4_OK = 0
Q4_ERR_NULL = -1
Q4_ERR_SHAPE = -2
Q4_ERR_ALIGN = -3
Q4_ERR_UNSUPPORTED = -4
Q4_ERR_WORKSPACE = -5
Q4_ERR_CUDA = -6
Q4_ERR_NONFINITE = -7
Q4_ERR_TIMEOUT = -8
Q4_ERR_BOUNDS = -9
Q4_OUT_F32 = 0
Q4_OUT_BF16 = 1

EXPORTED = ("q4_status_string", "q4_version", "q4_build_flags", "q4_last_cuda_error_string", "q4_quantize_pack", "q4_linear_w4a16", "q4_linear_w4a16_max_gemv_m",
            "q4_linear_w4a16_grouped", "q4_linear_w4a16_swiglu",
            "act_quant_per_token", "q4_linear_w4a8", "moe_q4_workspace_size", "moe_q4_forward",
            "moe_q4_forward_noalloc", "moe_q4_workspace_size_ex", "moe_q4_forward_ex", "q4_selftest_bounded_wait",
            "act_quant_per_token_f16", "moe_q4_workspace_size_a8", "moe_q4_forward_a8", "moe_q4_forward_classes",
            "moe_q4_forward_range", "q4_linear_w4a16_chain_sync_bytes", "q4_linear_w4a16_chain",
            "moe_q4_route_workspace_size", "moe_q4_route", "moe_q4_rows_workspace_size", "moe_q4_forward_rows",
            "moe_q4_combine", "q4_linear_workspace_size", "q4_linear_w4a16_ws", "q4_linear_w4a8_ws")
Q4_MOE_NOALLOC_SCRATCH_BYTES = 32 << 20


class q4_weight(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int32), ("k", ctypes.c_int32), ("group", ctypes.c_int32),
                ("symmetric", ctypes.c_int32), ("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("zeros", ctypes.c_void_p)]


_i32, _p, _sz = ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t
_lib.q4_status_string.restype = ctypes.c_char_p
_lib.q4_status_string.argtypes = [ctypes.c_int]
_lib.q4_version.restype = ctypes.c_int
_lib.q4_build_flags.restype = ctypes.c_int
_lib.q4_last_cuda_error_string.restype = ctypes.c_char_p
_lib.q4_linear_w4a16_max_gemv_m.restype = ctypes.c_int
_lib.q4_quantize_pack.argtypes = [_p, _i32, _i32, _i32, _i32, _p, _p, _p, _p, _p]
_lib.q4_linear_w4a16.argtypes = [_p, _i32, ctypes.POINTER(q4_weight), _p, _i32, _p, _p]
_lib.q4_linear_w4a16_swiglu.argtypes = [_p, _p, _i32, ctypes.POINTER(q4_weight), _p, _i32, _p, _p]
_lib.q4_linear_w4a16_grouped.argtypes = [_i32, ctypes.POINTER(_p), _i32, ctypes.POINTER(q4_weight),
                                         ctypes.POINTER(_p), _i32, _p, _p]
_lib.act_quant_per_token.argtypes = [_p, _i32, _i32, _p, _p, _p, _p]
_lib.act_quant_per_token_f16.argtypes = [_p, _i32, _i32, _p, _p, _p, _p]
_lib.q4_linear_w4a8.argtypes = [_p, _p, _i32, ctypes.POINTER(q4_weight), _p, _i32, _p, _p, _p]
_lib.q4_linear_workspace_size.restype = _sz
_lib.q4_linear_workspace_size.argtypes = [_i32, ctypes.POINTER(q4_weight)]
_lib.q4_linear_w4a16_ws.argtypes = [_p, _i32, ctypes.POINTER(q4_weight), _p, _i32, _p, _sz, _p, _p]
_lib.q4_linear_w4a8_ws.argtypes = [_p, _p, _i32, ctypes.POINTER(q4_weight), _p, _i32, _p, _p, _sz, _p, _p]
_lib.moe_q4_workspace_size.restype = _sz
_lib.moe_q4_workspace_size.argtypes = [_i32, _i32, _i32, _i32, _i32]
_lib.moe_q4_forward.argtypes = [_p, _i32, _i32, _p, _p, _i32, _i32, ctypes.POINTER(q4_weight), _i32, _p, _i32,
                                _p, _p, _p, _p, _p, _p, _sz, _p, _p]
_lib.q4_selftest_bounded_wait.argtypes = [_i32, _i32, _p, _p]
_lib.moe_q4_workspace_size_ex.restype = _sz
_lib.moe_q4_workspace_size_ex.argtypes = [_i32, _i32, _i32, _i32, _i32, _i32]
_lib.moe_q4_forward_ex.argtypes = [_p, _i32, _i32, _p, _p, _i32, _i32, ctypes.POINTER(q4_weight), _i32,
                                   ctypes.POINTER(q4_weight), _i32, _p, _i32, _p, _p, _p, _p, _p, _p, _sz, _p, _p]
_lib.moe_q4_workspace_size_a8.restype = _sz
_lib.moe_q4_workspace_size_a8.argtypes = [_i32, _i32, _i32, _i32, _i32, _i32]
_lib.moe_q4_forward_a8.argtypes = [_p, _i32, _i32, _p, _p, _i32, _i32, ctypes.POINTER(q4_weight), _i32, _i32,
                                   _p, _i32, _p, _p, _p, _p, _p, _p, _sz, _p, _p]
_lib.moe_q4_forward_classes.argtypes = [_p, _i32, _i32, _p, _p, _i32, _i32, _i32, ctypes.POINTER(_i32),
                                        ctypes.POINTER(q4_weight), _i32, _p, _i32, _p, _p, _p, _p, _p, _p, _sz, _p, _p]
_lib.moe_q4_forward_range.argtypes = [_p, _i32, _i32, _p, _p, _i32, _i32, _i32, _i32, ctypes.POINTER(q4_weight), _i32,
                                      _p, _p, _p, _p, _p, _p, _p, _sz, _p, _p]
_lib.q4_linear_w4a16_chain_sync_bytes.restype = _sz
_lib.q4_linear_w4a16_chain_sync_bytes.argtypes = [_i32]
_lib.q4_linear_w4a16_chain.argtypes = [_i32, ctypes.POINTER(_i32), ctypes.POINTER(_p), ctypes.POINTER(_p),
                                       ctypes.POINTER(_p), ctypes.POINTER(q4_weight), ctypes.POINTER(_p), _i32, _p, _p,
                                       _p]
_lib.moe_q4_route_workspace_size.restype = _sz
_lib.moe_q4_route_workspace_size.argtypes = [_i32, _i32, _i32]
_lib.moe_q4_route.argtypes = [_p, _i32, _i32, _p, _p, _i32, _i32, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p, _p]
_lib.moe_q4_rows_workspace_size.restype = _sz
_lib.moe_q4_rows_workspace_size.argtypes = [_i32, _i32, _i32, _i32]
_lib.moe_q4_forward_rows.argtypes = [_p, _i32, _i32, _p, _i32, _p, _i32, ctypes.POINTER(q4_weight), _i32, _p, _p, _sz,
                                     _p, _p]
_lib.moe_q4_combine.argtypes = [_p, _i32, _i32, _p, _p, _i32, _i32, _p, _i32, _p, _p]
_lib.moe_q4_forward_noalloc.argtypes = [_p, _i32, _i32, _p, _p, _i32, _i32, ctypes.POINTER(q4_weight), _i32, _p,
                                        _i32, _p, _p, _p, _p, _p, _p, _p]


class Q4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = f"{what}: {status} ({_lib.q4_status_string(status).decode()})"
        if status == Q4_ERR_CUDA:
            msg += ": " + _lib.q4_last_cuda_error_string().decode()
        super().__init__(msg)
        self.status = status


def _check(rc: int, what: str):
    if rc != Q4_OK:
        raise Q4Error(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_raw_current_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
_current_device = getattr(torch._C, "_cuda_getDevice", None)


def _stream(stream=None):
    """The cudaStream_t handle of `stream`, or of torch's current stream on the current device (looked up
    without building a Stream object: a decode step makes dozens of calls, each paying this)."""
    if stream is None:
        if _raw_current_stream is not None and _current_device is not None:
            return _raw_current_stream(_current_device())
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _weights_on(device, *weights):
    """Every Q4Weight of a call lives on the inputs' device (a host or other-device buffer would be read
    through a pointer the kernels cannot use)."""
    for w in weights:
        if w is not None and w.packed.device != device:
            raise ValueError(f"a weight is on {w.packed.device}, the inputs on {device}")


def _hold(stream, *tensors):
    """A call on a stream other than the current one: the caching allocator ties a tensor's memory to the
    stream it was allocated on, so a workspace or output that this wrapper made (and that may be dropped
    while the work is still queued) is marked in use by `stream` too, and is not handed out again before
    that work is done."""
    if stream is not None:
        for t in tensors:
            if t is not None:
                t.record_stream(stream)


def _dev(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _out(y, shape, device, name="y"):
    """Check a caller-supplied output: fp32 or bf16 (the two output dtypes of the ABI), the expected shape,
    contiguous, on the inputs' device.  Returns the ABI's out_dtype code."""
    if not isinstance(y, torch.Tensor):
        raise TypeError(f"{name} must be a CUDA tensor")
    if y.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"{name} must be torch.float32 or torch.bfloat16, got {y.dtype}")
    if tuple(y.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(y.shape)}")
    if not y.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not y.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if y.device != device:
        raise ValueError(f"{name} is on {y.device}, the inputs on {device}")
    return Q4_OUT_BF16 if y.dtype == torch.bfloat16 else Q4_OUT_F32


def _router(router_w, router_bias, H, device):
    """Check the router of a MoE call: router_w fp32 [E][H] and router_bias (fp32 [E], or None) on the
    inputs' device.  Returns E."""
    if router_w.dim() != 2 or router_w.shape[1] != H:
        raise ValueError(f"router_w must have shape [E][{H}], got {tuple(router_w.shape)}")
    if router_w.device != device:
        raise ValueError(f"router_w is on {router_w.device}, the inputs on {device}")
    E = router_w.shape[0]
    if router_bias is not None:
        if not isinstance(router_bias, torch.Tensor) or router_bias.dtype != torch.float32:
            raise TypeError("router_bias must be a torch.float32 tensor (or None)")
        if router_bias.numel() != E or not router_bias.is_contiguous():
            raise ValueError(f"router_bias must be a contiguous tensor of {E} values")
        if router_bias.device != device:
            raise ValueError(f"router_bias is on {router_bias.device}, the inputs on {device}")
    return E


def _workspace(ws, device):
    """Check a caller-supplied workspace: a contiguous uint8 tensor (its numel is its size in bytes) on the
    inputs' device."""
    if not isinstance(ws, torch.Tensor) or ws.dtype != torch.uint8:
        raise TypeError("workspace must be a torch.uint8 tensor")
    if not ws.is_contiguous():
        raise ValueError("workspace must be contiguous")
    if ws.device != device:
        raise ValueError(f"workspace is on {ws.device}, the inputs on {device}")
    return ws


def _numel(t, n, name):
    if t.numel() != n:
        raise ValueError(f"{name} must hold {n} elements, got {t.numel()}")
    return t


def status_string(status: int) -> str:
    return _lib.q4_status_string(status).decode()


def version() -> int:
    return _lib.q4_version()


class Q4Weight:
    """Device buffers of one INT4 weight matrix [n][k] plus its C descriptor."""

    def __init__(self, packed: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor | None, n: int, k: int,
                 group: int, symmetric: bool):
        # the library trusts these sizes: a buffer that is short, strided, of another type or on another
        # device than the sizes say would be read past its end (or from the host) by the kernels
        if n < 0 or k <= 0 or k % 2 or group <= 0 or k % group:
            raise ValueError(f"an INT4 weight needs n >= 0, an even k > 0 and k % group == 0 (n={n}, k={k}, group={group})")
        for t, dt, cnt, name in ((packed, torch.uint8, n * (k // 2), "packed"),
                                 (scales, torch.float16, n * (k // group), "scales"),
                                 (zeros, torch.float16, n * (k // group), "zeros")):
            if t is None:
                if name == "zeros" and not symmetric:
                    raise ValueError("an asymmetric INT4 weight needs its zero points")
                continue
            if not isinstance(t, torch.Tensor) or t.dtype != dt:
                raise TypeError(f"{name} must be a {dt} tensor")
            if not t.is_contiguous() or t.numel() != cnt:
                raise ValueError(f"{name} must be contiguous with {cnt} elements, got {tuple(t.shape)}")
            if t.device != packed.device:
                raise ValueError(f"{name} is on {t.device}, packed on {packed.device}")
        self.packed, self.scales, self.zeros = packed, scales, zeros
        self.n, self.k, self.group, self.symmetric = n, k, group, bool(symmetric)
        self.desc = q4_weight(n, k, group, int(bool(symmetric)), packed.data_ptr(), scales.data_ptr(),
                              zeros.data_ptr() if zeros is not None else None)

    @staticmethod
    def stack(ws) -> "Q4Weight":
        """The weights of several linears with the same k, group and symmetry stacked by rows (e.g. a layer's
        q, k and v projections, which read the same input): y of the stack = the parts' outputs side by
        side.  Quantization is per row and per group along k, so the stack's codes, scales and zero points
        are exactly the parts' rows one after another (copied, no arithmetic)."""
        ws = list(ws)
        w0 = ws[0]
        if any(w.k != w0.k or w.group != w0.group or w.symmetric != w0.symmetric for w in ws):
            raise ValueError("stacked weights must share k, group and symmetry")
        zeros = None if w0.symmetric else torch.cat([w.zeros for w in ws], 0).contiguous()
        return Q4Weight(torch.cat([w.packed for w in ws], 0).contiguous(), torch.cat([w.scales for w in ws], 0).contiguous(),
                        zeros, sum(w.n for w in ws), w0.k, w0.group, w0.symmetric)

    @staticmethod
    def empty(n: int, k: int, group: int, symmetric: bool, device="cuda") -> "Q4Weight":
        packed = torch.empty((n, k // 2), dtype=torch.uint8, device=device)
        scales = torch.empty((n, k // group), dtype=torch.float16, device=device)
        zeros = None if symmetric else torch.empty((n, k // group), dtype=torch.float16, device=device)
        return Q4Weight(packed, scales, zeros, n, k, group, symmetric)


def q4_quantize_pack(w: torch.Tensor, group: int, symmetric: bool, dev_status: torch.Tensor | None = None,
                     out: Q4Weight | None = None, stream=None) -> Q4Weight:
    """RTN group quantization + packing of an fp32 [n][k] CUDA tensor."""
    _dev(w, torch.float32, "w")
    n, k = w.shape
    if out is not None and (out.n, out.k, out.group, out.symmetric) != (n, k, group, bool(symmetric)):
        raise ValueError(f"out holds a [{out.n}][{out.k}] group-{out.group} weight, not [{n}][{k}] group-{group}")
    q = out or Q4Weight.empty(n, k, group, symmetric, device=w.device)
    _weights_on(w.device, q)
    _hold(stream, q.packed, q.scales, q.zeros)
    _check(_lib.q4_quantize_pack(_ptr(w), n, k, group, int(bool(symmetric)), _ptr(q.packed), _ptr(q.scales),
                                 _ptr(q.zeros), _ptr(dev_status), _stream(stream)), "q4_quantize_pack")
    return q


_SPLIT_WS = {}   # device -> the workspace of split-K GEMMs, grown to the largest size asked for


def linear_workspace(m: int, w: Q4Weight, device) -> torch.Tensor | None:
    """A device workspace for q4_linear_w4a16_ws / q4_linear_w4a8_ws at these sizes (None when the shape
    is not split along K), kept per device and grown as needed.  Calls that share it must be ordered on
    one stream; pass your own to run on several streams at once."""
    need = int(_lib.q4_linear_workspace_size(int(m), ctypes.byref(w.desc)))
    if need == 0:
        return None
    ws = _SPLIT_WS.get(device)
    if ws is None or ws.numel() < need:
        ws = torch.empty((need,), dtype=torch.uint8, device=device)
        _SPLIT_WS[device] = ws
    return ws


def q4_linear_w4a16(x: torch.Tensor, w: Q4Weight, out_dtype=torch.float32, y: torch.Tensor | None = None,
                    dev_status: torch.Tensor | None = None, stream=None, workspace="auto") -> torch.Tensor:
    """y[m][n] = x[m][k] . dequant(W)^T; x bf16 CUDA tensor.  workspace: "auto" (the per-device one of
    linear_workspace: a GEMM of few output tiles is split along K), None (never split) or a uint8 tensor."""
    _dev(x, torch.bfloat16, "x")
    _weights_on(x.device, w)
    if x.numel() % w.k:
        raise ValueError(f"x holds {x.numel()} values, not whole rows of k = {w.k}")
    m = x.numel() // w.k
    if y is None:
        y = torch.empty((m, w.n), dtype=out_dtype, device=x.device)
    od = _out(y, (m, w.n), x.device)
    if isinstance(workspace, str):
        workspace = linear_workspace(m, w, x.device) if m > q4_linear_w4a16_max_gemv_m() else None
    if workspace is not None:
        _workspace(workspace, x.device)
    _hold(stream, y, workspace)
    _check(_lib.q4_linear_w4a16_ws(_ptr(x), m, ctypes.byref(w.desc), _ptr(y), od, _ptr(workspace),
                                   workspace.numel() if workspace is not None else 0, _ptr(dev_status),
                                   _stream(stream)), "q4_linear_w4a16")
    return y


def q4_linear_w4a16_swiglu(gate: torch.Tensor, up: torch.Tensor, w: Q4Weight, out_dtype=torch.float32,
                           y: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                           stream=None) -> torch.Tensor:
    """y[m][n] = h[m][k] . dequant(W)^T with h = silu(gate) * up (fp32 CUDA tensors [m][k], m <= 4)."""
    _dev(gate, torch.float32, "gate")
    _dev(up, torch.float32, "up")
    _weights_on(gate.device, w)
    if gate.numel() % w.k:
        raise ValueError(f"gate holds {gate.numel()} values, not whole rows of k = {w.k}")
    _numel(up, gate.numel(), "up")
    m = gate.numel() // w.k
    if y is None:
        y = torch.empty((m, w.n), dtype=out_dtype, device=gate.device)
    od = _out(y, (m, w.n), gate.device)
    _hold(stream, y)
    _check(_lib.q4_linear_w4a16_swiglu(_ptr(gate), _ptr(up), m, ctypes.byref(w.desc), _ptr(y), od, _ptr(dev_status),
                                       _stream(stream)), "q4_linear_w4a16_swiglu")
    return y


class GroupedGemv:
    """Host-side argument arrays for q4_linear_w4a16_grouped, built once and reused (e.g. per layer)."""

    def __init__(self, xs, ws, ys):
        if not (len(xs) == len(ws) == len(ys) and 1 <= len(xs) <= 8):
            raise ValueError("a grouped call takes 1 to 8 problems, as many x, w and y")
        self.count = len(xs)
        _weights_on(xs[0].device, *ws)
        self.m = xs[0].numel() // ws[0].k
        for x, w in zip(xs, ws):
            _numel(x, self.m * w.k, "x")   # every problem has the same m
            if x.device != xs[0].device:
                raise ValueError("every x of a grouped call must be on one device")
        self.keep = (xs, ws, ys)
        self.x = (_p * self.count)(*[t.data_ptr() for t in xs])
        self.w = (q4_weight * self.count)(*[w.desc for w in ws])
        self.y = (_p * self.count)(*[t.data_ptr() for t in ys])
        ods = {_out(y, (self.m, w.n), xs[0].device) for y, w in zip(ys, ws)}
        if len(ods) != 1:
            raise TypeError("every y of a grouped call must have the same dtype")
        self.od = ods.pop()

    def __call__(self, dev_status: torch.Tensor | None = None, stream=None):
        _check(_lib.q4_linear_w4a16_grouped(self.count, self.x, self.m, self.w, self.y, self.od, _ptr(dev_status),
                                            _stream(stream)), "q4_linear_w4a16_grouped")


class GemvChain:
    """A chain of dependent GEMV stages at m = 1 in one launch (q4_linear_w4a16_chain), its argument arrays
    and its stage counters built once.  stages: a list of stages, each a list of problems (x, w, y): x a bf16
    CUDA tensor of w.k values, or a pair (gate, up) of fp32 CUDA tensors of w.k values (the input is then
    silu(gate) * up); w a Q4Weight; y an fp32 (or bf16, the same for every problem) CUDA tensor of w.n values.
    Stage s starts reading its inputs only once every output of the stages before it is written."""

    def __init__(self, stages):
        probs = [pr for st in stages for pr in st]
        if not stages or not probs:
            raise ValueError("a chain needs at least one stage with one problem")
        self.n_stages = len(stages)
        self.count = len(probs)
        begin = [0]
        for st in stages:
            begin.append(begin[-1] + len(st))
        dev = probs[0][2].device
        _weights_on(dev, *[w for _, w, _ in probs])
        ods = set()
        xs, gs, us = [], [], []
        for x, w, y in probs:
            ods.add(_out(y.view(-1), (w.n,), dev))
            for t in (x if isinstance(x, (tuple, list)) else (x,)):
                _numel(t, w.k, "a chain input")   # m = 1: one row of k values
                if t.device != dev:
                    raise ValueError(f"a chain input is on {t.device}, the outputs on {dev}")
            if isinstance(x, (tuple, list)):
                _dev(x[0], torch.float32, "gate")
                _dev(x[1], torch.float32, "up")
                xs.append(None)
                gs.append(x[0].data_ptr())
                us.append(x[1].data_ptr())
            else:
                _dev(x, torch.bfloat16, "x")
                xs.append(x.data_ptr())
                gs.append(None)
                us.append(None)
        if len(ods) != 1:
            raise TypeError("every y of a chain must have the same dtype")
        self.od = ods.pop()
        self.keep = stages
        self.begin = (_i32 * (self.n_stages + 1))(*begin)
        self.x = (_p * self.count)(*xs)
        self.g = (_p * self.count)(*gs)
        self.u = (_p * self.count)(*us)
        self.w = (q4_weight * self.count)(*[w.desc for _, w, _ in probs])
        self.y = (_p * self.count)(*[y.data_ptr() for _, _, y in probs])
        nbytes = int(_lib.q4_linear_w4a16_chain_sync_bytes(self.n_stages))
        self.sync = torch.zeros((nbytes // 4,), dtype=torch.int32, device=dev)

    def reset(self):
        """Zero the stage counters (needed only after a call that reported Q4_ERR_TIMEOUT)."""
        self.sync.zero_()

    def __call__(self, dev_status: torch.Tensor | None = None, stream=None):
        _hold(stream, self.sync)
        _check(_lib.q4_linear_w4a16_chain(self.n_stages, self.begin, self.x, self.g, self.u, self.w, self.y, self.od,
                                          _ptr(self.sync), _ptr(dev_status), _stream(stream)), "q4_linear_w4a16_chain")


def q4_linear_w4a16_grouped(xs, ws, ys, dev_status: torch.Tensor | None = None, stream=None):
    """y[i] = x[i] . dequant(W[i])^T for up to 8 independent small-m problems with the same k, in one launch."""
    for t in xs:
        _dev(t, torch.bfloat16, "x")
    GroupedGemv(xs, ws, ys)(dev_status=dev_status, stream=stream)
    return ys


def q4_linear_w4a16_max_gemv_m() -> int:
    return _lib.q4_linear_w4a16_max_gemv_m()


def act_quant_per_token(x: torch.Tensor, xq: torch.Tensor | None = None, scale_a: torch.Tensor | None = None,
                        dev_status: torch.Tensor | None = None, stream=None):
    """Per-token INT8 quantization of a bf16 (or fp16) [m][k] CUDA tensor -> (xq int8 [m][k], scale_a fp32 [m])."""
    f16 = isinstance(x, torch.Tensor) and x.dtype == torch.float16
    _dev(x, torch.float16 if f16 else torch.bfloat16, "x")
    m, k = x.shape
    xq = torch.empty((m, k), dtype=torch.int8, device=x.device) if xq is None else xq
    scale_a = torch.empty((m,), dtype=torch.float32, device=x.device) if scale_a is None else scale_a
    for t, dt, cnt, name in ((xq, torch.int8, m * k, "xq"), (scale_a, torch.float32, m, "scale_a")):
        _numel(_dev(t, dt, name), cnt, name)
        if t.device != x.device:
            raise ValueError(f"{name} is on {t.device}, x on {x.device}")
    fn = _lib.act_quant_per_token_f16 if f16 else _lib.act_quant_per_token
    _hold(stream, xq, scale_a)
    _check(fn(_ptr(x), m, k, _ptr(xq), _ptr(scale_a), _ptr(dev_status), _stream(stream)),
           "act_quant_per_token_f16" if f16 else "act_quant_per_token")
    return xq, scale_a


def q4_linear_w4a8(xq: torch.Tensor, scale_a: torch.Tensor, w: Q4Weight, out_dtype=torch.float32,
                   y: torch.Tensor | None = None, acc_dbg: torch.Tensor | None = None,
                   dev_status: torch.Tensor | None = None, stream=None, workspace="auto") -> torch.Tensor:
    """y[m][n] = scale_a[m] * sum_g scale_w[n][g] * (xq . (code - zero))_g; zero = 0 for symmetric W.
    workspace: as q4_linear_w4a16's."""
    _dev(xq, torch.int8, "xq")
    _dev(scale_a, torch.float32, "scale_a")
    _weights_on(xq.device, w)
    if xq.numel() % w.k:
        raise ValueError(f"xq holds {xq.numel()} codes, not whole rows of k = {w.k}")
    m = xq.numel() // w.k
    _numel(scale_a, m, "scale_a")
    if acc_dbg is not None:
        _numel(_dev(acc_dbg, torch.int32, "acc_dbg"), m * w.n * (w.k // w.group), "acc_dbg")
    if scale_a.device != xq.device or (acc_dbg is not None and acc_dbg.device != xq.device):
        raise ValueError("xq, scale_a and acc_dbg must be on one device")
    if y is None:
        y = torch.empty((m, w.n), dtype=out_dtype, device=xq.device)
    od = _out(y, (m, w.n), xq.device)
    if isinstance(workspace, str):
        workspace = linear_workspace(m, w, xq.device)
    if workspace is not None:
        _workspace(workspace, xq.device)
    _hold(stream, y, workspace)
    _check(_lib.q4_linear_w4a8_ws(_ptr(xq), _ptr(scale_a), m, ctypes.byref(w.desc), _ptr(y), od, _ptr(acc_dbg),
                                  _ptr(workspace), workspace.numel() if workspace is not None else 0,
                                  _ptr(dev_status), _stream(stream)), "q4_linear_w4a8")
    return y


def q4_selftest_bounded_wait(which: int, limit_us: int, dev_status: torch.Tensor, stream=None) -> None:
    """Launch a wait that nothing satisfies; it records Q4_ERR_TIMEOUT in dev_status after limit_us."""
    _check(_lib.q4_selftest_bounded_wait(which, limit_us, _ptr(dev_status), _stream(stream)), "q4_selftest_bounded_wait")


def moe_q4_workspace_size(T: int, H: int, I: int, E: int, topk: int, I_shared: int = 0, a8_mask: int = 0) -> int:
    if a8_mask:
        if I_shared:
            raise ValueError("the W4A8 expert path takes no shared expert")
        return int(_lib.moe_q4_workspace_size_a8(T, H, I, E, topk, a8_mask))
    if I_shared:
        return int(_lib.moe_q4_workspace_size_ex(T, H, I, E, topk, I_shared))
    return int(_lib.moe_q4_workspace_size(T, H, I, E, topk))


def moe_q4_forward(x: torch.Tensor, router_w: torch.Tensor, router_bias: torch.Tensor | None, topk: int,
                   experts: tuple, I: int, out_dtype=torch.float32, y: torch.Tensor | None = None,
                   workspace: torch.Tensor | None = None, want_routing: bool = False,
                   dev_status: torch.Tensor | None = None, stream=None, shared: tuple | None = None,
                   a8_mask: int = 0):
    """Top-k routed MoE SwiGLU layer with INT4 experts.  experts = (gate, up, down) Q4Weight, stacked by expert;
    shared (optional) = (gate, up, down) Q4Weight of a shared expert every token passes through.
    a8_mask: bit 0 runs gate/up, bit 1 runs down on per-row INT8 activation codes (W4A8; no shared expert).
    Returns y, or (y, topk_ids, topk_w, perm, offsets, counts) when want_routing."""
    _dev(x, torch.bfloat16, "x")
    _dev(router_w, torch.float32, "router_w")
    T, H = x.shape
    dev = x.device
    E = _router(router_w, router_bias, H, dev)
    _weights_on(dev, *experts, *(shared or ()))
    if y is None:
        y = torch.empty((T, H), dtype=out_dtype, device=dev)
    od = _out(y, (T, H), dev)
    I_s = shared[0].n if shared is not None else 0
    ws_bytes = moe_q4_workspace_size(T, H, I, E, topk, I_s, a8_mask)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=dev)
    _workspace(workspace, dev)
    descs = (q4_weight * 3)(*[e.desc for e in experts])
    sdescs = (q4_weight * 3)(*[e.desc for e in shared]) if shared is not None else None
    ids = wts = perm = offs = cnts = None
    if want_routing:
        ids = torch.empty((T, topk), dtype=torch.int32, device=dev)
        wts = torch.empty((T, topk), dtype=torch.float32, device=dev)
        perm = torch.empty((T * topk,), dtype=torch.int32, device=dev)
        offs = torch.empty((E + 1,), dtype=torch.int32, device=dev)
        cnts = torch.empty((E,), dtype=torch.int32, device=dev)
    _hold(stream, y, workspace, ids, wts, perm, offs, cnts)
    if a8_mask:
        _check(_lib.moe_q4_forward_a8(_ptr(x), T, H, _ptr(router_w), _ptr(router_bias), E, topk, descs, I, a8_mask,
                                      _ptr(y), od, _ptr(ids), _ptr(wts), _ptr(perm), _ptr(offs), _ptr(cnts),
                                      _ptr(workspace), workspace.numel(), _ptr(dev_status), _stream(stream)),
               "moe_q4_forward_a8")
    else:
        _check(_lib.moe_q4_forward_ex(_ptr(x), T, H, _ptr(router_w), _ptr(router_bias), E, topk, descs, I, sdescs,
                                      I_s, _ptr(y), od, _ptr(ids), _ptr(wts), _ptr(perm), _ptr(offs), _ptr(cnts),
                                      _ptr(workspace), workspace.numel(), _ptr(dev_status), _stream(stream)),
               "moe_q4_forward")
    if want_routing:
        return y, ids, wts, perm, offs, cnts
    return y


def moe_q4_forward_classes(x: torch.Tensor, router_w: torch.Tensor, router_bias: torch.Tensor | None, topk: int,
                           class_begin, class_experts, I: int, out_dtype=torch.float32, y: torch.Tensor | None = None,
                           workspace: torch.Tensor | None = None, want_routing: bool = False,
                           dev_status: torch.Tensor | None = None, stream=None):
    """moe_q4_forward with expert classes: class c = experts class_begin[c] .. class_begin[c+1]-1, whose
    (gate, up, down) Q4Weight triple class_experts[c] is stacked over the class's experts and has its own
    group size and symmetry."""
    _dev(x, torch.bfloat16, "x")
    _dev(router_w, torch.float32, "router_w")
    T, H = x.shape
    dev = x.device
    E = _router(router_w, router_bias, H, dev)
    n = len(class_experts)
    _weights_on(dev, *[w for trip in class_experts for w in trip])
    if len(class_begin) != n + 1:
        raise ValueError("class_begin needs one more entry than there are classes")
    if y is None:
        y = torch.empty((T, H), dtype=out_dtype, device=dev)
    od = _out(y, (T, H), dev)
    if workspace is None:
        workspace = torch.empty((max(moe_q4_workspace_size(T, H, I, E, topk), 1),), dtype=torch.uint8, device=dev)
    _workspace(workspace, dev)
    begin = (_i32 * (n + 1))(*[int(v) for v in class_begin])
    descs = (q4_weight * (3 * n))(*[w.desc for trip in class_experts for w in trip])
    ids = wts = perm = offs = cnts = None
    if want_routing:
        ids = torch.empty((T, topk), dtype=torch.int32, device=dev)
        wts = torch.empty((T, topk), dtype=torch.float32, device=dev)
        perm = torch.empty((T * topk,), dtype=torch.int32, device=dev)
        offs = torch.empty((E + 1,), dtype=torch.int32, device=dev)
        cnts = torch.empty((E,), dtype=torch.int32, device=dev)
    _hold(stream, y, workspace, ids, wts, perm, offs, cnts)
    _check(_lib.moe_q4_forward_classes(_ptr(x), T, H, _ptr(router_w), _ptr(router_bias), E, topk, n, begin, descs,
                                       I, _ptr(y), od, _ptr(ids), _ptr(wts), _ptr(perm), _ptr(offs), _ptr(cnts),
                                       _ptr(workspace), workspace.numel(), _ptr(dev_status), _stream(stream)),
           "moe_q4_forward_classes")
    if want_routing:
        return y, ids, wts, perm, offs, cnts
    return y


def moe_q4_forward_range(x: torch.Tensor, router_w: torch.Tensor, router_bias: torch.Tensor | None, topk: int,
                         e_begin: int, e_end: int, experts: tuple, I: int, y: torch.Tensor | None = None,
                         workspace: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """The contribution of experts e_begin .. e_end-1 (weights stacked over that range) to the MoE layer,
    fp32 [T][H]; disjoint ranges covering every expert sum to the layer."""
    _dev(x, torch.bfloat16, "x")
    _dev(router_w, torch.float32, "router_w")
    T, H = x.shape
    E = _router(router_w, router_bias, H, x.device)
    _weights_on(x.device, *experts)
    if y is None:
        y = torch.empty((T, H), dtype=torch.float32, device=x.device)
    _dev(y, torch.float32, "y")
    _out(y, (T, H), x.device)
    if workspace is None:
        workspace = torch.empty((max(moe_q4_workspace_size(T, H, I, E, topk), 1),), dtype=torch.uint8, device=x.device)
    _workspace(workspace, x.device)
    descs = (q4_weight * 3)(*[e.desc for e in experts])
    _hold(stream, y, workspace)
    _check(_lib.moe_q4_forward_range(_ptr(x), T, H, _ptr(router_w), _ptr(router_bias), E, topk, e_begin, e_end, descs,
                                     I, _ptr(y), None, None, None, None, None, _ptr(workspace), workspace.numel(),
                                     _ptr(dev_status), _stream(stream)), "moe_q4_forward_range")
    return y


def expert_range(rank: int, world: int, E: int) -> tuple:
    """The experts rank `rank` of `world` owns under expert parallelism: a contiguous, near-equal split."""
    return (rank * E) // world, ((rank + 1) * E) // world


def moe_q4_forward_expert_parallel(x: torch.Tensor, router_w: torch.Tensor, router_bias: torch.Tensor | None,
                                   topk: int, local_experts: tuple, I: int, group=None, range_fn=None,
                                   **kw) -> torch.Tensor:
    """Expert-parallel MoE layer: this rank holds the weights of expert_range(rank, world, E) only; every
    rank routes the same tokens, computes its experts' contribution and the contributions are summed by an
    all-reduce (fp32) over `group` (torch.distributed; NCCL on GPUs).  range_fn replaces
    moe_q4_forward_range (tests on CPU ranks)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    e0, e1 = expert_range(rank, world, router_w.shape[0])
    y = (range_fn or moe_q4_forward_range)(x, router_w, router_bias, topk, e0, e1, local_experts, I, **kw)
    dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    return y


def moe_q4_forward_noalloc(x: torch.Tensor, router_w: torch.Tensor, router_bias: torch.Tensor | None, topk: int,
                           experts: tuple, I: int, out_dtype=torch.float32, y: torch.Tensor | None = None,
                           dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """moe_q4_forward using the library's fixed device scratch instead of a caller workspace, for callers
    that cannot allocate device memory (see include/q4.h).  Sizes needing more than
    Q4_MOE_NOALLOC_SCRATCH_BYTES of scratch raise Q4Error(Q4_ERR_WORKSPACE).  Calls share the scratch:
    keep them ordered on one stream."""
    _dev(x, torch.bfloat16, "x")
    _dev(router_w, torch.float32, "router_w")
    T, H = x.shape
    E = _router(router_w, router_bias, H, x.device)
    _weights_on(x.device, *experts)
    if y is None:
        y = torch.empty((T, H), dtype=out_dtype, device=x.device)
    od = _out(y, (T, H), x.device)
    descs = (q4_weight * 3)(*[e.desc for e in experts])
    _hold(stream, y)
    _check(_lib.moe_q4_forward_noalloc(_ptr(x), T, H, _ptr(router_w), _ptr(router_bias), E, topk, descs, I, _ptr(y),
                                       od, None, None, None, None, None, _ptr(dev_status), _stream(stream)),
           "moe_q4_forward_noalloc")
    return y


# ---------------------------------------------------------------------------------------------- #
# the layer's steps as separate calls, and expert parallelism in its all-to-all form
# ---------------------------------------------------------------------------------------------- #

def moe_q4_route(x: torch.Tensor, router_w: torch.Tensor, router_bias: torch.Tensor | None, topk: int,
                 dev_status: torch.Tensor | None = None, stream=None) -> dict:
    """Routing and the permutation of the MoE layer (moe_q4_route): returns a dict of device tensors
    topk_ids [T][topk] i32, topk_w [T][topk] f32, offsets [E+1] i32, pair_pos [T*topk] i32 (the permuted
    position of each (token, slot) pair), x_perm [T*topk][H] bf16 (the rows in expert order: the dispatch
    buffer), row_expert [T*topk] i32 (the expert of each permuted row)."""
    _dev(x, torch.bfloat16, "x")
    _dev(router_w, torch.float32, "router_w")
    T, H = x.shape
    dev = x.device
    E = _router(router_w, router_bias, H, dev)
    P = T * topk
    out = {"topk_ids": torch.empty((T, topk), dtype=torch.int32, device=dev),
           "topk_w": torch.empty((T, topk), dtype=torch.float32, device=dev),
           "offsets": torch.empty((E + 1,), dtype=torch.int32, device=dev),
           "pair_pos": torch.empty((P,), dtype=torch.int32, device=dev),
           "x_perm": torch.empty((P, H), dtype=torch.bfloat16, device=dev),
           "row_expert": torch.empty((P,), dtype=torch.int32, device=dev)}
    ws = torch.empty((max(int(_lib.moe_q4_route_workspace_size(T, E, topk)), 1),), dtype=torch.uint8, device=dev)
    _hold(stream, ws, *out.values())
    _check(_lib.moe_q4_route(_ptr(x), T, H, _ptr(router_w), _ptr(router_bias), E, topk, _ptr(out["topk_ids"]),
                             _ptr(out["topk_w"]), _ptr(out["offsets"]), _ptr(out["pair_pos"]), _ptr(out["x_perm"]),
                             _ptr(out["row_expert"]), None, None, _ptr(ws), ws.numel(), _ptr(dev_status),
                             _stream(stream)), "moe_q4_route")
    return out


def moe_q4_forward_rows(x_rows: torch.Tensor, row_expert: torch.Tensor, e_base: int, experts: tuple, I: int,
                        row_weight: torch.Tensor | None = None, y: torch.Tensor | None = None,
                        workspace: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """The expert FFN on rows routed elsewhere (moe_q4_forward_rows): y[r] = row_weight[r] *
    FFN_{row_expert[r] - e_base}(x_rows[r]), fp32 [R][H]; experts = (gate, up, down) stacked over the E
    local experts (E = gate.n / I)."""
    _dev(x_rows, torch.bfloat16, "x_rows")
    _dev(row_expert, torch.int32, "row_expert")
    R, H = x_rows.shape
    _weights_on(x_rows.device, *experts)
    E = experts[0].n // I
    _numel(row_expert, R, "row_expert")
    if row_weight is not None:
        _numel(_dev(row_weight, torch.float32, "row_weight"), R, "row_weight")
    if y is None:
        y = torch.empty((R, H), dtype=torch.float32, device=x_rows.device)
    _dev(y, torch.float32, "y")
    _out(y, (R, H), x_rows.device)
    if workspace is None:
        workspace = torch.empty((max(int(_lib.moe_q4_rows_workspace_size(R, H, I, E)), 1),), dtype=torch.uint8,
                                device=x_rows.device)
    _workspace(workspace, x_rows.device)
    descs = (q4_weight * 3)(*[e.desc for e in experts])
    _hold(stream, y, workspace)
    _check(_lib.moe_q4_forward_rows(_ptr(x_rows), R, H, _ptr(row_expert), int(e_base), _ptr(row_weight), E, descs, I,
                                    _ptr(y), _ptr(workspace), workspace.numel(), _ptr(dev_status), _stream(stream)),
           "moe_q4_forward_rows")
    return y


def moe_q4_combine(o_rows: torch.Tensor, pair_pos: torch.Tensor, topk_w: torch.Tensor, out_dtype=torch.float32,
                   y: torch.Tensor | None = None, dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y[t] = sum_j topk_w[t][j] * o_rows[pair_pos[t*topk + j]] (moe_q4_combine), slot order j."""
    _dev(o_rows, torch.float32, "o_rows")
    _dev(pair_pos, torch.int32, "pair_pos")
    _dev(topk_w, torch.float32, "topk_w")
    P, H = o_rows.shape
    T, topk = topk_w.shape
    _numel(pair_pos, T * topk, "pair_pos")
    if y is None:
        y = torch.empty((T, H), dtype=out_dtype, device=o_rows.device)
    od = _out(y, (T, H), o_rows.device)
    _hold(stream, y)
    _check(_lib.moe_q4_combine(_ptr(o_rows), P, H, _ptr(pair_pos), _ptr(topk_w), T, topk, _ptr(y), od,
                               _ptr(dev_status), _stream(stream)), "moe_q4_combine")
    return y


def moe_q4_forward_ep(x: torch.Tensor, router_w: torch.Tensor, router_bias: torch.Tensor | None, topk: int,
                      local_experts: tuple, I: int, group=None, out_dtype=torch.float32, fns: dict | None = None,
                      dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """Expert-parallel MoE layer, all-to-all form.  Every rank holds its own tokens x [T_r][H] and the weights
    of its experts expert_range(rank, world, E) only.  Per rank: route its tokens (the permutation puts the
    rows in expert order, so the rows for rank d are one contiguous block); exchange the block sizes; send
    each block to the rank that owns its experts and receive the rows routed to this rank's experts (one
    all-to-all of bf16 rows and one of their expert ids); run the local experts on the received rows; send
    the fp32 results back (the reverse all-to-all) and combine them with the routing weights in token
    order.  Each routed row crosses the interconnect once each way.  fns replaces the three device steps
    (route, rows, combine) with host implementations for tests on CPU ranks."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    E = router_w.shape[0]
    T, H = x.shape
    fns = fns or {}
    route = fns.get("route", lambda: moe_q4_route(x, router_w, router_bias, topk, dev_status=dev_status))
    r = route()
    bounds = [expert_range(d, world, E) for d in range(world)]
    off = r["offsets"].to("cpu")
    send = [int(off[e1] - off[e0]) for (e0, e1) in bounds]
    cdev = r["offsets"].device if dist.get_backend(group) == "nccl" else torch.device("cpu")
    send_t = torch.tensor(send, dtype=torch.int64, device=cdev)
    recv_t = torch.empty_like(send_t)
    dist.all_to_all_single(recv_t, send_t, group=group)
    recv = [int(v) for v in recv_t.to("cpu")]
    # rows travel as bytes (2 H per row), which every backend moves as they are
    rows_in = torch.empty((sum(recv), 2 * H), dtype=torch.uint8, device=r["x_perm"].device)
    dist.all_to_all_single(rows_in, r["x_perm"].contiguous().view(torch.uint8), recv, send, group=group)
    exp_in = torch.empty((sum(recv),), dtype=torch.int32, device=r["row_expert"].device)
    dist.all_to_all_single(exp_in, r["row_expert"], recv, send, group=group)
    e0, e1 = bounds[rank]
    rows_fn = fns.get("rows", lambda xr, er, eb: moe_q4_forward_rows(xr, er, eb, local_experts, I, dev_status=dev_status))
    o_in = rows_fn(rows_in.view(torch.bfloat16), exp_in, e0)
    o_back = torch.empty((T * topk, H), dtype=torch.float32, device=o_in.device)
    dist.all_to_all_single(o_back, o_in, send, recv, group=group)
    combine = fns.get("combine", lambda o, pp, w: moe_q4_combine(o, pp, w, out_dtype=out_dtype, dev_status=dev_status))
    return combine(o_back, r["pair_pos"], r["topk_w"])
