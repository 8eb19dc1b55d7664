"""The oracle: a plain, slow, obviously correct CPU implementation of the INT4 linear layers and the
INT4 MoE expert FFN (see q4_oracle.c for the arithmetic and the passages each function follows).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product path (the CUDA
library under ``moe_linear_layers_b200``) never imports it, and the two share no code.

This module marshals numpy arrays into the C functions.  Apart from the composition helpers below
(``silu_mul``, ``linear_w4a16_swiglu``, ``moe_experts_classes``), which combine the pinned C functions
with plain fp64 numpy arithmetic, the arithmetic is in q4_oracle.c.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "q4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# Every float operation in the source is one IEEE operation: no fast-math, no contraction.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
          "-fno-unsafe-math-optimizations", "-frounding-math"]


def build(force: bool = False) -> str:
    """Compile q4_oracle.c into liboracle.so next to it (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        # Q4_ORACLE_LIB substitutes a library built from a modified copy of q4_oracle.c: the test that
        # plants mistakes in the oracle checks that the pins reject each one
        _lib = ctypes.CDLL(os.environ.get("Q4_ORACLE_LIB") or build())
        _lib.orc_f32_to_f16.restype = ctypes.c_uint16
        _lib.orc_f32_to_f16.argtypes = [ctypes.c_float]
        _lib.orc_f16_to_f32.restype = ctypes.c_float
        _lib.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
        _lib.orc_router_logit.restype = ctypes.c_float
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    pass


def f32_to_f16_bits(v: float) -> int:
    return int(lib().orc_f32_to_f16(ctypes.c_float(v)))


def f16_bits_to_f32(b: int) -> float:
    return float(lib().orc_f16_to_f32(ctypes.c_uint16(b)))


def quantize(w: np.ndarray, group: int, symmetric: bool):
    """RTN group quantization + packing.  w: fp32 [n][k].
    Returns (packed u8 [n][k/2], scales u16 fp16-bits [n][k/g], zeros u16 fp16-bits [n][k/g] or None)."""
    w = _c(w, np.float32)
    n, k = w.shape
    packed = np.empty((n, k // 2), np.uint8)
    scales = np.empty((n, k // group), np.uint16)
    zeros = None if symmetric else np.empty((n, k // group), np.uint16)
    rc = lib().orc_quantize(_p(w), n, k, group, int(bool(symmetric)), _p(packed), _p(scales), _p(zeros))
    if rc != 0:
        raise OracleError(f"orc_quantize returned {rc}")
    return packed, scales, zeros


def unpack_codes(packed: np.ndarray, k: int, symmetric: bool) -> np.ndarray:
    packed = _c(packed, np.uint8)
    n = packed.shape[0]
    codes = np.empty((n, k), np.int8)
    lib().orc_unpack_codes(_p(packed), n, k, int(bool(symmetric)), _p(codes))
    return codes


def dequant(packed, scales, zeros, k: int, group: int, symmetric: bool) -> np.ndarray:
    packed = _c(packed, np.uint8)
    n = packed.shape[0]
    out = np.empty((n, k), np.float32)
    lib().orc_dequant(_p(packed), _p(_c(scales, np.uint16)), _p(_c(zeros, np.uint16)),
                      n, k, group, int(bool(symmetric)), _p(out))
    return out


def linear_w4a16(x_bf16_bits, packed, scales, zeros, n: int, k: int, group: int, symmetric: bool,
                 rows_m=None, rows_n=None) -> np.ndarray:
    """fp64 y[m][n] = sum_k x * dequant(W); x given as bf16 bit patterns (uint16) [M][k]."""
    x = _c(x_bf16_bits, np.uint16).reshape(-1, k)
    rm = _c(rows_m, np.int32)
    rn = _c(rows_n, np.int32)
    cm = x.shape[0] if rm is None else len(rm)
    cn = n if rn is None else len(rn)
    y = np.empty((cm, cn), np.float64)
    lib().orc_linear_w4a16(_p(x), x.shape[0], k, _p(_c(packed, np.uint8)), _p(_c(scales, np.uint16)),
                           _p(_c(zeros, np.uint16)), n, group, int(bool(symmetric)),
                           _p(rm), 0 if rm is None else len(rm), _p(rn), 0 if rn is None else len(rn), _p(y))
    return y


def silu_mul(gate_f32, up_f32):
    """h = silu(g) * u = g / (1 + e^-g) * u in fp64 from fp32 inputs (the SwiGLU gating of the dense FFN
    and of every expert: "高效大语言模型推理实践：INT4量化与MoE架构的融合探索" MoE架构设计)."""
    g = np.asarray(gate_f32, np.float32).astype(np.float64)
    u = np.asarray(up_f32, np.float32).astype(np.float64)
    return g / (1.0 + np.exp(-g)) * u


def linear_w4a16_swiglu(gate_f32, up_f32, packed, scales, zeros, n: int, k: int, group: int,
                        symmetric: bool) -> np.ndarray:
    """fp64 y[m][n] = sum_k silu(g) * u * dequant(W): the dense FFN's down projection on its gated input."""
    h = silu_mul(gate_f32, up_f32).reshape(-1, k)
    w = dequant(packed, scales, zeros, k, group, symmetric).astype(np.float64)
    return h @ w.T


def act_quant(x_bf16_bits, k: int):
    x = _c(x_bf16_bits, np.uint16).reshape(-1, k)
    m = x.shape[0]
    q = np.empty((m, k), np.int8)
    s = np.empty((m,), np.float32)
    rc = lib().orc_act_quant(_p(x), m, k, _p(q), _p(s))
    if rc != 0:
        raise OracleError(f"orc_act_quant returned {rc}")
    return q, s


def act_quant_f16(x_f16_bits, k: int):
    """Per-token INT8 quantization of fp16 rows (given as fp16 bit patterns, uint16 [M][k])."""
    x = _c(x_f16_bits, np.uint16).reshape(-1, k)
    m = x.shape[0]
    q = np.empty((m, k), np.int8)
    s = np.empty((m,), np.float32)
    rc = lib().orc_act_quant_f16(_p(x), m, k, _p(q), _p(s))
    if rc != 0:
        raise OracleError(f"orc_act_quant_f16 returned {rc}")
    return q, s


def linear_w4a8(xq, s_a, packed, scales, n: int, k: int, group: int, rows_m=None, rows_n=None,
                want_acc: bool = False, zeros=None, symmetric: bool = True):
    xq = _c(xq, np.int8).reshape(-1, k)
    s_a = _c(s_a, np.float32)
    rm = _c(rows_m, np.int32)
    rn = _c(rows_n, np.int32)
    cm = xq.shape[0] if rm is None else len(rm)
    cn = n if rn is None else len(rn)
    y = np.empty((cm, cn), np.float64)
    acc = np.empty((cm, cn, k // group), np.int32) if want_acc else None
    if not symmetric and zeros is None:
        raise OracleError("asymmetric W4A8 needs the zero points")
    lib().orc_linear_w4a8(_p(xq), _p(s_a), xq.shape[0], k, _p(_c(packed, np.uint8)), _p(_c(scales, np.uint16)),
                          _p(None if symmetric else _c(zeros, np.uint16)), int(bool(symmetric)), n, group, _p(rm), 0 if rm is None else len(rm), _p(rn), 0 if rn is None else len(rn),
                          _p(acc), _p(y))
    return (y, acc) if want_acc else y


def router_logit(x_row_bf16_bits, w_row_f32) -> float:
    x = _c(x_row_bf16_bits, np.uint16)
    w = _c(w_row_f32, np.float32)
    return float(lib().orc_router_logit(_p(x), _p(w), len(x)))


def route(x_bf16_bits, H: int, Wr, bias, topk: int):
    """Returns (logits f32 [T][E], ids i32 [T][topk], weights f64 [T][topk], counts i32 [E])."""
    x = _c(x_bf16_bits, np.uint16).reshape(-1, H)
    Wr = _c(Wr, np.float32)
    E = Wr.shape[0]
    T = x.shape[0]
    logits = np.empty((T, E), np.float32)
    ids = np.empty((T, topk), np.int32)
    w = np.empty((T, topk), np.float64)
    counts = np.empty((E,), np.int32)
    rc = lib().orc_route(_p(x), T, H, _p(Wr), _p(_c(bias, np.float32)), E, topk, _p(logits), _p(ids), _p(w),
                         _p(counts))
    if rc != 0:
        raise OracleError(f"orc_route returned {rc}")
    return logits, ids, w, counts


def permute(ids, E: int):
    ids = _c(ids, np.int32)
    T, topk = ids.shape
    offsets = np.empty((E + 1,), np.int32)
    perm = np.empty((T * topk,), np.int32)
    lib().orc_permute(_p(ids), T, topk, E, _p(offsets), _p(perm))
    return offsets, perm


def shared_expert(x_bf16_bits, H: int, gate, up, down, I_s: int, group: int, symmetric: bool, tokens=None):
    """A shared expert every token passes through (the MoE architecture sections of the W4A8 and
    INT4+MoE pages): one SwiGLU FFN with routing weight 1, i.e. the routed-expert computation with a
    single expert chosen by every token.  Returns fp64 [n_tok][H]."""
    T = np.asarray(x_bf16_bits).reshape(-1, H).shape[0]
    ids = np.zeros((T, 1), np.int32)
    w = np.ones((T, 1), np.float64)
    return moe_experts(x_bf16_bits, H, ids, w, gate, up, down, I_s, group, symmetric, tokens=tokens)


def moe_experts(x_bf16_bits, H: int, ids, w, gate, up, down, I: int, group: int, symmetric: bool,
                tokens=None):
    """gate/up/down: (packed, scales, zeros) of the stacked expert matrices.  Returns fp64 [n_tok][H]."""
    x = _c(x_bf16_bits, np.uint16).reshape(-1, H)
    ids = _c(ids, np.int32)
    w = _c(w, np.float64)
    T, topk = ids.shape
    tk = _c(tokens, np.int32)
    cnt = T if tk is None else len(tk)
    y = np.empty((cnt, H), np.float64)
    args = []
    for (pk, sc, zr) in (gate, up, down):
        args += [_p(_c(pk, np.uint8)), _p(_c(sc, np.uint16)), _p(_c(zr, np.uint16))]
    lib().orc_moe_experts(_p(x), T, H, _p(ids), _p(w), topk, *args, I, group, int(bool(symmetric)),
                          _p(tk), 0 if tk is None else len(tk), _p(y))
    return y


def moe_experts_a8(x_bf16_bits, H: int, ids, w, gate, up, down, I: int, group: int, symmetric: bool,
                   a8_mask: int, tokens=None):
    """The expert FFN with INT8 activations: a8_mask bit 0 = gate/up W4A8 on the token's INT8 codes,
    bit 1 = down W4A8 on the INT8 codes of h (quantized per row as an fp16 activation).  Returns fp64 [n_tok][H]."""
    x = _c(x_bf16_bits, np.uint16).reshape(-1, H)
    ids = _c(ids, np.int32)
    w = _c(w, np.float64)
    T, topk = ids.shape
    tk = _c(tokens, np.int32)
    cnt = T if tk is None else len(tk)
    y = np.empty((cnt, H), np.float64)
    args = []
    for (pk, sc, zr) in (gate, up, down):
        args += [_p(_c(pk, np.uint8)), _p(_c(sc, np.uint16)), _p(_c(zr, np.uint16))]
    rc = lib().orc_moe_experts_a8(_p(x), T, H, _p(ids), _p(w), topk, *args, I, group, int(bool(symmetric)),
                                  int(a8_mask), _p(tk), 0 if tk is None else len(tk), _p(y))
    if rc != 0:
        raise OracleError(f"orc_moe_experts_a8 returned {rc}")
    return y


def moe_experts_classes(x_bf16_bits, H: int, ids, w, class_begin, classes, I: int, tokens=None):
    """The expert FFN with per-class quantization (the W4A8 page §5.3: group size chosen by how often an
    expert is used).  class c = experts class_begin[c] .. class_begin[c+1]-1; classes[c] = (gate, up, down,
    group, symmetric) with gate/up/down = (packed, scales, zeros) stacked over the class's experts.  Each
    class is evaluated by moe_experts on the slots routed to it (the other slots get weight 0, so they add
    exact zeros) and the classes' outputs are summed.  Returns fp64 [n_tok][H]."""
    ids = np.asarray(ids, np.int32)
    w = np.asarray(w, np.float64)
    y = None
    for c, (gate, up, down, group, symmetric) in enumerate(classes):
        e0, e1 = int(class_begin[c]), int(class_begin[c + 1])
        mine = (ids >= e0) & (ids < e1)
        ids_c = np.where(mine, ids - e0, 0).astype(np.int32)
        w_c = np.where(mine, w, 0.0)
        yc = moe_experts(x_bf16_bits, H, ids_c, w_c, gate, up, down, I, group, symmetric, tokens=tokens)
        y = yc if y is None else y + yc
    return y
