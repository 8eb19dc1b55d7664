"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle's callers.

This module holds none of the method's arithmetic: it only draws random numbers (the generator
itself is ``synth_gen.c``, compiled into ``libsynth.so``).

Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014) used counter-style: value i of a stream with 64-bit key ``key`` is
``mix(key + (i + 1) * 0x9E3779B97F4A7C15)`` where ``mix`` is SplitMix64's output function.  A stream
key is derived from a tuple of labels (seed, workload, layer, tensor name ...) by chaining ``mix``.
Uniforms take the top 53 bits; normals use Box-Muller on two uniforms (fp64), rounded to fp32;
bf16 inputs are the fp32 values rounded to nearest-even.

Distributions follow the workloads:
  * weights ~ N(0, 0.02^2), each entry multiplied by 20 with probability 0.001 (outliers);
  * activations ~ N(0, 1); optionally with round(0.01*K) seeded channels scaled x10 (shared by all
    rows), or i.i.d. Student-t with 3 degrees of freedom (Z / sqrt(chi2_3 / 3));
  * router weights ~ N(0, 1/H) in fp32; router bias b_e = -1.1 * ln(e + 1) (Zipf-like skew over the
    experts, expert 0 hottest).
"""
from __future__ import annotations

import ctypes
import hashlib
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth_gen.c")
_SO = os.path.join(_HERE, "libsynth.so")
_MASK = 0xFFFFFFFFFFFFFFFF
GAMMA = 0x9E3779B97F4A7C15


def build(force: bool = False) -> str:
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


_lib = None


def _g():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        u64, i64, dbl, p = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        _lib.syn_u64.argtypes = [u64, i64, i64, p]
        _lib.syn_uniform.argtypes = [u64, i64, p]
        _lib.syn_normal.argtypes = [u64, i64, p]
        _lib.syn_weights.argtypes = [u64, u64, i64, dbl, dbl, ctypes.c_float, p]
        _lib.syn_normal_f32.argtypes = [u64, i64, dbl, p]
        _lib.syn_student_t3_f32.argtypes = [u64, u64, u64, u64, i64, p]
    return _lib


def mix64(z: int) -> int:
    """SplitMix64's output function on a Python int (used to chain stream labels)."""
    z &= _MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK
    return z ^ (z >> 31)


def stream_key(*labels) -> int:
    """64-bit key of a stream named by a tuple of labels (ints or strings)."""
    k = 0x5EED5EED5EED5EED
    for lab in labels:
        if isinstance(lab, str):
            v = int.from_bytes(hashlib.sha256(lab.encode()).digest()[:8], "little")
        else:
            v = int(lab) & _MASK
        k = mix64(k + v * GAMMA + GAMMA)
    return k


def raw_u64(key: int, n: int, start: int = 0) -> np.ndarray:
    out = np.empty(n, np.uint64)
    _g().syn_u64(key, start, n, out.ctypes.data)
    return out


def uniform(key: int, n: int) -> np.ndarray:
    out = np.empty(n, np.float64)
    _g().syn_uniform(key, n, out.ctypes.data)
    return out


def normal(key: int, n: int) -> np.ndarray:
    out = np.empty(n, np.float64)
    _g().syn_normal(key, n, out.ctypes.data)
    return out


def to_bf16_bits(a_f32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even (torch's conversion)."""
    t = torch.from_numpy(np.ascontiguousarray(a_f32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def weights(key_labels: tuple, n: int, k: int, std: float = 0.02, outlier_p: float = 0.001,
            outlier_mul: float = 20.0) -> np.ndarray:
    """fp32 [n][k] ~ N(0, std^2) with a fraction outlier_p of entries multiplied by outlier_mul."""
    out = np.empty((n, k), np.float32)
    _g().syn_weights(stream_key(*key_labels, "normal"), stream_key(*key_labels, "outlier"), n * k,
                     std, outlier_p, outlier_mul, out.ctypes.data)
    return out


def activations(key_labels: tuple, m: int, k: int, kind: str = "normal") -> np.ndarray:
    """bf16 bit patterns [m][k].  kind: 'normal', 'outlier_channels' (1% channels x10), 'student_t3'."""
    a = np.empty((m, k), np.float32)
    if kind in ("normal", "outlier_channels"):
        _g().syn_normal_f32(stream_key(*key_labels, "normal"), m * k, 1.0, a.ctypes.data)
        if kind == "outlier_channels":
            nch = int(round(0.01 * k))
            order = np.argsort(uniform(stream_key(*key_labels, "channels"), k), kind="stable")
            a[:, order[:nch]] *= np.float32(10.0)
    elif kind == "student_t3":
        _g().syn_student_t3_f32(stream_key(*key_labels, "z"), stream_key(*key_labels, "chi0"),
                                stream_key(*key_labels, "chi1"), stream_key(*key_labels, "chi2"), m * k,
                                a.ctypes.data)
    else:
        raise ValueError(kind)
    return to_bf16_bits(a)


def router(key_labels: tuple, E: int, H: int, skew: float = 1.1):
    """(Wr fp32 [E][H] ~ N(0, 1/H), bias fp32 [E] = -skew * ln(e + 1))."""
    Wr = np.empty((E, H), np.float32)
    _g().syn_normal_f32(stream_key(*key_labels, "router"), E * H, 1.0 / np.sqrt(H), Wr.ctypes.data)
    bias = (-skew * np.log(np.arange(1, E + 1, dtype=np.float64))).astype(np.float32)
    return Wr, bias


# The LLaMA-3.2-1B-shaped linear layers: (name, N, K) per decoder layer.
LLAMA_1B_LINEARS = (
    ("q", 2048, 2048),
    ("k", 512, 2048),
    ("v", 512, 2048),
    ("o", 2048, 2048),
    ("gate", 8192, 2048),
    ("up", 8192, 2048),
    ("down", 2048, 8192),
)
LLAMA_1B_LAYERS = 16
