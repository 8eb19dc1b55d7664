"""Helpers shared by the GPU parity tests (tolerance checks, host<->device marshalling)."""
import numpy as np
import torch

# Floating outputs must satisfy max|y - y_ref| <= REL_TOL * rms(y_ref), y_ref the fp64 oracle over the
# dequantized weights (the bar the workloads state).
REL_TOL = 1e-2


def rel_err(y, ref) -> float:
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(y - ref))) / (rms if rms > 0 else 1.0)


def assert_close(y, ref, tol=REL_TOL, what=""):
    e = rel_err(y, ref)
    assert e <= tol, f"{what}: max|err|/rms = {e:.3e} > {tol}"
    return e


def cuda_u16_as(a_u16: np.ndarray, dtype) -> torch.Tensor:
    """Upload uint16 bit patterns as a CUDA tensor of a 16-bit float dtype."""
    t = torch.from_numpy(np.ascontiguousarray(a_u16).view(np.int16)).cuda()
    return t.view(dtype)


def cpu_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_rne(a_f32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits with round to nearest even (torch's conversion)."""
    return torch.from_numpy(np.ascontiguousarray(a_f32, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def upload_weight(q4, packed, scales, zeros, n, k, group, sym):
    pk = torch.from_numpy(np.ascontiguousarray(packed)).cuda()
    sc = cuda_u16_as(scales, torch.float16)
    zr = None if zeros is None else cuda_u16_as(zeros, torch.float16)
    return q4.Q4Weight(pk, sc, zr, n, k, group, sym)
