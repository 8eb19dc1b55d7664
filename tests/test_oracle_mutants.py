"""The pins reject a wrong oracle: each case below plants one plausible mistake in a copy of
oracle/q4_oracle.c (a dropped term, a wrong sign, divisor, index, rounding or reduction order, a
transposed operand), builds it with the oracle's own flags, and runs the pin file against it through
Q4_ORACLE_LIB.  Every mutant must make at least one pin fail; the unmodified source must pass them all.

The mistakes are planted in the oracle, on the CPU; nothing here touches the CUDA library."""
import concurrent.futures as cf
import os
import re
import subprocess
import sys

import numpy as np

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# (name, the function it is planted in, text replaced, replacement)
MUTANTS = [
    # fp16 and bf16 conversion
    ("f16 rounding: ties away from zero", "uint16_t orc_f32_to_f16(float f)",
     "if (rest > 0x1000u || (rest == 0x1000u && (keep & 1u))) keep++;", "if (rest >= 0x1000u) keep++;"),
    ("f16 rounding: subnormal ties away from zero", "uint16_t orc_f32_to_f16(float f)",
     "if (rest > half || (rest == half && (keep & 1u))) keep++;", "if (rest >= half) keep++;"),
    ("f16 rounding: truncation", "uint16_t orc_f32_to_f16(float f)",
     "if (rest > 0x1000u || (rest == 0x1000u && (keep & 1u))) keep++;", ""),
    ("f16 widening: exponent bias off by one", "float orc_f16_to_f32(uint16_t h)",
     "(exp + 112u) << 23", "(exp + 111u) << 23"),
    ("f16 widening: subnormal scale 2^-25", "float orc_f16_to_f32(uint16_t h)",
     "(float)man * 0x1p-24f", "(float)man * 0x1p-25f"),
    # quantizer
    ("symmetric scale amax/8", "int orc_quantize(", "float s32 = amax / 7.0f;", "float s32 = amax / 8.0f;"),
    ("asymmetric scale range/16", "int orc_quantize(", "(mx - mn) / 15.0f", "(mx - mn) / 16.0f"),
    ("asymmetric range not widened to 0", "int orc_quantize(",
     "float mn = 0.0f, mx = 0.0f;", "float mn = src[0], mx = src[0];"),
    ("zero point sign", "int orc_quantize(", "rne(-mn / S)", "rne(mn / S)"),
    ("zero point added before rounding", "int orc_quantize(",
     "rne(src[i] / S) + (float)z", "rne(src[i] / S + (float)z)"),
    ("codes from the fp32 scale, not the stored fp16 one", "int orc_quantize(",
     "(int)clampf(rne(src[i] / S), -8.0f, 7.0f)", "(int)clampf(rne(src[i] / s32), -8.0f, 7.0f)"),
    ("asymmetric codes clamped to 0..14", "int orc_quantize(",
     "rne(src[i] / S) + (float)z, 0.0f, 15.0f)", "rne(src[i] / S) + (float)z, 0.0f, 14.0f)"),
    ("nibbles packed high first", "int orc_quantize(",
     "(uint8_t)((codes[i] & 0xF) | ((codes[i + 1] & 0xF) << 4))",
     "(uint8_t)((codes[i + 1] & 0xF) | ((codes[i] & 0xF) << 4))"),
    # unpacking and dequantization
    ("nibbles unpacked high first", "static int code_at(",
     "(kk & 1) ? (b >> 4) : (b & 0xF)", "(kk & 1) ? (b & 0xF) : (b >> 4)"),
    ("two's complement threshold 9", "static int code_at(", "if (symmetric && v >= 8) v -= 16;",
     "if (symmetric && v > 8) v -= 16;"),
    ("dequantization adds the zero point", "static float deq_at(",
     "((float)code_at(packed, k, r, kk, symmetric) - z) * S", "((float)code_at(packed, k, r, kk, symmetric) + z) * S"),
    ("dequantization takes the next group's scale", "static float deq_at(",
     "int g = kk / group, ng = k / group;", "int ng = k / group, g = (kk / group + 1) % ng;"),
    # W4A16 linear
    ("linear: x read in reverse", "void orc_linear_w4a16(",
     "acc += (double)orc_bf16_to_f32(xr[kk]) * wrow[kk];", "acc += (double)orc_bf16_to_f32(xr[k - 1 - kk]) * wrow[kk];"),
    ("linear: last term dropped", "void orc_linear_w4a16(",
     "for (int kk = 0; kk < k; kk++) acc +=", "for (int kk = 0; kk < k - 1; kk++) acc +="),
    ("linear: x widened as fp16", "void orc_linear_w4a16(",
     "acc += (double)orc_bf16_to_f32(xr[kk])", "acc += (double)orc_f16_to_f32(xr[kk])"),
    # per-token INT8 activations
    ("activation scale amax/128", "static float act_quant_row(", "float sc = amax / 127.0f;",
     "float sc = amax / 128.0f;"),
    ("activation rounding ties away from zero", "static float act_quant_row(",
     "rne(v[kk] / sc)", "roundf(v[kk] / sc)"),
    ("activation codes by the reciprocal", "static float act_quant_row(",
     "rne(v[kk] / sc)", "rne(v[kk] * (1.0f / sc))"),
    ("fp16 activations widened as bf16", "int orc_act_quant_f16(",
     "v[kk] = orc_f16_to_f32(x[", "v[kk] = orc_bf16_to_f32(x["),
    # W4A8 linear
    ("W4A8: zero point added", "void orc_linear_w4a8(",
     "((int32_t)code_at(packed, k, r, kk, symmetric) - z)", "((int32_t)code_at(packed, k, r, kk, symmetric) + z)"),
    ("W4A8: activation scale dropped", "void orc_linear_w4a8(", " * (double)s_a[mi];", ";"),
    ("W4A8: first group's weight scale for every group", "void orc_linear_w4a8(",
     "(double)orc_f16_to_f32(scales[(size_t)r * ng + g])", "(double)orc_f16_to_f32(scales[(size_t)r * ng])"),
    # router
    ("router: butterfly in the opposite order", "float orc_router_logit(",
     "for (int s = 16; s >= 1; s >>= 1)", "for (int s = 1; s <= 16; s <<= 1)"),
    ("router: multiply then add, not fused", "float orc_router_logit(",
     "p[l] = fmaf(orc_bf16_to_f32(xrow[kk]), wrow[kk], p[l]);", "p[l] = p[l] + orc_bf16_to_f32(xrow[kk]) * wrow[kk];"),
    ("router: lanes over contiguous blocks", "float orc_router_logit(",
     "for (int kk = l; kk < H; kk += 32)", "for (int kk = l * (H / 32); kk < (l + 1) * (H / 32); kk++)"),
    ("router: bias ignored", "int orc_route(", "if (bias) v = v + bias[e];", "if (bias) v = v + 0.0f * bias[e];"),
    ("router: ties keep the higher id", "int orc_route(", "l[e] > l[best]", "l[e] >= l[best]"),
    ("router: weights not normalised", "int orc_route(",
     "exp((double)l[ids[(size_t)t * topk + j]] - l0) / den;", "exp((double)l[ids[(size_t)t * topk + j]] - l0);"),
    ("router: weights from the softmax of the first logit only", "int orc_route(",
     "for (int j = 0; j < topk; j++) den += exp(", "for (int j = 0; j < 1; j++) den += exp("),
    # permutation
    ("permutation not stable (tokens descending)", "void orc_permute(",
     "for (int t = 0; t < T; t++)", "for (int t = T - 1; t >= 0; t--)"),
    # MoE expert FFN
    ("SiLU with the wrong sign", "void orc_moe_experts(",
     "h[i] = gv / (1.0 + exp(-gv)) * uv;", "h[i] = gv / (1.0 + exp(gv)) * uv;"),
    ("gate and up exchanged", "void orc_moe_experts(",
     "h[i] = gv / (1.0 + exp(-gv)) * uv;", "h[i] = uv / (1.0 + exp(-uv)) * gv;"),
    ("sigmoid instead of SiLU", "void orc_moe_experts(",
     "h[i] = gv / (1.0 + exp(-gv)) * uv;", "h[i] = 1.0 / (1.0 + exp(-gv)) * uv;"),
    ("h rounded to fp16 between the projections", "void orc_moe_experts(",
     "h[i] = gv / (1.0 + exp(-gv)) * uv;",
     "h[i] = orc_f16_to_f32(orc_f32_to_f16((float)(gv / (1.0 + exp(-gv)) * uv)));"),
    ("combine weight dropped", "void orc_moe_experts(", "yr[c] += wj * o;", "yr[c] += o;"),
    ("every token takes expert 0's down codes", "void orc_moe_experts(",
     "const uint8_t* dp = d_packed + (size_t)e * H * (I / 2);", "const uint8_t* dp = d_packed;"),
    ("up matrix read from the gate block", "void orc_moe_experts(",
     "const uint8_t* up = u_packed + (size_t)e * I * (H / 2);", "const uint8_t* up = g_packed + (size_t)e * I * (H / 2);"),
    # MoE with INT8 activations
    ("a8: h quantized from fp32, not its fp16 value", "int orc_moe_experts_a8(",
     "hf[i] = orc_f16_to_f32(orc_f32_to_f16((float)h[i]));", "hf[i] = (float)h[i];"),
    ("a8: gate/up follow the down projection's mask bit", "int orc_moe_experts_a8(",
     "if (a8_mask & 1) {", "if (a8_mask & 2) {"),
    ("a8: combine weight dropped", "int orc_moe_experts_a8(", "yr[c] += wj * o;", "yr[c] += o;"),
    ("a8: zero point added in the INT8 dot", "static double w4a8_dot(",
     "((int32_t)code_at(packed, k, r, kk, symmetric) - z)", "((int32_t)code_at(packed, k, r, kk, symmetric) + z)"),
    ("a8: down projection's activation scale dropped", "int orc_moe_experts_a8(",
     "o = w4a8_dot(hq, sh, dp, ds, dz, symmetric, I, group, c);", "o = w4a8_dot(hq, 1.0, dp, ds, dz, symmetric, I, group, c);"),
    ("a8: gate codes rescaled by the up matrix's scales", "int orc_moe_experts_a8(",
     "gv = w4a8_dot(xq, sa, gp, gs, gz, symmetric, H, group, i);", "gv = w4a8_dot(xq, sa, gp, us, gz, symmetric, H, group, i);"),
    ("router: top-k takes the smallest logits", "int orc_route(", "l[e] > l[best]", "l[e] < l[best]"),
    ("two's complement by 8 instead of 16", "static int code_at(", "if (symmetric && v >= 8) v -= 16;",
     "if (symmetric && v >= 8) v -= 8;"),
    ("symmetric codes truncated, not rounded", "int orc_quantize(",
     "(int)clampf(rne(src[i] / S), -8.0f, 7.0f)", "(int)clampf(truncf(src[i] / S), -8.0f, 7.0f)"),
    ("W4A8: symmetric codes read as unsigned", "void orc_linear_w4a8(",
     "((int32_t)code_at(packed, k, r, kk, symmetric) - z)", "((int32_t)code_at(packed, k, r, kk, 0) - z)"),
    ("bf16 widening shifted by 15", "float orc_bf16_to_f32(uint16_t b)", "(uint32_t)b << 16", "(uint32_t)b << 15"),
    ("act quant: amax over the first half of the row", "static float act_quant_row(",
     "for (int kk = 0; kk < k; kk++) {\n        if (!isfinite(v[kk])) *bad = 1;",
     "for (int kk = 0; kk < k / 2; kk++) {\n        if (!isfinite(v[kk])) *bad = 1;"),
    ("MoE: the last chosen expert left out", "void orc_moe_experts(",
     "for (int j = 0; j < topk; j++) {\n            int e = ids[(size_t)t * topk + j];\n            /* the expert's row blocks",
     "for (int j = 0; j < topk - 1; j++) {\n            int e = ids[(size_t)t * topk + j];\n            /* the expert's row blocks"),
]


def plant(src: str, scope: str, old: str, new: str) -> str:
    """Replace the one occurrence of `old` inside the function that starts at `scope`."""
    a = src.index(scope)
    b = src.index("\n}\n", a)
    body = src[a:b]
    assert body.count(old) == 1, (scope, old, body.count(old))
    return src[:a] + body.replace(old, new) + src[b:]


def _run_pins(lib_path: str):
    env = dict(os.environ, Q4_ORACLE_LIB=lib_path, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", PINS, "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    failed = re.findall(r"^FAILED (\S+)", r.stdout, re.M)
    return r.returncode, failed, r.stdout[-2000:]


def _build_and_run(src: str, path: str):
    with open(path + ".c", "w") as f:
        f.write(src)
    subprocess.check_call(["gcc", *oracle.CFLAGS, path + ".c", "-o", path + ".so", "-lm"])
    return _run_pins(path + ".so")


def test_every_planted_mistake_fails_a_pin(tmp_path):
    with open(os.path.join(ROOT, "oracle", "q4_oracle.c")) as f:
        src = f.read()
    planted = [(name, plant(src, scope, old, new)) for name, scope, old, new in MUTANTS]
    assert len({name for name, _ in planted}) == len(planted)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        clean = ex.submit(_build_and_run, src, str(tmp_path / "clean"))
        runs = {name: ex.submit(_build_and_run, s, str(tmp_path / f"m{i}")) for i, (name, s) in enumerate(planted)}
        rc, failed, out = clean.result()
        assert rc == 0 and not failed, f"the unmodified oracle must pass its pins:\n{out}"
        survivors, crashed = [], []
        for name, fut in runs.items():
            rc, failed, out = fut.result()
            if rc == 1 and failed:
                continue                       # a pin failed: the mistake is caught
            (survivors if rc == 0 else crashed).append((name, rc, out[-400:]))
    assert not crashed, f"mutants that did not run to a pin failure: {crashed}"
    assert not survivors, f"mistakes no pin catches: {[s[0] for s in survivors]}"


# The compositions the oracle does in numpy (oracle/__init__.py): each replaced, in this process, by a
# plausible wrong version; the pins that cover it must fail.  (Only mistakes that stay inside the arrays:
# the C functions they call are not bounds-checked.)
def _silu_wrong_sign(g, u):
    g = np.asarray(g, np.float32).astype(np.float64)
    return g / (1.0 + np.exp(g)) * np.asarray(u, np.float32).astype(np.float64)


def _sigmoid_not_silu(g, u):
    g = np.asarray(g, np.float32).astype(np.float64)
    return 1.0 / (1.0 + np.exp(-g)) * np.asarray(u, np.float32).astype(np.float64)


def _silu_in_fp32(g, u):
    g, u = np.asarray(g, np.float32), np.asarray(u, np.float32)
    return (g / (np.float32(1.0) + np.exp(-g)) * u).astype(np.float64)


def _swiglu_gate_only(gate, up, packed, scales, zeros, n, k, group, symmetric):
    h = _REAL["silu_mul"](gate, np.ones_like(np.asarray(up, np.float32))).reshape(-1, k)
    return h @ oracle.dequant(packed, scales, zeros, k, group, symmetric).astype(np.float64).T


def _swiglu_untransposed(gate, up, packed, scales, zeros, n, k, group, symmetric):
    h = _REAL["silu_mul"](gate, up).reshape(-1, k)
    return h @ oracle.dequant(packed, scales, zeros, k, group, symmetric).astype(np.float64)


def _shared_half_weight(x, H, gate, up, down, I_s, group, symmetric, tokens=None):
    return 0.5 * _REAL["shared_expert"](x, H, gate, up, down, I_s, group, symmetric, tokens=tokens)


def _classes_foreign_slots_kept(x, H, ids, w, class_begin, classes, I, tokens=None):
    ids = np.asarray(ids, np.int32)
    y = None
    for c, (gate, up, down, group, symmetric) in enumerate(classes):
        e0, e1 = int(class_begin[c]), int(class_begin[c + 1])
        mine = (ids >= e0) & (ids < e1)
        ids_c = np.where(mine, ids - e0, 0).astype(np.int32)
        yc = oracle.moe_experts(x, H, ids_c, np.asarray(w, np.float64), gate, up, down, I, group, symmetric,
                                tokens=tokens)
        y = yc if y is None else y + yc
    return y


_REAL = {name: getattr(oracle, name) for name in ("silu_mul", "shared_expert")}


def test_every_planted_mistake_in_the_numpy_compositions_fails_a_pin(monkeypatch):
    from tests import test_oracle_pins as pins
    swiglu_pins = [pins.test_silu_mul_identities, pins.test_swiglu_linear_reduces_to_plain_linear_for_saturated_gate]
    class_pins = [pins.test_moe_classes_one_class_and_equal_classes_are_the_layer,
                  pins.test_moe_classes_each_expert_uses_its_class_quantization]
    cases = [
        ("silu_mul", _silu_wrong_sign, swiglu_pins),
        ("silu_mul", _sigmoid_not_silu, swiglu_pins),
        ("silu_mul", _silu_in_fp32, swiglu_pins),
        ("linear_w4a16_swiglu", _swiglu_gate_only, swiglu_pins),
        ("linear_w4a16_swiglu", _swiglu_untransposed, swiglu_pins),
        ("shared_expert", _shared_half_weight, [pins.test_shared_expert_is_the_dense_swiglu_ffn]),
        ("moe_experts_classes", _classes_foreign_slots_kept, class_pins),
    ]
    for _, _, checks in cases:          # the real compositions pass their pins
        for check in checks:
            check()
    survivors = []
    for name, wrong, checks in cases:
        monkeypatch.setattr(oracle, name, wrong)
        caught = False
        for check in checks:
            try:
                check()
            except Exception:
                caught = True
                break
        monkeypatch.undo()
        if not caught:
            survivors.append(f"{name}: {wrong.__name__}")
    assert not survivors, f"mistakes no pin catches: {survivors}"
