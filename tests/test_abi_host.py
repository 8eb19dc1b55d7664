"""The C ABI library loads, exports every function include/q4.h declares, and rejects bad arguments on
the host before any CUDA call (no GPU needed: every call below returns before touching the device)."""
import ctypes
import os
import re

import pytest

from moe_linear_layers_b200 import q4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            with open(os.path.join(ROOT, "include", fn)) as f:
                src = f.read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(\w+)\s*\(", src, flags=re.M)
    return names


def test_exports_every_declared_function():
    names = _declared_functions()
    assert {"q4_quantize_pack", "q4_linear_w4a16", "act_quant_per_token", "q4_linear_w4a8",
            "moe_q4_forward", "moe_q4_workspace_size"} <= set(names)
    lib = ctypes.CDLL(q4.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(q4.EXPORTED)


def test_status_strings():
    assert q4.status_string(0) == "ok"
    assert "aligned" in q4.status_string(q4.Q4_ERR_ALIGN)
    assert q4.version() >= 1


FAKE = 0x10000  # never dereferenced: every call below fails validation first


def _w(n=128, k=256, group=64, sym=1, packed=FAKE, scales=FAKE, zeros=None):
    return q4.q4_weight(n, k, group, sym, packed, scales, zeros)


@pytest.mark.parametrize("args,expect", [
    (dict(w=None), q4.Q4_ERR_NULL),
    (dict(w=_w(packed=None)), q4.Q4_ERR_NULL),
    (dict(w=_w(sym=0, zeros=None)), q4.Q4_ERR_NULL),
    (dict(w=_w(group=32)), q4.Q4_ERR_SHAPE),      # group 32 serves the MoE expert GEMMs only
    (dict(w=_w(k=200)), q4.Q4_ERR_SHAPE),
    (dict(w=_w(packed=FAKE + 4)), q4.Q4_ERR_ALIGN),
    (dict(x=FAKE + 2), q4.Q4_ERR_ALIGN),
    (dict(x=None), q4.Q4_ERR_NULL),
    (dict(m=-1), q4.Q4_ERR_SHAPE),
    (dict(out_dtype=7), q4.Q4_ERR_UNSUPPORTED),
])
def test_linear_w4a16_validation(args, expect):
    a = dict(x=FAKE, m=1, w=_w(), y=FAKE, out_dtype=0)
    a.update(args)
    w = a["w"]
    rc = q4._lib.q4_linear_w4a16(a["x"], a["m"], ctypes.byref(w) if w is not None else None, a["y"],
                                 a["out_dtype"], None, None)
    assert rc == expect


def test_w4a8_asymmetric_weights_need_zero_points():
    w = _w(sym=0, zeros=None)
    rc = q4._lib.q4_linear_w4a8(FAKE, FAKE, 16, ctypes.byref(w), FAKE, 0, None, None, None)
    assert rc == q4.Q4_ERR_NULL


def test_quantize_validation():
    L = q4._lib
    assert L.q4_quantize_pack(None, 4, 128, 64, 1, FAKE, FAKE, None, None, None) == q4.Q4_ERR_NULL
    assert L.q4_quantize_pack(FAKE, 4, 128, 48, 1, FAKE, FAKE, None, None, None) == q4.Q4_ERR_SHAPE
    assert L.q4_quantize_pack(FAKE, 4, 128, 256, 1, FAKE, FAKE, None, None, None) == q4.Q4_ERR_SHAPE   # k % 256
    assert L.q4_quantize_pack(FAKE, 4, 512, 256, 1, FAKE + 8, FAKE, None, None, None) == q4.Q4_ERR_ALIGN  # 256 accepted
    assert L.q4_quantize_pack(FAKE, 4, 1024, 512, 1, FAKE, FAKE, None, None, None) == q4.Q4_ERR_SHAPE
    assert L.q4_quantize_pack(FAKE, 4, 96, 32, 1, FAKE + 8, FAKE, None, None, None) == q4.Q4_ERR_ALIGN  # 32 accepted
    assert L.q4_quantize_pack(FAKE, 4, 100, 64, 1, FAKE, FAKE, None, None, None) == q4.Q4_ERR_SHAPE
    assert L.q4_quantize_pack(FAKE + 8, 4, 128, 64, 1, FAKE, FAKE, None, None, None) == q4.Q4_ERR_ALIGN
    assert L.q4_quantize_pack(FAKE, 4, 128, 64, 0, FAKE, FAKE, None, None, None) == q4.Q4_ERR_NULL


def test_act_quant_validation():
    L = q4._lib
    assert L.act_quant_per_token(None, 4, 128, FAKE, FAKE, None, None) == q4.Q4_ERR_NULL
    assert L.act_quant_per_token(FAKE, 4, 12, FAKE, FAKE, None, None) == q4.Q4_ERR_SHAPE
    assert L.act_quant_per_token(FAKE + 2, 4, 128, FAKE, FAKE, None, None) == q4.Q4_ERR_ALIGN
    assert L.act_quant_per_token_f16(None, 4, 128, FAKE, FAKE, None, None) == q4.Q4_ERR_NULL
    assert L.act_quant_per_token_f16(FAKE, 4, 12, FAKE, FAKE, None, None) == q4.Q4_ERR_SHAPE
    assert L.act_quant_per_token_f16(FAKE, 4, 128, FAKE + 8, FAKE, None, None) == q4.Q4_ERR_ALIGN


def test_moe_a8_validation_and_workspace():
    L = q4._lib
    T, H, I, E, topk = 64, 256, 128, 8, 2
    base = L.moe_q4_workspace_size(T, H, I, E, topk)
    # each INT8 path adds its codes and scales: x codes + token and row scales; h codes + row scales
    assert L.moe_q4_workspace_size_a8(T, H, I, E, topk, 0) == base
    assert L.moe_q4_workspace_size_a8(T, H, I, E, topk, 1) >= base + T * H + 4 * T + 4 * T * topk
    assert L.moe_q4_workspace_size_a8(T, H, I, E, topk, 2) >= base + T * topk * I + 4 * T * topk
    assert L.moe_q4_workspace_size_a8(T, H, I, E, topk, 4) == 0
    ex = (q4.q4_weight * 3)(_w(n=E * I, k=H), _w(n=E * I, k=H), _w(n=E * H, k=I))
    args = (FAKE, T, H, FAKE, None, E, topk, ex, I)
    assert L.moe_q4_forward_a8(*args, 4, FAKE, 0, None, None, None, None, None, FAKE, 1 << 30, None, None) == q4.Q4_ERR_UNSUPPORTED
    assert L.moe_q4_forward_a8(*args, -1, FAKE, 0, None, None, None, None, None, FAKE, 1 << 30, None, None) == q4.Q4_ERR_UNSUPPORTED
    need = L.moe_q4_workspace_size_a8(T, H, I, E, topk, 3)
    assert L.moe_q4_forward_a8(*args, 3, FAKE, 0, None, None, None, None, None, FAKE, need - 1, None, None) == q4.Q4_ERR_WORKSPACE
    assert L.moe_q4_forward_a8(None, T, H, FAKE, None, E, topk, ex, I, 3, FAKE, 0, None, None, None, None, None, FAKE,
                               need, None, None) == q4.Q4_ERR_NULL


def test_grouped_validation():
    L = q4._lib
    ws = (q4.q4_weight * 2)(_w(), _w(k=512))
    xs = (ctypes.c_void_p * 2)(FAKE, FAKE)
    ys = (ctypes.c_void_p * 2)(FAKE, FAKE)
    assert L.q4_linear_w4a16_grouped(2, xs, 1, ws, ys, 0, None, None) == q4.Q4_ERR_SHAPE   # k differs
    ws2 = (q4.q4_weight * 2)(_w(), _w())
    assert L.q4_linear_w4a16_grouped(9, xs, 1, ws2, ys, 0, None, None) == q4.Q4_ERR_SHAPE  # too many
    assert L.q4_linear_w4a16_grouped(2, xs, 5, ws2, ys, 0, None, None) == q4.Q4_ERR_SHAPE  # m > 4
    xs_bad = (ctypes.c_void_p * 2)(FAKE, FAKE + 2)
    assert L.q4_linear_w4a16_grouped(2, xs_bad, 1, ws2, ys, 0, None, None) == q4.Q4_ERR_ALIGN


def test_moe_classes_validation():
    L = q4._lib
    T, H, I, E, topk = 64, 256, 128, 8, 2
    ws = L.moe_q4_workspace_size(T, H, I, E, topk)

    def call(begin, ex):
        b = (ctypes.c_int32 * len(begin))(*begin)
        n = len(begin) - 1
        return L.moe_q4_forward_classes(FAKE, T, H, FAKE, None, E, topk, n, b, ex, I, FAKE, 0, None, None, None,
                                        None, None, FAKE, ws, None, None)

    two = (q4.q4_weight * 6)(_w(n=3 * I, k=H), _w(n=3 * I, k=H), _w(n=3 * H, k=I),
                             _w(n=5 * I, k=H, group=128, sym=0, zeros=FAKE), _w(n=5 * I, k=H, group=128, sym=0, zeros=FAKE),
                             _w(n=5 * H, k=I, group=128, sym=0, zeros=FAKE))
    assert call([0, 3, 9], two) == q4.Q4_ERR_SHAPE          # last bound != E
    assert call([0, 4, 8], two) == q4.Q4_ERR_SHAPE          # class sizes do not match the weights
    assert call([1, 3, 8], two) == q4.Q4_ERR_SHAPE          # first bound != 0
    assert call([0, 0, 8], two) == q4.Q4_ERR_SHAPE          # empty class
    mixed = (q4.q4_weight * 6)(*two)
    mixed[4] = _w(n=5 * I, k=H, group=64, sym=0, zeros=FAKE)  # up of class 1 with another group
    assert call([0, 3, 8], mixed) == q4.Q4_ERR_UNSUPPORTED
    assert L.moe_q4_forward_classes(FAKE, T, H, FAKE, None, E, topk, 2, None, two, I, FAKE, 0, None, None, None,
                                    None, None, FAKE, ws, None, None) == q4.Q4_ERR_NULL
    ok = (ctypes.c_int32 * 3)(0, 3, 8)
    assert L.moe_q4_forward_classes(FAKE, T, H, FAKE, None, E, topk, 2, ok, two, I, FAKE, 0, None, None, None,
                                    None, None, FAKE, ws - 1, None, None) == q4.Q4_ERR_WORKSPACE


def test_moe_group32_only_on_the_16bit_path():
    L = q4._lib
    T, H, I, E, topk = 64, 256, 128, 8, 2
    ex = (q4.q4_weight * 3)(_w(n=E * I, k=H, group=32), _w(n=E * I, k=H, group=32), _w(n=E * H, k=I, group=32))
    need = L.moe_q4_workspace_size_a8(T, H, I, E, topk, 3)
    assert L.moe_q4_forward_a8(FAKE, T, H, FAKE, None, E, topk, ex, I, 3, FAKE, 0, None, None, None, None, None, FAKE,
                               need, None, None) == q4.Q4_ERR_UNSUPPORTED


def test_moe_range_validation():
    L = q4._lib
    T, H, I, E, topk = 64, 256, 128, 8, 2
    ws = L.moe_q4_workspace_size(T, H, I, E, topk)
    ex3 = (q4.q4_weight * 3)(_w(n=3 * I, k=H), _w(n=3 * I, k=H), _w(n=3 * H, k=I))

    def call(e0, e1, ex=ex3, wsb=ws):
        return L.moe_q4_forward_range(FAKE, T, H, FAKE, None, E, topk, e0, e1, ex, I, FAKE, None, None, None, None,
                                      None, FAKE, wsb, None, None)

    assert call(3, 3) == q4.Q4_ERR_SHAPE          # empty range
    assert call(6, 9) == q4.Q4_ERR_SHAPE          # past the last expert
    assert call(-1, 2) == q4.Q4_ERR_SHAPE
    assert call(2, 4) == q4.Q4_ERR_SHAPE          # 2 experts, weights stacked for 3
    assert call(2, 5, wsb=ws - 1) == q4.Q4_ERR_WORKSPACE


@pytest.mark.parametrize("y,err", [
    (lambda: __import__("torch").empty((4, 8), dtype=__import__("torch").float16), TypeError),   # fp16: no ABI code
    (lambda: __import__("torch").empty((4, 7), dtype=__import__("torch").float32), ValueError),  # smaller than [T][H]
    (lambda: __import__("torch").empty((8, 4), dtype=__import__("torch").float32).t(), ValueError),  # not contiguous
    (lambda: __import__("torch").empty((4, 8), dtype=__import__("torch").float32), TypeError),   # host memory
    (lambda: [0.0] * 32, TypeError),
])
def test_output_checked_before_any_launch(y, err):
    """A caller-supplied output of the wrong dtype, shape, layout or memory is refused by the binding (the
    ABI would read an fp16 buffer as fp32 and write past a short one)."""
    import torch
    with pytest.raises(err):
        q4._out(y(), (4, 8), torch.device("cuda", 0))


def test_chain_validation():
    L = q4._lib
    P = ctypes.c_void_p
    assert L.q4_linear_w4a16_chain_sync_bytes(64) == 65 * 128 and L.q4_linear_w4a16_chain_sync_bytes(0) == 0

    def call(begin, ws, xs=None, ys=None, sync=FAKE, gate=None, up=None, out=0):
        n = len(ws)
        b = (ctypes.c_int32 * len(begin))(*begin)
        w = (q4.q4_weight * n)(*ws)
        x = xs if xs is not None else (P * n)(*([FAKE] * n))
        y = ys if ys is not None else (P * n)(*([FAKE] * n))
        return L.q4_linear_w4a16_chain(len(begin) - 1, b, x, gate, up, w, y, out, sync, None, None)

    w2 = [_w(group=128, sym=0, zeros=FAKE), _w(group=128, sym=0, zeros=FAKE)]
    assert call([0, 1, 2], w2, sync=None) == q4.Q4_ERR_NULL
    assert call([0, 1, 2], w2, sync=FAKE + 2) == q4.Q4_ERR_ALIGN
    assert call([1, 2], w2) == q4.Q4_ERR_SHAPE                    # stage_begin[0] != 0
    assert call([0, 0, 2], w2) == q4.Q4_ERR_SHAPE                 # an empty stage
    assert call([0, 9] + [9] * 0, [w2[0]] * 9) == q4.Q4_ERR_SHAPE  # 9 problems in one stage
    assert call([0, 1, 2], [w2[0], _w(group=64)]) == q4.Q4_ERR_UNSUPPORTED   # group/symmetry differ
    assert call([0, 1, 2], w2, out=5) == q4.Q4_ERR_UNSUPPORTED
    assert call([0, 1, 2], w2, xs=(P * 2)(FAKE, None)) == q4.Q4_ERR_NULL
    assert call([0, 1, 2], w2, ys=(P * 2)(FAKE, FAKE + 4)) == q4.Q4_ERR_ALIGN
    g = (P * 2)(None, FAKE)
    assert call([0, 1, 2], w2, gate=g, up=(P * 2)(None, None)) == q4.Q4_ERR_NULL   # gated without up
    assert call([0, 1, 2], w2, gate=g, up=(P * 2)(None, FAKE + 8)) == q4.Q4_ERR_ALIGN


def test_moe_steps_validation():
    L = q4._lib
    T, H, I, E, topk = 64, 256, 128, 8, 2
    rws = L.moe_q4_route_workspace_size(T, E, topk)
    assert rws > 0 and L.moe_q4_route_workspace_size(T, 0, topk) == 0

    def route(x=FAKE, ids=FAKE, pp=FAKE, e=E, k=topk, ws=FAKE, wsb=rws, xp=None):
        return L.moe_q4_route(x, T, H, FAKE, None, e, k, ids, FAKE, FAKE, pp, xp, None, None, None, ws, wsb, None, None)

    assert route(ids=None) == q4.Q4_ERR_NULL
    assert route(pp=None) == q4.Q4_ERR_NULL
    assert route(k=9, e=8) == q4.Q4_ERR_SHAPE
    assert route(e=300) == q4.Q4_ERR_SHAPE
    assert route(x=FAKE + 2) == q4.Q4_ERR_ALIGN
    assert route(xp=FAKE + 8) == q4.Q4_ERR_ALIGN
    assert route(ws=FAKE + 16) == q4.Q4_ERR_ALIGN
    assert route(wsb=rws - 1) == q4.Q4_ERR_WORKSPACE
    ex = (q4.q4_weight * 3)(_w(n=E * I, k=H), _w(n=E * I, k=H), _w(n=E * H, k=I))
    need = L.moe_q4_rows_workspace_size(T, H, I, E)

    def rows(exw=ex, y=FAKE, wsb=need, e=E):
        return L.moe_q4_forward_rows(FAKE, T, H, FAKE, 0, None, e, exw, I, y, FAKE, wsb, None, None)

    assert rows(y=None) == q4.Q4_ERR_NULL
    assert rows(e=7) == q4.Q4_ERR_SHAPE            # weights stacked for 8 experts
    assert rows(y=FAKE + 4) == q4.Q4_ERR_ALIGN
    assert rows(wsb=need - 1) == q4.Q4_ERR_WORKSPACE
    assert L.moe_q4_combine(None, 10, H, FAKE, FAKE, 5, 2, FAKE, 0, None, None) == q4.Q4_ERR_NULL
    assert L.moe_q4_combine(FAKE, 10, 6, FAKE, FAKE, 5, 2, FAKE, 0, None, None) == q4.Q4_ERR_SHAPE
    assert L.moe_q4_combine(FAKE, 10, H, FAKE, FAKE, 5, 2, FAKE, 3, None, None) == q4.Q4_ERR_UNSUPPORTED
    assert L.moe_q4_combine(FAKE, 10, H, FAKE, FAKE, 5, 2, FAKE + 8, 0, None, None) == q4.Q4_ERR_ALIGN


def test_binding_argument_checks():
    """The binding's checks of MoE arguments the C ABI cannot see (it takes pointers and sizes): the router's
    shape, the bias's dtype, length and device, a caller workspace's dtype and device, and input lengths;
    each raises before any library call."""
    import torch
    cpu = torch.device("cpu")
    w = torch.zeros((8, 256), dtype=torch.float32)
    assert q4._router(w, None, 256, cpu) == 8
    assert q4._router(w, torch.zeros(8, dtype=torch.float32), 256, cpu) == 8
    with pytest.raises(ValueError):
        q4._router(w, None, 512, cpu)                                    # x is [T][512]
    with pytest.raises(ValueError):
        q4._router(torch.zeros(8 * 256, dtype=torch.float32), None, 256, cpu)   # not 2-D
    with pytest.raises(TypeError):
        q4._router(w, torch.zeros(8, dtype=torch.float64), 256, cpu)
    with pytest.raises(ValueError):
        q4._router(w, torch.zeros(7, dtype=torch.float32), 256, cpu)
    with pytest.raises(ValueError):
        q4._router(w, torch.zeros(16, dtype=torch.float32)[::2], 256, cpu)     # not contiguous
    with pytest.raises(ValueError):
        q4._router(w, None, 256, torch.device("meta"))                   # on another device than x
    ws = torch.zeros(64, dtype=torch.uint8)
    assert q4._workspace(ws, cpu) is ws
    with pytest.raises(TypeError):
        q4._workspace(torch.zeros(16, dtype=torch.float32), cpu)        # numel would not be bytes
    with pytest.raises(ValueError):
        q4._workspace(ws, torch.device("meta"))
    with pytest.raises(ValueError):
        q4._workspace(torch.zeros(128, dtype=torch.uint8)[::2], cpu)
    assert q4._numel(torch.zeros(6), 6, "t") is not None
    with pytest.raises(ValueError):
        q4._numel(torch.zeros(5), 6, "pair_pos")


def test_linear_workspace_validation():
    """Split-K workspace of the dense GEMM: its size rule and the checks of a caller workspace."""
    L = q4._lib
    w = _w(n=2048, k=2048, group=128, sym=1)
    need = L.q4_linear_workspace_size(64, ctypes.byref(w))
    assert need > 0 and need % 256 == 0                          # 16 output tiles: split
    assert L.q4_linear_workspace_size(4096, ctypes.byref(_w(n=8192, k=2048, group=128))) == 0   # enough tiles
    assert L.q4_linear_workspace_size(64, ctypes.byref(_w(n=2048, k=256, group=128))) == 0      # 2 K blocks
    assert L.q4_linear_workspace_size(0, ctypes.byref(w)) == 0
    P = ctypes.c_void_p
    call = lambda ws, nb: L.q4_linear_w4a16_ws(P(FAKE), 64, ctypes.byref(w), P(FAKE), 0, P(ws) if ws else None, nb,
                                               None, None)
    assert call(FAKE + 16, need) == q4.Q4_ERR_ALIGN
    assert call(FAKE, need - 1) == q4.Q4_ERR_WORKSPACE
    call8 = lambda ws, nb: L.q4_linear_w4a8_ws(P(FAKE), P(FAKE), 64, ctypes.byref(w), P(FAKE), 0, None,
                                               P(ws) if ws else None, nb, None, None)
    assert call8(FAKE + 16, need) == q4.Q4_ERR_ALIGN
    assert call8(FAKE, need - 1) == q4.Q4_ERR_WORKSPACE


def test_weight_stack_is_a_row_concatenation():
    """Q4Weight.stack copies the parts' packed rows, scales and zero points one after another (CPU tensors:
    no library call) and refuses parts of different k, group or symmetry."""
    import torch
    def part(n, k=256, group=128, sym=False, fill=0):
        packed = torch.full((n, k // 2), fill, dtype=torch.uint8)
        scales = torch.full((n, k // group), float(fill), dtype=torch.float16)
        zeros = None if sym else torch.full((n, k // group), float(fill + 1), dtype=torch.float16)
        return q4.Q4Weight(packed, scales, zeros, n, k, group, sym)
    a, b, c = part(64, fill=1), part(16, fill=2), part(16, fill=3)
    st = q4.Q4Weight.stack([a, b, c])
    assert (st.n, st.k, st.group, st.symmetric) == (96, 256, 128, False)
    assert torch.equal(st.packed[64:80], b.packed) and torch.equal(st.scales[80:], c.scales)
    assert torch.equal(st.zeros[:64], a.zeros)
    assert q4.Q4Weight.stack([part(8, sym=True), part(8, sym=True)]).zeros is None
    for bad in (part(8, k=512), part(8, group=64), part(8, sym=True)):
        with pytest.raises(ValueError):
            q4.Q4Weight.stack([a, bad])


def test_empty_problems_launch_nothing():
    """A problem without rows is valid: its sizes, options and weights are still checked, then the call
    returns Q4_OK without launching, and the arrays that hold no elements may be NULL (a zero-element
    tensor has no storage).  No call below reaches the device: every pointer given is a placeholder."""
    L = q4._lib
    w = _w(n=128, k=256, group=64)
    assert L.q4_linear_w4a16(None, 0, ctypes.byref(w), None, 0, None, None) == q4.Q4_OK
    assert L.q4_linear_w4a16_ws(None, 0, ctypes.byref(w), None, 1, None, 0, None, None) == q4.Q4_OK
    assert L.q4_linear_w4a8(None, None, 0, ctypes.byref(w), None, 0, None, None, None) == q4.Q4_OK
    assert L.act_quant_per_token(None, 0, 128, None, None, None, None) == q4.Q4_OK
    assert L.act_quant_per_token_f16(None, 0, 128, None, None, None, None) == q4.Q4_OK
    assert L.q4_quantize_pack(None, 0, 128, 64, 0, None, None, None, None, None) == q4.Q4_OK
    assert L.q4_quantize_pack(None, 0, 100, 64, 0, None, None, None, None, None) == q4.Q4_ERR_SHAPE
    # what an empty problem can still get wrong is still reported
    assert L.q4_linear_w4a16(None, 0, ctypes.byref(_w(k=200)), None, 0, None, None) == q4.Q4_ERR_SHAPE
    assert L.q4_linear_w4a16(None, 0, ctypes.byref(w), None, 7, None, None) == q4.Q4_ERR_UNSUPPORTED
    assert L.q4_linear_w4a16(None, -1, ctypes.byref(w), None, 0, None, None) == q4.Q4_ERR_SHAPE
    assert L.act_quant_per_token(None, 0, 12, None, None, None, None) == q4.Q4_ERR_SHAPE
    assert L.q4_linear_w4a16(None, 1, ctypes.byref(w), FAKE, 0, None, None) == q4.Q4_ERR_NULL   # one row needs x
    # the MoE layer and its steps with no tokens / rows (no optional routing outputs: nothing to zero)
    H, I, E, topk = 256, 128, 8, 2
    ex = (q4.q4_weight * 3)(_w(n=E * I, k=H), _w(n=E * I, k=H), _w(n=E * H, k=I))
    ws = L.moe_q4_workspace_size(0, H, I, E, topk)
    assert L.moe_q4_forward(None, 0, H, FAKE, None, E, topk, ex, I, None, 0, None, None, None, None, None, FAKE, ws,
                            None, None) == q4.Q4_OK
    assert L.moe_q4_forward(None, 0, 200, FAKE, None, E, topk, ex, I, None, 0, None, None, None, None, None, FAKE,
                            ws, None, None) == q4.Q4_ERR_UNSUPPORTED           # H % 128
    assert L.moe_q4_forward(None, 0, H, None, None, E, topk, ex, I, None, 0, None, None, None, None, None, FAKE, ws,
                            None, None) == q4.Q4_ERR_NULL                      # the router is still needed
    assert L.moe_q4_forward(None, 1, H, FAKE, None, E, topk, ex, I, FAKE, 0, None, None, None, None, None, FAKE,
                            L.moe_q4_workspace_size(1, H, I, E, topk), None, None) == q4.Q4_ERR_NULL
    rws = L.moe_q4_rows_workspace_size(0, H, I, E)
    assert L.moe_q4_forward_rows(None, 0, H, None, 0, None, E, ex, I, None, FAKE, rws, None, None) == q4.Q4_OK
    assert L.moe_q4_combine(None, 0, H, None, None, 0, topk, None, 0, None, None) == q4.Q4_OK
    assert L.moe_q4_combine(None, 0, H, None, None, 0, 0, None, 0, None, None) == q4.Q4_ERR_SHAPE   # topk 0


def test_size_limits_are_refused_before_any_launch():
    """The largest problems a call takes: 256 experts and top-16 in the MoE layer (top-k <= E), k <= 16384
    for the decode GEMV calls.  Beyond them the call reports the size and launches nothing (every case
    here fails validation; none would reach the placeholder pointers)."""
    L = q4._lib
    T, H, I = 64, 256, 128

    def moe(E, topk):
        ex = (q4.q4_weight * 3)(_w(n=E * I, k=H), _w(n=E * I, k=H), _w(n=E * H, k=I))
        return L.moe_q4_forward(FAKE, T, H, FAKE, None, E, topk, ex, I, FAKE, 0, None, None, None, None, None, FAKE,
                                1 << 40, None, None)

    assert moe(257, 8) == q4.Q4_ERR_SHAPE      # more experts than one launch holds
    assert moe(64, 17) == q4.Q4_ERR_SHAPE      # top-k above 16
    assert moe(4, 5) == q4.Q4_ERR_SHAPE        # top-k above the expert count
    assert moe(4, 0) == q4.Q4_ERR_SHAPE
    wide = _w(n=128, k=16384 + 64, group=64)
    assert L.q4_linear_w4a16_swiglu(FAKE, FAKE, 1, ctypes.byref(wide), FAKE, 0, None, None) == q4.Q4_ERR_UNSUPPORTED
    xs, ys = (ctypes.c_void_p * 1)(FAKE), (ctypes.c_void_p * 1)(FAKE)
    assert L.q4_linear_w4a16_grouped(1, xs, 1, (q4.q4_weight * 1)(wide), ys, 0, None, None) == q4.Q4_ERR_UNSUPPORTED
    assert L.q4_linear_w4a16_swiglu(FAKE, FAKE, 5, ctypes.byref(_w()), FAKE, 0, None, None) == q4.Q4_ERR_SHAPE  # m > 4


def test_wrapper_tensors_are_held_for_the_callers_stream():
    """A call given a stream marks the tensors its wrapper made as in use by that stream (the allocator
    would otherwise hand their memory out again while the work there is queued); without a stream the
    current stream orders everything and nothing is marked."""
    class T:
        def __init__(self):
            self.streams = []

        def record_stream(self, s):
            self.streams.append(s)

    a, b = T(), T()
    q4._hold(None, a, b)
    assert a.streams == [] and b.streams == []
    q4._hold("side", a, None, b)
    assert a.streams == ["side"] and b.streams == ["side"]


def test_pair_positions_fit_int32():
    """Positions of (token, slot) pairs are int32: a call with T * topk above 2^31 - 1 is refused before
    anything is launched (a route workspace of 12 bytes per pair and the tokens themselves would still fit
    in a B200's memory at 2^28 tokens of hidden 128)."""
    L = q4._lib
    T, H, E, topk = 1 << 28, 128, 16, 16
    assert L.moe_q4_route(FAKE, T, H, FAKE, None, E, topk, FAKE, FAKE, FAKE, FAKE, None, None, None, None, FAKE,
                          1 << 40, None, None) == q4.Q4_ERR_SHAPE
    assert L.moe_q4_combine(FAKE, 0, H, FAKE, FAKE, T, topk, FAKE, 0, None, None) == q4.Q4_ERR_SHAPE
    ex = (q4.q4_weight * 3)(_w(n=E * 128, k=H), _w(n=E * 128, k=H), _w(n=E * H, k=128))
    assert L.moe_q4_forward(FAKE, T, H, FAKE, None, E, topk, ex, 128, FAKE, 0, None, None, None, None, None, FAKE,
                            1 << 40, None, None) == q4.Q4_ERR_SHAPE


def test_weight_buffers_are_checked_against_their_sizes():
    """The kernels trust a weight's n, k and group: a Q4Weight whose buffers are of another type, short,
    strided, split across devices or missing its zero points is refused when it is made, and a weight on
    another device than a call's inputs is refused at the call."""
    import torch
    n, k, g = 8, 256, 64

    def make(packed=None, scales=None, zeros="default", sym=False, **kw):
        packed = torch.zeros((n, k // 2), dtype=torch.uint8) if packed is None else packed
        scales = torch.zeros((n, k // g), dtype=torch.float16) if scales is None else scales
        zeros = torch.zeros((n, k // g), dtype=torch.float16) if isinstance(zeros, str) else zeros
        return q4.Q4Weight(packed, scales, zeros, kw.get("n", n), kw.get("k", k), kw.get("group", g), sym)

    w = make()
    assert (w.n, w.k, w.group) == (n, k, g)
    make(zeros=None, sym=True)                                             # symmetric: no zero points
    q4.Q4Weight(torch.zeros((0, k // 2), dtype=torch.uint8), torch.zeros((0, k // g), dtype=torch.float16),
                None, 0, k, g, True)                                        # an empty weight
    bad = [
        (TypeError, dict(packed=torch.zeros((n, k // 2), dtype=torch.int8))),
        (TypeError, dict(scales=torch.zeros((n, k // g), dtype=torch.float32))),
        (ValueError, dict(packed=torch.zeros((n, k // 2 - 1), dtype=torch.uint8))),     # short
        (ValueError, dict(scales=torch.zeros((k // g, n), dtype=torch.float16).t())),   # strided
        (ValueError, dict(zeros=None)),                                                 # asymmetric, no zeros
        (ValueError, dict(zeros=torch.zeros((n, k // g), dtype=torch.float16, device="meta"))),
        (ValueError, dict(k=255)),
        (ValueError, dict(group=0)),
        (ValueError, dict(k=192, group=128)),
    ]
    for err, kw in bad:
        with pytest.raises(err):
            make(**kw)
    q4._weights_on(torch.device("cpu"), w, None)
    with pytest.raises(ValueError):
        q4._weights_on(torch.device("meta"), w)
