"""The debug build (libq4_debug.so, Q4_DEBUG): every global-memory index a kernel computes is checked
against its buffer before the access, and a failed check is reported as Q4_ERR_BOUNDS instead of being
made -- the stand-in for a memory checker.  Here it runs a small case of every kernel family (GEMV, the
GEMV chain, act-quant, the W4A16 and W4A8 tensor-core GEMMs, the MoE layer and its steps) in a process of
its own: no check fires on valid inputs, and the results match the oracle as the release build's do."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import numpy as np, torch
import oracle
from moe_linear_layers_b200 import q4, synth
from tests._util import assert_close, cuda_u16_as, upload_weight
assert q4.LIB_PATH.endswith("libq4_debug.so") and q4._lib.q4_build_flags() & 1
st = torch.zeros(1, dtype=torch.int32, device="cuda")
# GEMV (m = 1 and 3) and the GEMV chain
for m, (n, k) in ((1, (200, 512)), (3, (130, 8192))):
    W = synth.weights(("dbg", n, k), n, k); q = oracle.quantize(W, 128, False)
    w = upload_weight(q4, *q, n, k, 128, False)
    x = synth.activations(("dbg-x", m, k), m, k)
    y = q4.q4_linear_w4a16(cuda_u16_as(x, torch.bfloat16), w, dev_status=st)
    torch.cuda.synchronize(); assert int(st.item()) == 0
    assert_close(y.cpu().numpy(), oracle.linear_w4a16(x, *q, n, k, 128, False), what=f"gemv m={m}")
    if m == 1:
        y2 = torch.empty((n,), dtype=torch.float32, device="cuda")
        xs = cuda_u16_as(x, torch.bfloat16).view(-1)
        q4.GemvChain([[(xs, w, y2)], [(xs, w, y)]])(dev_status=st)
        torch.cuda.synchronize(); assert int(st.item()) == 0
        assert_close(y2.cpu().numpy(), oracle.linear_w4a16(x, *q, n, k, 128, False)[0], what="chain")
# act-quant, W4A16 and W4A8 GEMMs with a ragged tile
n, k, m = 300, 1024, 150
W = synth.weights(("dbg-gemm",), n, k)
qa, qs = oracle.quantize(W, 128, False), oracle.quantize(W, 128, True)
x = synth.activations(("dbg-gemm-x",), m, k)
y = q4.q4_linear_w4a16(cuda_u16_as(x, torch.bfloat16), upload_weight(q4, *qa, n, k, 128, False), dev_status=st)
xq, sa = q4.act_quant_per_token(cuda_u16_as(x, torch.bfloat16), dev_status=st)
acc = torch.empty((m, n, k // 128), dtype=torch.int32, device="cuda")
y8 = q4.q4_linear_w4a8(xq, sa, upload_weight(q4, *qs, n, k, 128, True), acc_dbg=acc, dev_status=st)
torch.cuda.synchronize(); assert int(st.item()) == 0
assert_close(y.cpu().numpy(), oracle.linear_w4a16(x, *qa, n, k, 128, False), what="w4a16 gemm")
xq_r, sa_r = oracle.act_quant(x, k)
y8_r, acc_r = oracle.linear_w4a8(xq_r, sa_r, qs[0], qs[1], n, k, 128, want_acc=True)
assert np.array_equal(acc.cpu().numpy(), acc_r)
assert_close(y8.cpu().numpy(), y8_r, what="w4a8 gemm")
# the MoE layer (16-bit and INT8 experts) and its steps as separate calls
T, H, I, E, topk = 70, 256, 128, 6, 2
x = synth.activations(("dbg-moe-x",), T, H)
Wr, bias = synth.router(("dbg-moe",), E, H)
qx = [oracle.quantize(synth.weights(("dbg-moe", nm), nn, kk), 64, False)
      for nm, nn, kk in (("g", E * I, H), ("u", E * I, H), ("d", E * H, I))]
ex = tuple(upload_weight(q4, *q, nn, kk, 64, False) for q, nn, kk in zip(qx, (E * I, E * I, E * H), (H, H, I)))
_, ids, w, _ = oracle.route(x, H, Wr, bias, topk)
ref = oracle.moe_experts(x, H, ids, w, *qx, I, 64, False)
xd, Wrd, bd = cuda_u16_as(x, torch.bfloat16), torch.from_numpy(Wr).cuda(), torch.from_numpy(bias).cuda()
ym = q4.moe_q4_forward(xd, Wrd, bd, topk, ex, I, dev_status=st)
y8m = q4.moe_q4_forward(xd, Wrd, bd, topk, ex, I, dev_status=st, a8_mask=3)
r = q4.moe_q4_route(xd, Wrd, bd, topk, dev_status=st)
o = q4.moe_q4_forward_rows(r["x_perm"], r["row_expert"], 0, ex, I, dev_status=st)
yc = q4.moe_q4_combine(o, r["pair_pos"], r["topk_w"], dev_status=st)
torch.cuda.synchronize(); assert int(st.item()) == 0
assert_close(ym.cpu().numpy(), ref, what="moe")
assert_close(yc.cpu().numpy(), ref, what="moe steps")
assert_close(y8m.cpu().numpy(), oracle.moe_experts_a8(x, H, ids, w, *qx, I, 64, False, 3), what="moe a8")
print("debug build ok")
'''


def test_debug_build_no_false_positives_and_same_results():
    lib = os.path.join(ROOT, "moe_linear_layers_b200", "libq4_debug.so")
    assert os.path.exists(lib), "libq4_debug.so is missing: build it with build_lib --debug"
    env = dict(os.environ, Q4_DEBUG_LIBRARY="1", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "debug build ok" in r.stdout
