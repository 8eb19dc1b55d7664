"""moe_q4_forward_noalloc: the MoE entry point for callers that cannot allocate device memory (for
example a plugin whose host application owns all device memory, or a latency-critical loop that must
not call cudaMalloc).  It uses the library's fixed device scratch array instead of a caller workspace.

Checked through the C ABI against the oracle (routing bit-exact, outputs within the tolerance the other
parity tests use) and against the existing entry point (moe_q4_forward with a caller workspace), on two
calls in a row (the second call reuses the scratch the first one left behind); once more through the
Python wrapper with a bf16 output.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from moe_linear_layers_b200 import synth
from tests._util import REL_TOL, assert_close, cuda_u16_as, upload_weight

pytestmark = pytest.mark.gpu


def _setup(q4, T, H, I, E, topk, group, sym):
    x = synth.activations(("noalloc", "x", T), T, H)
    Wr, bias = synth.router(("noalloc", "router"), E, H)
    Ws = [synth.weights(("noalloc", nm), n, k) for nm, n, k in (("g", E * I, H), ("u", E * I, H), ("d", E * H, I))]
    qs = [oracle.quantize(W, group, sym) for W in Ws]
    ex = (upload_weight(q4, *qs[0], E * I, H, group, sym), upload_weight(q4, *qs[1], E * I, H, group, sym),
          upload_weight(q4, *qs[2], E * H, I, group, sym))
    return x, Wr, bias, qs, ex


@pytest.mark.parametrize("T,H,I,E,topk,group,sym,sample", [
    (64, 256, 128, 8, 2, 128, False, None),
    (200, 2048, 1024, 64, 8, 128, False, np.arange(0, 200, 9)),
])
def test_noalloc_matches_oracle_and_workspace_entry_point(T, H, I, E, topk, group, sym, sample):
    from moe_linear_layers_b200 import q4
    x, Wr, bias, qs, ex = _setup(q4, T, H, I, E, topk, group, sym)
    assert q4.moe_q4_workspace_size(T, H, I, E, topk) <= q4.Q4_MOE_NOALLOC_SCRATCH_BYTES
    _, ids, w, _ = oracle.route(x, H, Wr, bias, topk)
    ref = oracle.moe_experts(x, H, ids, w, qs[0], qs[1], qs[2], I, group, sym, tokens=sample)
    xd, Wrd, bd = cuda_u16_as(x, torch.bfloat16), torch.from_numpy(Wr).cuda(), torch.from_numpy(bias).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws_y = q4.moe_q4_forward(xd, Wrd, bd, topk, ex, I, dev_status=st).cpu().numpy()
    descs = (q4.q4_weight * 3)(*[e.desc for e in ex])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rows = slice(None) if sample is None else sample
    for call in range(2):
        y = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
        ids_d = torch.full((T, topk), -1, dtype=torch.int32, device="cuda")
        rc = q4._lib.moe_q4_forward_noalloc(xd.data_ptr(), T, H, Wrd.data_ptr(), bd.data_ptr(), E, topk, descs, I,
                                            y.data_ptr(), q4.Q4_OUT_F32, ids_d.data_ptr(), None, None, None, None,
                                            st.data_ptr(), stream)
        assert rc == q4.Q4_OK, q4.status_string(rc)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert np.array_equal(ids_d.cpu().numpy(), ids), f"expert ids differ from the oracle (call {call})"
        yn = y.cpu().numpy()
        assert_close(yn[rows], ref, what=f"noalloc call {call} vs oracle")
        assert_close(yn, ws_y, what=f"noalloc call {call} vs moe_q4_forward")


def test_noalloc_python_wrapper_bf16_output():
    """The Python wrapper on the current stream with a bf16 output: within the tolerance of the fp32
    value plus the bf16 rounding of the output (2^-8 relative)."""
    from moe_linear_layers_b200 import q4
    T, H, I, E, topk, group, sym = 48, 256, 128, 8, 2, 64, True
    x, Wr, bias, qs, ex = _setup(q4, T, H, I, E, topk, group, sym)
    _, ids, w, _ = oracle.route(x, H, Wr, bias, topk)
    ref = oracle.moe_experts(x, H, ids, w, qs[0], qs[1], qs[2], I, group, sym)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = q4.moe_q4_forward_noalloc(cuda_u16_as(x, torch.bfloat16), torch.from_numpy(Wr).cuda(),
                                  torch.from_numpy(bias).cuda(), topk, ex, I, out_dtype=torch.bfloat16, dev_status=st)
    torch.cuda.synchronize()
    assert y.dtype == torch.bfloat16 and int(st.item()) == 0
    err = np.abs(y.float().cpu().numpy().astype(np.float64) - ref)
    rms = np.sqrt(np.mean(ref * ref))
    assert np.all(err <= REL_TOL * rms + 2.0 ** -8 * np.abs(ref))


def test_noalloc_rejects_sizes_beyond_the_scratch():
    from moe_linear_layers_b200 import q4
    T, H, I, E, topk = 4096, 2048, 1024, 64, 8
    assert q4.moe_q4_workspace_size(T, H, I, E, topk) > q4.Q4_MOE_NOALLOC_SCRATCH_BYTES
    FAKE = 0x10000   # never dereferenced: the size check comes first
    descs = (q4.q4_weight * 3)()
    rc = q4._lib.moe_q4_forward_noalloc(FAKE, T, H, FAKE, None, E, topk, descs, I, FAKE, q4.Q4_OUT_F32,
                                        None, None, None, None, None, None, None)
    assert rc == q4.Q4_ERR_WORKSPACE
