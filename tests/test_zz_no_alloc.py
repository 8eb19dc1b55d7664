"""moe_q4_forward_noalloc: the MoE entry point for callers that cannot allocate device memory (for
example a plugin whose host application owns all device memory, or a latency-critical loop that must
not call cudaMalloc).  It uses the library's fixed device scratch array instead of a caller workspace.

Checked through the C ABI against the existing entry point (moe_q4_forward with a caller workspace),
within the tolerance the other parity tests use, on two calls in a row (the second call reuses the
scratch the first one left behind).  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from moe_linear_layers_b200 import synth
from tests._util import assert_close, cuda_u16_as, upload_weight

pytestmark = pytest.mark.gpu


def _setup(q4, T, H, I, E, topk, group, sym):
    x = synth.activations(("noalloc", "x", T), T, H)
    Wr, bias = synth.router(("noalloc", "router"), E, H)
    Ws = [synth.weights(("noalloc", nm), n, k) for nm, n, k in (("g", E * I, H), ("u", E * I, H), ("d", E * H, I))]
    qs = [oracle.quantize(W, group, sym) for W in Ws]
    ex = (upload_weight(q4, *qs[0], E * I, H, group, sym), upload_weight(q4, *qs[1], E * I, H, group, sym),
          upload_weight(q4, *qs[2], E * H, I, group, sym))
    return cuda_u16_as(x, torch.bfloat16), torch.from_numpy(Wr).cuda(), torch.from_numpy(bias).cuda(), ex


@pytest.mark.parametrize("T,H,I,E,topk,group,sym", [(64, 256, 128, 8, 2, 128, False), (200, 2048, 1024, 64, 8, 128, False)])
def test_noalloc_matches_workspace_entry_point(T, H, I, E, topk, group, sym):
    from moe_linear_layers_b200 import q4
    x, Wr, bias, ex = _setup(q4, T, H, I, E, topk, group, sym)
    assert q4.moe_q4_workspace_size(T, H, I, E, topk) <= q4.Q4_MOE_NOALLOC_SCRATCH_BYTES
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = q4.moe_q4_forward(x, Wr, bias, topk, ex, I, dev_status=st).cpu().numpy()
    descs = (q4.q4_weight * 3)(*[e.desc for e in ex])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        y = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
        rc = q4._lib.moe_q4_forward_noalloc(x.data_ptr(), T, H, Wr.data_ptr(), bias.data_ptr(), E, topk, descs, I,
                                            y.data_ptr(), q4.Q4_OUT_F32, None, None, None, None, None,
                                            st.data_ptr(), stream)
        assert rc == q4.Q4_OK, q4.status_string(rc)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert_close(y.cpu().numpy(), ref, what=f"noalloc call {call}")


def test_noalloc_rejects_sizes_beyond_the_scratch():
    from moe_linear_layers_b200 import q4
    T, H, I, E, topk = 4096, 2048, 1024, 64, 8
    assert q4.moe_q4_workspace_size(T, H, I, E, topk) > q4.Q4_MOE_NOALLOC_SCRATCH_BYTES
    FAKE = 0x10000   # never dereferenced: the size check comes first
    descs = (q4.q4_weight * 3)()
    rc = q4._lib.moe_q4_forward_noalloc(FAKE, T, H, FAKE, None, E, topk, descs, I, FAKE, q4.Q4_OUT_F32,
                                        None, None, None, None, None, None, None)
    assert rc == q4.Q4_ERR_WORKSPACE
