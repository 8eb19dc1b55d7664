"""Empty problems through the binding: a batch without rows (m = 0, T = 0 tokens, R = 0 rows) returns
empty outputs of the right shape, and the routing outputs it is asked for say that every expert's range
is empty (offsets and counts 0).  A zero-element CUDA tensor has no storage, so these calls reach the
library with NULL data pointers, which it accepts for arrays that hold no elements."""
import pytest
import torch

pytestmark = pytest.mark.gpu

H, I, E, TOPK, K, N = 256, 128, 4, 2, 256, 128


@pytest.fixture(scope="module")
def q4():
    from moe_linear_layers_b200 import q4 as mod
    return mod


def _weights(q4, n, k, seed, sym=False):
    g = torch.Generator().manual_seed(seed)
    return q4.q4_quantize_pack((0.02 * torch.randn((n, k), generator=g)).cuda(), 128, sym)


@pytest.fixture(scope="module")
def experts(q4):
    return (_weights(q4, E * I, H, 1), _weights(q4, E * I, H, 2), _weights(q4, E * H, I, 3))


@pytest.fixture(scope="module")
def router():
    g = torch.Generator().manual_seed(4)
    return (0.05 * torch.randn((E, H), generator=g)).cuda(), torch.zeros((E,), device="cuda")


def test_linear_and_act_quant_without_rows(q4):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    w, ws = _weights(q4, N, K, 5), _weights(q4, N, K, 6, sym=True)
    x = torch.empty((0, K), dtype=torch.bfloat16, device="cuda")
    for od in (torch.float32, torch.bfloat16):
        y = q4.q4_linear_w4a16(x, w, out_dtype=od, dev_status=st)
        assert y.shape == (0, N) and y.dtype == od
    xq, sa = q4.act_quant_per_token(x, dev_status=st)
    assert xq.shape == (0, K) and sa.shape == (0,)
    y8 = q4.q4_linear_w4a8(xq, sa, ws, dev_status=st)
    assert y8.shape == (0, N)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def test_moe_layer_without_tokens(q4, experts, router):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    Wr, bias = router
    x = torch.empty((0, H), dtype=torch.bfloat16, device="cuda")
    y, ids, wts, perm, offs, cnts = q4.moe_q4_forward(x, Wr, bias, TOPK, experts, I, want_routing=True, dev_status=st)
    torch.cuda.synchronize()
    assert y.shape == (0, H) and ids.shape == (0, TOPK) and perm.shape == (0,)
    assert offs.tolist() == [0] * (E + 1) and cnts.tolist() == [0] * E
    assert q4.moe_q4_forward_noalloc(x, Wr, bias, TOPK, experts, I, dev_status=st).shape == (0, H)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def test_moe_steps_without_tokens_or_rows(q4, experts, router):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    Wr, bias = router
    r = q4.moe_q4_route(torch.empty((0, H), dtype=torch.bfloat16, device="cuda"), Wr, bias, TOPK, dev_status=st)
    torch.cuda.synchronize()
    assert r["offsets"].tolist() == [0] * (E + 1) and r["x_perm"].shape == (0, H)
    o = q4.moe_q4_forward_rows(r["x_perm"], r["row_expert"], 0, experts, I, dev_status=st)
    assert o.shape == (0, H)
    y = q4.moe_q4_combine(o, r["pair_pos"], r["topk_w"], dev_status=st)
    torch.cuda.synchronize()
    assert y.shape == (0, H) and int(st.item()) == 0
