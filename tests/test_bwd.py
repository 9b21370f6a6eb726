"""GPU parity of the backward (row-term pre-pass, dK/dV recompute kernel and
the separate dQ recompute kernel; no atomics) against the float64 oracle's
gradients, which are themselves pinned by finite differences and by torch
autograd (tests/test_oracle.py).
Tolerance: max|g - g_ref| / max|g_ref| <= 5e-2 for dQ, dK and dV."""
import numpy as np
import pytest
import torch

import exact_attention_112_b200 as fa
from exact_attention_112_b200 import inputs
from gpu_util import check_backward, gpu_backward

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
def test_small(D, dtype, causal):
    check_backward(1, 2, 256, 256, D, dtype, causal, seed=21)


@pytest.mark.parametrize("Nq,Nk", [(1, 1), (7, 7), (129, 129), (300, 300), (128, 640),
                                   (200, 333), (333, 200), (5, 700)])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged(Nq, Nk, causal):
    check_backward(1, 2, Nq, Nk, 64, "bf16", causal, seed=Nq + 7 * Nk)


def test_key_bias():
    check_backward(2, 2, 384, 520, 64, "bf16", False, seed=3, bias_frac=0.1)
    check_backward(1, 2, 256, 300, 128, "bf16", True, seed=4, bias_frac=0.2)


def test_large_scores():
    check_backward(1, 2, 512, 512, 64, "bf16", False, seed=6, qk_std=4.0, v_dist="uniform")


def test_many_tiles():
    check_backward(2, 3, 1024, 1024, 128, "bf16", True, seed=8)


def test_head_groups_full_and_partial():
    # 9 heads: one full group of 8 work units per tile rank and a partial
    # group of 1, in both recompute kernels
    check_backward(3, 3, 384, 384, 64, "bf16", True, seed=9)
    check_backward(1, 9, 200, 330, 128, "f16", False, seed=10)


def test_no_keys_and_no_queries():
    dev = torch.device("cuda")
    # Nk == 0: every output row empty, dQ = 0
    inp = inputs.make_inputs(1, 2, 100, 0, 64, dtype="bf16", seed=1, with_dO=True)
    dq, dk, dv = gpu_backward(inp, False)
    assert np.all(dq == 0) and dk.size == 0 and dv.size == 0
    # Nq == 0: no query sees any key, dK = dV = 0
    q = torch.empty((1, 2, 0, 64), dtype=torch.bfloat16, device=dev)
    k = torch.randn((1, 2, 50, 64), dtype=torch.bfloat16, device=dev)
    v = torch.randn_like(k)
    o = torch.empty_like(q)
    lse = torch.empty((1, 2, 0), dtype=torch.float32, device=dev)
    dq = torch.empty_like(q)
    dk = torch.full_like(k, 7.0)
    dv = torch.full_like(v, 7.0)
    ws = torch.empty((16,), dtype=torch.uint8, device=dev)
    fa.fa_bwd(q, k, v, o, lse, q, dq, dk, dv, ws, causal=True)
    torch.cuda.synchronize()
    assert torch.all(dk == 0) and torch.all(dv == 0)


def test_workspace_too_small():
    dev = torch.device("cuda")
    q = torch.randn((1, 1, 128, 64), dtype=torch.bfloat16, device=dev)
    o, lse = fa.attention_forward(q, q, q)
    ws = torch.empty((fa.fa_bwd_workspace_bytes(1, 1, 128, 128, 64) - 256,), dtype=torch.uint8, device=dev)
    with pytest.raises(fa.FaError) as e:
        fa.fa_bwd(q, q, q, o, lse, q, torch.empty_like(q), torch.empty_like(q),
                  torch.empty_like(q), ws)
    assert e.value.status == fa.FA_ERR_WORKSPACE


def test_bwd_workload_full_size():
    """B=2 H=32 N=4096 D=128 bf16 causal: full gradients on 4 seeded (b, h)
    pairs (dK/dV need every query row, so whole heads are compared)."""
    w = inputs.workload("bwd")
    rng = np.random.default_rng(w["seed"])
    bh = sorted(rng.choice(w["B"] * w["H"], size=4, replace=False).tolist())
    check_backward(w["B"], w["H"], w["Nq"], w["Nk"], w["D"], w["dtype"], w["causal"],
                   seed=w["seed"], bh_list=bh)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_is_bitwise_reproducible(causal):
    """No atomics anywhere in the backward: two runs on the same inputs give
    identical bits, including with a workspace left dirty by another problem."""
    dev = torch.device("cuda")
    inp = inputs.make_inputs(2, 3, 700, 650, 128, dtype="bf16", seed=77, with_dO=True)
    q, k, v, do = (inp[x].to(dev) for x in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=causal)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(2, 3, 700, 650, 128), dtype=torch.uint8, device=dev)
    runs = []
    for r in range(3):
        ws.fill_(r * 85)
        g = [torch.full_like(t, float("nan")) for t in (q, k, v)]
        fa.fa_bwd(q, k, v, o, lse, do, *g, ws, causal=causal)
        torch.cuda.synchronize()
        runs.append(g)
    assert fa.fa_device_status() == fa.FA_OK
    for r in (1, 2):
        for a, b in zip(runs[0], runs[r]):
            assert torch.equal(a, b)
