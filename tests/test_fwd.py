"""GPU parity of the fused forward (libfa.so via the C ABI) against the float64
oracle on identical seeded inputs.  Small shapes span several 128-row tiles
and a ragged tail; the full-size workloads are checked on sampled query rows
(every tile-boundary row plus 512 random ones), which is exact for those rows
because each output row depends only on its own query and all of K, V."""
import math

import numpy as np
import pytest
import torch

import exact_attention_112_b200 as fa
import oracle
from exact_attention_112_b200 import inputs
from gpu_util import check_forward, compare_fwd, gpu_forward, TOL_O

pytestmark = pytest.mark.gpu


def test_tiny_workload_full():
    w = inputs.workload("tiny")
    check_forward(w["B"], w["H"], w["Nq"], w["Nk"], w["D"], w["dtype"], w["causal"], seed=w["seed"])


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_shapes(D, dtype, causal):
    # 300 rows = one full 256-row unit + a unit whose second tile is empty
    check_forward(2, 3, 300, 300, D, dtype, causal, seed=11)


@pytest.mark.parametrize("Nq,Nk", [(1, 1), (7, 7), (129, 129), (255, 255), (128, 640),
                                   (200, 333), (333, 200), (5, 1000), (1000, 5)])
@pytest.mark.parametrize("causal", [False, True])
def test_edge_sizes(Nq, Nk, causal):
    check_forward(1, 2, Nq, Nk, 64, "bf16", causal, seed=Nq * 1000 + Nk)


@pytest.mark.parametrize("D", [64, 128])
def test_output_base_16_byte_aligned(D):
    """O whose base is 16- but not 32-byte aligned (a view 16 bytes into a
    larger buffer) takes the 16-byte store path; the result is bit-identical
    to the same call with a 32-byte aligned O, and matches the oracle."""
    B, H, N = 1, 3, 300
    inp = inputs.make_inputs(B, H, N, N, D, dtype="bf16", seed=77)
    dev = torch.device("cuda")
    q, k, v = (inp[x].to(dev) for x in "qkv")
    o_ref = torch.empty_like(q)
    lse_ref = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    fa.fa_fwd(q, k, v, o_ref, lse_ref, causal=True)
    buf = torch.empty(q.numel() + 8, dtype=q.dtype, device=dev)
    o = buf[8:].view(q.shape)
    assert o.data_ptr() % 32 == 16
    lse = torch.empty_like(lse_ref)
    fa.fa_fwd(q, k, v, o, lse, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    f = inputs.to_f64
    ref_o, ref_lse = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), None, True, 1.0 / math.sqrt(D))
    assert float(np.abs(o.float().cpu().numpy() - ref_o).max()) <= TOL_O["bf16"]
    assert float(np.abs(lse.cpu().numpy() - ref_lse).max()) <= 1e-3


def test_many_units_and_heads():
    check_forward(3, 5, 1024, 1024, 128, "bf16", True, seed=5)


@pytest.mark.parametrize("causal", [False, True])
def test_key_bias(causal):
    check_forward(2, 2, 384, 520, 64, "bf16", causal, seed=3, bias_frac=0.1)
    check_forward(2, 2, 256, 260, 128, "f16", causal, seed=4, bias_frac=0.3)


@pytest.mark.parametrize("causal", [False, True])
def test_key_bias_unaligned_rows(causal):
    # Nk % 4 != 0: the bias rows of batches b > 0 start off 16-byte boundaries,
    # and the last key tile is ragged
    check_forward(3, 2, 200, 301, 64, "bf16", causal, seed=21, bias_frac=0.2)
    check_forward(2, 2, 129, 333, 128, "f16", causal, seed=22, bias_frac=0.1)


def test_key_bias_many_units_per_cta():
    # more work units than SMs, batches interleaved: the bias staged for one
    # unit's last tile must not leak into the next unit's first tile
    check_forward(4, 16, 1024, 1024, 64, "bf16", False, seed=23, bias_frac=0.1)
    check_forward(3, 8, 768, 1000, 128, "bf16", True, seed=24, bias_frac=0.25)


def test_large_scores_rescale():
    # scores spanning hundreds of nats: exercises the lazy max rescale
    check_forward(2, 2, 512, 512, 64, "bf16", False, seed=6, qk_std=8.0, v_dist="uniform")
    check_forward(1, 2, 640, 640, 128, "bf16", True, seed=7, qk_std=6.0)


def test_no_keys():
    # Nk == 0: every row is empty -> O = 0, LSE = -inf
    inp = inputs.make_inputs(1, 2, 100, 0, 64, dtype="bf16", seed=1)
    o, lse = gpu_forward(inp, False)
    assert np.all(o == 0) and np.all(lse == -np.inf)


def test_causal_prefix_means_exact_indexing():
    """Q = 0 makes every visible score equal, so O_i is the mean of the visible
    V rows and LSE_i = ln(#visible): a causal off-by-one anywhere shows up at
    full strength for the short prefixes."""
    for (Nq, Nk) in [(300, 300), (130, 400), (400, 130)]:
        inp = inputs.make_inputs(1, 2, Nq, Nk, 64, dtype="bf16", seed=2)
        inp["q"] = torch.zeros_like(inp["q"])
        o, lse = gpu_forward(inp, True)
        v = inputs.to_f64(inp["v"])
        for i in range(Nq):
            n_vis = min(max(i + (Nk - Nq) + 1, 0), Nk)
            if n_vis == 0:
                assert lse[0, 0, i] == -np.inf and np.all(o[0, :, i] == 0)
                continue
            want = v[0, :, :n_vis].mean(axis=1)
            assert np.abs(o[0, :, i] - want).max() <= 1.5e-2, (Nq, Nk, i)
            assert abs(lse[0, 0, i] - math.log(n_vis)) <= 1e-3


def test_one_hot_dominant_key():
    """Q_i = c e_i, K_j = c e_j with c^2 * scale = 30 (in fp16-exact values):
    row i returns V_i."""
    N, D = 128, 128
    scale = 1.0 / math.sqrt(D)
    c = math.sqrt(30.0 / scale)
    q = torch.zeros((1, 1, N, D))
    for i in range(N):
        q[0, 0, i, i] = c
    inp = {"q": q.to(torch.float16), "k": q.to(torch.float16),
           "v": (torch.rand((1, 1, N, D), generator=torch.Generator().manual_seed(9)) * 2 - 1).to(torch.float16),
           "key_bias": None}
    o, lse = gpu_forward(inp, False)
    assert np.abs(o[0, 0] - inputs.to_f64(inp["v"])[0, 0]).max() <= 1e-2


# ---------------- full-size workloads (sampled rows) ----------------

def _full(name, **over):
    w = inputs.workload(name, **over)
    rows = inputs.sample_rows(w["Nq"], seed=w["seed"])
    return check_forward(w["B"], w["H"], w["Nq"], w["Nk"], w["D"], w["dtype"], w["causal"],
                         seed=w["seed"], qk_std=w["qk_std"], v_dist=w["v_dist"],
                         bias_frac=w["bias_frac"], rows=rows)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_llama_layer_full_size(dtype):
    _full("llama", dtype=dtype)


def test_stress_full_size():
    _full("stress")


@pytest.mark.parametrize("N", [512, 1024, 2048, 4096, 8192, 16384, 32768])
@pytest.mark.parametrize("causal", [False, True])
def test_sweep_full_size(N, causal):
    # every sequence length of the sweep, B = max(1, 16384 // N), causal and not
    _full("sweep", N=N, causal=causal)


def test_timeout_self_test_leaves_context_usable():
    """A wait that nothing completes gives up after its limit, latches
    FA_ERR_DEVICE_TIMEOUT, and the next call works normally."""
    assert fa.fa_debug_wait_timeout(20000) == fa.FA_OK   # 20 ms
    assert fa.fa_device_status() == fa.FA_ERR_DEVICE_TIMEOUT
    assert fa.fa_device_status() == fa.FA_OK             # cleared
    check_forward(1, 1, 256, 256, 64, "f16", False, seed=1)
