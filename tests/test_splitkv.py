"""Split-KV forward (fa_fwd_splitkv) against the float64 oracle: the keys are
processed in contiguous ranges whose partial (O_s, LSE_s) are merged with the
associative log-sum-exp merge; the merged result must equal plain attention
(the merge itself is pinned on the CPU in tests/test_oracle.py)."""
import math

import numpy as np
import pytest
import torch

import exact_attention_112_b200 as fa
import oracle
from exact_attention_112_b200 import inputs
from gpu_util import compare_fwd

pytestmark = pytest.mark.gpu


def split_forward(inp, causal, num_splits):
    dev = torch.device("cuda")
    q, k, v = (inp[x].to(dev) for x in ("q", "k", "v"))
    bias = None if inp.get("key_bias") is None else inp["key_bias"].to(dev)
    B, H, Nq, D = q.shape
    Nk = k.shape[2]
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device=dev)
    ws = torch.full((fa.fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, D, num_splits),), 0xFF,
                    dtype=torch.uint8, device=dev)
    fa.fa_fwd_splitkv(q, k, v, o, lse, num_splits, ws, causal=causal, key_bias=bias)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    return o.float().cpu().numpy(), lse.cpu().numpy()


def check(B, H, Nq, Nk, D, dtype, causal, splits, seed, bias_frac=0.0):
    inp = inputs.make_inputs(B, H, Nq, Nk, D, dtype=dtype, seed=seed, bias_frac=bias_frac)
    o, lse = split_forward(inp, causal, splits)
    f = inputs.to_f64
    ref_o, ref_lse = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["key_bias"]), causal,
                                1.0 / math.sqrt(D))
    return compare_fwd(o, lse, ref_o, ref_lse, dtype)


@pytest.mark.parametrize("Nq", [1, 4, 17])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("D", [64, 128])
def test_decode_shapes(Nq, causal, D):
    check(2, 4, Nq, 3000, D, "bf16", causal, splits=6, seed=Nq + D)


@pytest.mark.parametrize("splits", [2, 3, 8, 40])
def test_split_counts(splits):
    # 40 splits of a 1000-key problem: most ranges are empty or one tile
    check(1, 3, 9, 1000, 128, "f16", False, splits, seed=splits)


def test_key_bias_and_long_queries():
    check(2, 2, 300, 2000, 64, "bf16", False, 5, seed=3, bias_frac=0.1)


def test_key_bias_unaligned_rows():
    # Nk % 4 != 0: bias rows of batches b > 0 start off 16-byte boundaries
    check(3, 2, 17, 1501, 128, "bf16", True, 4, seed=5, bias_frac=0.2)
    check(1, 2, 520, 1400, 128, "bf16", True, 4, seed=4)


def test_matches_single_pass_forward():
    inp = inputs.make_inputs(1, 4, 64, 8192, 128, dtype="bf16", seed=9)
    o1, l1 = split_forward(inp, True, 16)
    dev = torch.device("cuda")
    q, k, v = (inp[x].to(dev) for x in ("q", "k", "v"))
    o2, l2 = fa.attention_forward(q, k, v, causal=True)
    assert np.abs(o1 - o2.float().cpu().numpy()).max() <= 2e-2
    assert np.abs(l1 - l2.cpu().numpy()).max() <= 1e-3


def test_argument_errors():
    dev = torch.device("cuda")
    q = torch.randn((1, 1, 4, 64), dtype=torch.bfloat16, device=dev)
    k = torch.randn((1, 1, 512, 64), dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, 4), dtype=torch.float32, device=dev)
    need = fa.fa_fwd_splitkv_workspace_bytes(1, 1, 4, 512, 64, 4)
    small = torch.empty((need - 512,), dtype=torch.uint8, device=dev)
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd_splitkv(q, k, k, o, lse, 4, small)
    assert e.value.status == fa.FA_ERR_WORKSPACE
    ws = torch.empty((need,), dtype=torch.uint8, device=dev)
    for bad in (0, 257):
        with pytest.raises(fa.FaError) as e:
            fa.fa_fwd_splitkv(q, k, k, o, lse, bad, ws)
        assert e.value.status == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("causal", [False, True])
def test_library_split_count(causal):
    # the count fa_splitkv_num_splits picks for a decoding shape on this GPU
    # (one query block of 8 heads over 16384 keys: more splits than SMs/units)
    B, H, Nq, Nk, D = 1, 8, 64, 16384, 128
    s = fa.fa_splitkv_num_splits(B, H, Nq, Nk)
    assert 1 < s <= 256
    check(B, H, Nq, Nk, D, "bf16", causal, s, seed=77)
