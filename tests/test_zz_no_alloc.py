"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory
(services with a fixed memory budget, plugin hosts that only pass buffers,
latency-critical paths).  Its scratch is a fixed array inside libfa.so; this
test calls it through the C ABI twice in a row and checks both results against
fa_bwd with a caller workspace, within the backward's parity tolerance.

The file name sorts last so that a run stopping at the first failure has
already run every other test."""
import ctypes
import math

import numpy as np
import pytest
import torch

import exact_attention_112_b200 as fa
from exact_attention_112_b200 import inputs
from gpu_util import TOL_GRAD_REL

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _run_case(B, H, Nq, Nk, D, dtype, causal, bias_frac, seed):
    dev = torch.device("cuda")
    inp = inputs.make_inputs(B, H, Nq, Nk, D, dtype=dtype, seed=seed, bias_frac=bias_frac,
                             with_dO=True)
    q, k, v, do = (inp[x].to(dev) for x in ("q", "k", "v", "do"))
    bias = None if inp["key_bias"] is None else inp["key_bias"].to(dev)
    scale = 1.0 / math.sqrt(D)
    o, lse = fa.attention_forward(q, k, v, causal=causal, key_bias=bias)
    ref = fa.attention_backward(q, k, v, o, lse, do, causal=causal, key_bias=bias)
    torch.cuda.synchronize()
    ref = [t.float() for t in ref]
    L = fa.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = fa.FA_BF16 if dtype == "bf16" else fa.FA_F16
    for call in range(2):
        dq = torch.full_like(q, float("nan"))
        dk = torch.full_like(k, float("nan"))
        dv = torch.full_like(v, float("nan"))
        st = L.fa_bwd_noalloc(_p(q), _p(k), _p(v), _p(o), _p(lse), _p(do), _p(dq), _p(dk), _p(dv),
                              B, H, Nq, Nk, D, int(causal), ctypes.c_float(scale), code, _p(bias),
                              stream)
        assert st == fa.FA_OK, fa.fa_status_string(st)
        torch.cuda.synchronize()
        assert fa.fa_device_status() == fa.FA_OK
        for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            g = g.float()
            assert not torch.isnan(g).any(), f"call {call}: NaN in {name}"
            denom = float(r.abs().max())
            err = float((g - r).abs().max()) / denom
            assert err <= TOL_GRAD_REL, f"call {call}: {name} rel-to-max {err}"


def test_noalloc_matches_workspace_backward_causal():
    _run_case(2, 3, 300, 300, 128, "bf16", True, 0.0, seed=41)


def test_noalloc_matches_workspace_backward_bias():
    _run_case(1, 2, 384, 520, 64, "f16", False, 0.1, seed=42)


def test_noalloc_rejects_rows_beyond_its_scratch():
    L = fa.lib()
    B, H, Nq = 1, 16, fa.FA_BWD_NOALLOC_MAX_ROWS // 16 + 1
    one = ctypes.c_void_p(256)
    st = L.fa_bwd_noalloc(one, one, one, one, one, one, one, one, one, B, H, Nq, 128, 64, 0,
                          ctypes.c_float(0.125), fa.FA_BF16, None, None)
    assert st == fa.FA_ERR_WORKSPACE
