"""GPU parity of the FP8 (E4M3) forward (fa_fwd_fp8, the low-precision path the
lastdictionary.com "FlashAttention" entry credits to FlashAttention-3) against
the float64 oracle.

Reading: the oracle receives the dequantised inputs q_descale*Q, k_descale*K,
v_descale*V (the E4M3 values exactly, upcast), so input quantisation is not an
error; the error is the kernel's own rounding of P to E4M3 before P.V.

Tolerance, derived from that rounding.  E4M3 keeps 3 mantissa bits, so round
to nearest even moves a value in the normal range (>= 2^-6) by at most 2^-4 of
itself and a subnormal by at most 2^-10.  With l the fp32 sum of the
unrounded p_j, the output error of row i, column d is then at most
    2^-4 * sum_j p_j |v_jd| / l  =  2^-4 * A_id,
where A = softmax(S) |V| is the oracle's attention output with |V| in place
of V, plus the subnormal part (2^-10 per key, relative to l >= 1, random in
sign), the bf16 rounding of O (2^-9 |O|) and fp32 accumulation.  The test
bound is |O - O_ref| <= 2^-4 A + 2^-8 |O_ref| + 2e-3; the mean error must also
stay below 2^-6 of mean(A) (rounding to nearest even has no bias; a wrong
scale or packing would).  LSE is computed from the exact E4M3 products in
fp32: max-abs <= 1e-3 as for the 16-bit forward."""
import math

import numpy as np
import pytest
import torch

import exact_attention_112_b200 as fa
import oracle
from exact_attention_112_b200 import inputs

pytestmark = pytest.mark.gpu


def run_fp8(B, H, Nq, Nk, causal, seed, descales=(1.0, 1.0, 1.0), bias_frac=0.0, rows=None):
    D = 128
    inp = inputs.make_inputs(B, H, Nq, Nk, D, dtype="e4m3", seed=seed, bias_frac=bias_frac)
    dev = torch.device("cuda")
    q, k, v = (inp[x].to(dev) for x in ("q", "k", "v"))
    bias = None if inp["key_bias"] is None else inp["key_bias"].to(dev)
    o = torch.full((B, H, Nq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device=dev)
    qd, kd, vd = descales
    fa.fa_fwd_fp8(q, k, v, o, lse, causal=causal, q_descale=qd, k_descale=kd, v_descale=vd,
                  key_bias=bias)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    f = inputs.to_f64
    qf, kf, vf = f(inp["q"]) * qd, f(inp["k"]) * kd, f(inp["v"]) * vd
    scale = 1.0 / math.sqrt(D)
    ref_o, ref_lse = oracle.fwd(qf, kf, vf, f(inp["key_bias"]), causal, scale, rows=rows)
    ref_a, _ = oracle.fwd(qf, kf, np.abs(vf), f(inp["key_bias"]), causal, scale, rows=rows)
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    if rows is not None:
        o, lse = o[:, :, rows], lse[:, :, rows]
    assert not np.isnan(o).any() and not np.isnan(lse).any()
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.all(o[~fin] == 0.0)
    err = np.abs(o - ref_o)
    bound = ref_a / 16.0 + np.abs(ref_o) / 256.0 + 2e-3
    worst = float((err - bound).max()) if err.size else 0.0
    assert worst <= 0.0, f"O error exceeds the E4M3 rounding bound by {worst}"
    if err.size:
        assert err.mean() <= ref_a.mean() / 64.0, (err.mean(), ref_a.mean())
    if fin.any():
        err_l = float(np.abs(lse[fin] - ref_lse[fin]).max())
        assert err_l <= 1e-3, err_l
    return float(err.max()) if err.size else 0.0


@pytest.mark.parametrize("causal", [False, True])
def test_small_and_ragged(causal):
    run_fp8(1, 2, 300, 300, causal, seed=1)
    run_fp8(2, 3, 129, 517, causal, seed=2)
    run_fp8(1, 2, 517, 129, causal, seed=3)


def test_descales_and_bias():
    run_fp8(2, 2, 384, 640, False, seed=4, descales=(0.5, 2.0, 0.25), bias_frac=0.1)
    run_fp8(1, 3, 256, 256, True, seed=5, descales=(1.5, 0.75, 3.0))


def test_edge_sizes():
    for Nq, Nk in [(1, 1), (7, 7), (5, 1000), (1000, 5), (128, 0)]:
        run_fp8(1, 2, Nq, Nk, True, seed=Nq + Nk)


def test_llama_shape_sampled_rows():
    """B=1 H=32 N=8192 causal: every tile-boundary row plus 512 seeded rows."""
    w = inputs.workload("llama")
    rows = inputs.sample_rows(w["Nq"], seed=w["seed"])
    run_fp8(w["B"], w["H"], w["Nq"], w["Nk"], True, seed=w["seed"], rows=rows)


def test_rejects_other_head_dims_and_descales():
    dev = torch.device("cuda")
    q = torch.zeros((1, 1, 16, 64), dtype=torch.float8_e4m3fn, device=dev)
    o = torch.empty((1, 1, 16, 64), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((1, 1, 16), dtype=torch.float32, device=dev)
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd_fp8(q, q, q, o, lse)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    q = torch.zeros((1, 1, 16, 128), dtype=torch.float8_e4m3fn, device=dev)
    o = torch.empty((1, 1, 16, 128), dtype=torch.bfloat16, device=dev)
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        with pytest.raises(fa.FaError) as e:
            fa.fa_fwd_fp8(q, q, q, o, lse, k_descale=bad)
        assert e.value.status == fa.FA_ERR_INVALID_ARG
