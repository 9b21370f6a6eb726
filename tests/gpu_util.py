"""Shared helpers of the GPU parity tests (CUDA path vs the float64 oracle)."""
import math

import numpy as np
import torch

import exact_attention_112_b200 as fa
import oracle
from exact_attention_112_b200 import inputs

# tolerances of the method's acceptance bar
TOL_O = {"f16": 1e-2, "bf16": 2e-2}
TOL_LSE = 1e-3
TOL_GRAD_REL = 5e-2


def gpu_forward(inp, causal, scale=None, canary=True):
    dev = torch.device("cuda")
    q, k, v = (inp[x].to(dev) for x in ("q", "k", "v"))
    bias = None if inp.get("key_bias") is None else inp["key_bias"].to(dev)
    B, H, Nq, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    if canary:
        o.fill_(float("nan"))
        lse.fill_(float("nan"))
    fa.fa_fwd(q, k, v, o, lse, causal=causal, scale=scale, key_bias=bias)
    torch.cuda.synchronize()
    st = fa.fa_device_status()
    assert st == fa.FA_OK, fa.fa_status_string(st)
    return o.float().cpu().numpy(), lse.cpu().numpy()


def compare_fwd(o, lse, ref_o, ref_lse, dtype):
    """Element-wise comparison; returns (max|dO|, max|dLSE|)."""
    assert not np.isnan(o).any(), "NaN in O (unwritten or invalid output)"
    assert not np.isnan(lse).any(), "NaN in LSE"
    assert np.isfinite(o).all()
    fin = np.isfinite(ref_lse)
    # -inf LSE exactly where the oracle has no visible key
    assert np.array_equal(np.isfinite(lse), fin), "empty-row pattern differs"
    assert np.all(o[~fin] == 0.0), "empty rows must give O = 0"
    err_o = float(np.abs(o - ref_o).max()) if o.size else 0.0
    err_l = float(np.abs(lse[fin] - ref_lse[fin]).max()) if fin.any() else 0.0
    assert err_o <= TOL_O[dtype], f"O max-abs error {err_o} > {TOL_O[dtype]}"
    assert err_l <= TOL_LSE, f"LSE max-abs error {err_l} > {TOL_LSE}"
    return err_o, err_l


def check_forward(B, H, Nq, Nk, D, dtype, causal, seed=0, qk_std=1.0, v_dist="normal",
                  bias_frac=0.0, rows=None, scale=None):
    inp = inputs.make_inputs(B, H, Nq, Nk, D, dtype=dtype, seed=seed, qk_std=qk_std,
                             v_dist=v_dist, bias_frac=bias_frac)
    o, lse = gpu_forward(inp, causal, scale)
    f = inputs.to_f64
    ref_o, ref_lse = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["key_bias"]),
                                causal, scale if scale else 1.0 / math.sqrt(D), rows=rows)
    if rows is not None:
        o, lse = o[:, :, rows], lse[:, :, rows]
    return compare_fwd(o, lse, ref_o, ref_lse, dtype)


def gpu_backward(inp, causal, scale=None):
    """Forward then backward on the GPU; returns float arrays dq, dk, dv and
    the forward outputs."""
    dev = torch.device("cuda")
    q, k, v, do = (inp[x].to(dev) for x in ("q", "k", "v", "do"))
    bias = None if inp.get("key_bias") is None else inp["key_bias"].to(dev)
    o, lse = fa.attention_forward(q, k, v, causal=causal, scale=scale, key_bias=bias)
    dq = torch.full_like(q, float("nan"))
    dk = torch.full_like(k, float("nan"))
    dv = torch.full_like(v, float("nan"))
    B, H, Nq, D = q.shape
    ws = torch.full((fa.fa_bwd_workspace_bytes(B, H, Nq, k.shape[2], D),), 0xFF,
                    dtype=torch.uint8, device=dev)       # garbage workspace on entry
    fa.fa_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, causal=causal, scale=scale, key_bias=bias)
    torch.cuda.synchronize()
    st = fa.fa_device_status()
    assert st == fa.FA_OK, fa.fa_status_string(st)
    return [t.float().cpu().numpy() for t in (dq, dk, dv)]


def compare_grads(got, ref, tol=TOL_GRAD_REL):
    """max|g - g_ref| / max|g_ref| per gradient; returns the three ratios."""
    out = []
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g = g.reshape(r.shape)
        assert not np.isnan(g).any(), f"NaN in {name}"
        denom = float(np.abs(r).max())
        err = float(np.abs(g - r).max()) / denom if denom > 0 else float(np.abs(g).max())
        assert err <= tol, f"{name}: rel-to-max error {err} > {tol}"
        out.append(err)
    return out


def check_backward(B, H, Nq, Nk, D, dtype, causal, seed=0, qk_std=1.0, v_dist="normal",
                   bias_frac=0.0, bh_list=None, scale=None):
    inp = inputs.make_inputs(B, H, Nq, Nk, D, dtype=dtype, seed=seed, qk_std=qk_std,
                             v_dist=v_dist, bias_frac=bias_frac, with_dO=True)
    got = gpu_backward(inp, causal, scale)
    f = inputs.to_f64
    ref = oracle.bwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["do"]), f(inp["key_bias"]),
                     causal, scale if scale else 1.0 / math.sqrt(D), bh_list=bh_list)
    if bh_list is None:
        bh_list = list(range(B * H))
    sel = [g.reshape(B * H, *g.shape[2:])[bh_list] for g in got]
    return compare_grads(sel, ref)
