"""GPU parity of the packed variable-length path (fa_fwd_varlen, fa_bwd_varlen):
sequences of different lengths stored one after another along the row axis,
each an independent exact-attention problem.  The reference is the float64
oracle applied to every sequence on its own (unpacked from the same seeded
values); rows that belong to no sequence must keep their canary values.
Tolerances as for the fixed-layout forward and backward."""
import math

import numpy as np
import pytest
import torch

import exact_attention_112_b200 as fa
import oracle
from exact_attention_112_b200 import inputs
from gpu_util import TOL_GRAD_REL, TOL_LSE, TOL_O

pytestmark = pytest.mark.gpu


def _packed(lens_q, lens_k, H, D, dtype, seed, spare_q=0, spare_k=0):
    """Seeded packed tensors [H, total, D] (+ `spare` trailing rows that belong
    to no sequence) and the int32 sequence tables."""
    tq, tk = sum(lens_q) + spare_q, sum(lens_k) + spare_k
    inp = inputs.make_inputs(1, H, tq, tk, D, dtype=dtype, seed=seed, with_dO=True)
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    return inp, cu_q, cu_k, tq, tk


def _run(lens_q, lens_k, H, D, dtype, causal, seed, backward=True, spare=(0, 0)):
    inp, cu_q, cu_k, tq, tk = _packed(lens_q, lens_k, H, D, dtype, seed, *spare)
    dev = torch.device("cuda")
    q, k, v, do = (inp[x][0].to(dev) for x in ("q", "k", "v", "do"))     # [H, total, D]
    cq, ck = torch.from_numpy(cu_q).to(dev), torch.from_numpy(cu_k).to(dev)
    mq, mk = max(lens_q), max(lens_k)
    o = torch.full_like(q, float("nan"))
    lse = torch.full((H, tq), float("nan"), dtype=torch.float32, device=dev)
    fa.fa_fwd_varlen(q, k, v, o, lse, cq, ck, mq, mk, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    go, gl = o.float().cpu().numpy(), lse.cpu().numpy()
    if backward:
        dq = torch.full_like(q, float("nan"))
        dk = torch.full_like(k, float("nan"))
        dv = torch.full_like(v, float("nan"))
        ws = torch.full((fa.fa_bwd_workspace_bytes(1, H, tq, tk, D),), 0xFF, dtype=torch.uint8, device=dev)
        fa.fa_bwd_varlen(q, k, v, o, lse, do, dq, dk, dv, ws, cq, ck, mq, mk, causal=causal)
        torch.cuda.synchronize()
        assert fa.fa_device_status() == fa.FA_OK
        gdq, gdk, gdv = (t.float().cpu().numpy() for t in (dq, dk, dv))
    f = inputs.to_f64
    scale = 1.0 / math.sqrt(D)
    for b in range(len(lens_q)):
        sq = slice(cu_q[b], cu_q[b + 1])
        sk = slice(cu_k[b], cu_k[b + 1])
        qb = f(inp["q"])[:, :, sq]
        kb, vb = f(inp["k"])[:, :, sk], f(inp["v"])[:, :, sk]
        if lens_q[b] == 0:
            continue
        ref_o, ref_l = oracle.fwd(qb, kb, vb, None, causal, scale)
        o_b, l_b = go[:, sq][None], gl[:, sq][None]
        fin = np.isfinite(ref_l)
        assert np.array_equal(np.isfinite(l_b), fin), f"sequence {b}: empty-row pattern"
        assert np.all(o_b[~fin] == 0.0)
        assert float(np.abs(o_b - ref_o).max()) <= TOL_O[dtype], f"sequence {b}: O"
        if fin.any():
            assert float(np.abs(l_b[fin] - ref_l[fin]).max()) <= TOL_LSE, f"sequence {b}: LSE"
        if backward:
            rq, rk, rv = oracle.bwd(qb, kb, vb, f(inp["do"])[:, :, sq], None, causal, scale)
            # the oracle's gradients are [B*H, N, D] with B = 1: one slice per head
            for name, g, r in (("dq", gdq[:, sq], rq), ("dk", gdk[:, sk], rk), ("dv", gdv[:, sk], rv)):
                assert g.shape == r.shape, (name, g.shape, r.shape)
                assert not np.isnan(g).any(), f"sequence {b}: NaN in {name}"
                denom = float(np.abs(r).max()) if r.size else 0.0
                err = float(np.abs(g - r).max()) / denom if denom > 0 else float(np.abs(g).max() if g.size else 0.0)
                assert err <= TOL_GRAD_REL, f"sequence {b}: {name} rel-to-max {err}"
    if backward:
        for b in range(len(lens_q)):
            if lens_q[b] == 0 and lens_k[b] > 0:   # keys nobody queries: zero gradients
                sk = slice(cu_k[b], cu_k[b + 1])
                assert np.all(gdk[:, sk] == 0) and np.all(gdv[:, sk] == 0)
    # rows that belong to no sequence are not written
    if spare[0]:
        assert np.isnan(go[:, tq - spare[0]:]).all() and np.isnan(gl[:, tq - spare[0]:]).all()
        if backward:
            assert np.isnan(gdq[:, tq - spare[0]:]).all()
    if spare[1] and backward:
        assert np.isnan(gdk[:, tk - spare[1]:]).all() and np.isnan(gdv[:, tk - spare[1]:]).all()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("D,dtype", [(64, "bf16"), (128, "f16"), (128, "bf16")])
def test_self_attention_mixed_lengths(causal, D, dtype):
    lens = [300, 1, 17, 513, 128, 256, 0, 77]
    _run(lens, lens, 2, D, dtype, causal, seed=31)


@pytest.mark.parametrize("causal", [False, True])
def test_different_query_and_key_lengths(causal):
    # per sequence Nq != Nk in both directions (bottom-right causal alignment)
    _run([5, 200, 333, 1, 129], [700, 130, 200, 9, 0], 3, 64, "bf16", causal, seed=32)


def test_rows_outside_every_sequence_are_untouched():
    _run([100, 250], [100, 250], 2, 128, "bf16", True, seed=33, spare=(37, 21))


def test_many_short_sequences_and_one_long():
    lens = [3] * 40 + [2048]
    _run(lens, lens, 2, 128, "bf16", True, seed=34)


def test_forward_only_long_sequences():
    lens = [4096, 1000, 3000]
    _run(lens, lens, 4, 128, "bf16", True, seed=35, backward=False)
