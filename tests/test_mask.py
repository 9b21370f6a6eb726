"""GPU parity of the general additive mask path (fa_fwd_mask, fa_bwd_mask:
the "+ mask" of the SDPA formula on the FlashAttention case-study slides,
"Attention is where tokens meet", in full) against the float64 oracle's
general-mask forward and backward, which are pinned on the CPU by torch SDPA
and autograd in float64, the per-row shift identity and the visible-mean
closed form (tests/test_oracle.py).

Masks: seeded random finite/-inf values, a sliding window, packed documents
(block-diagonal causal) and masks with whole rows hidden; broadcast over
batches and/or heads or one plane per (b, h); rows padded to a wider stride;
combined with the causal flag.  Tolerances as for the plain forward and
backward."""
import math

import numpy as np
import pytest
import torch

import exact_attention_112_b200 as fa
import oracle
from exact_attention_112_b200 import inputs
from gpu_util import TOL_GRAD_REL, compare_fwd, compare_grads

pytestmark = pytest.mark.gpu


def _case(B, H, Nq, Nk, D, dtype, causal, kind, planes, seed, ldm=None, backward=True, rows=None,
          use_flags=False):
    inp = inputs.make_inputs(B, H, Nq, Nk, D, dtype=dtype, seed=seed, with_dO=backward)
    Bm = B if planes[0] else 1
    Hm = H if planes[1] else 1
    mask = inputs.make_mask(kind, Nq, Nk, seed + 1, planes=(Bm, Hm), ldm=ldm)
    dev = torch.device("cuda")
    q, k, v = (inp[x].to(dev) for x in ("q", "k", "v"))
    mbuf = mask._base if mask._base is not None else mask
    mdev = mbuf.to(dev)[..., :Nk]
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device=dev)
    flags = fa.mask_tile_flags(mdev) if use_flags else None
    fa.fa_fwd_mask(q, k, v, o, lse, mdev, causal=causal, tile_flags=flags)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    f = inputs.to_f64
    scale = 1.0 / math.sqrt(D)
    m64 = mask.contiguous().double().numpy()
    ref_o, ref_lse = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), None, causal, scale,
                                rows=rows, mask=m64)
    go, gl = o.float().cpu().numpy(), lse.cpu().numpy()
    if rows is not None:
        go, gl = go[:, :, rows], gl[:, :, rows]
    compare_fwd(go, gl, ref_o, ref_lse, dtype)
    if not backward:
        return
    do = inp["do"].to(dev)
    dq = torch.full_like(q, float("nan"))
    dk = torch.full_like(k, float("nan"))
    dv = torch.full_like(v, float("nan"))
    ws = torch.full((fa.fa_bwd_workspace_bytes(B, H, Nq, Nk, D),), 0xFF, dtype=torch.uint8, device=dev)
    fa.fa_bwd_mask(q, k, v, o, lse, do, dq, dk, dv, ws, mdev, causal=causal, tile_flags=flags)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    ref = oracle.bwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["do"]), None, causal, scale,
                     mask=m64)
    got = [t.float().cpu().numpy().reshape(B * H, *t.shape[2:]) for t in (dq, dk, dv)]
    for name, g in zip(("dq", "dk", "dv"), got):
        assert not np.isnan(g).any(), name
    compare_grads(got, ref)


@pytest.mark.parametrize("kind", ["random", "window", "document", "rows"])
@pytest.mark.parametrize("causal", [False, True])
def test_mask_kinds(kind, causal):
    _case(2, 2, 300, 300, 64, "bf16", causal, kind, (False, False), seed=11)


@pytest.mark.parametrize("planes", [(True, False), (False, True), (True, True)])
def test_mask_planes(planes):
    _case(2, 3, 200, 333, 128, "f16", False, "random", planes, seed=12)


def test_mask_padded_rows_and_ragged():
    # row stride wider than Nk (padding filled with NaN must never be read)
    _case(1, 2, 129, 517, 64, "bf16", False, "random", (False, True), seed=13, ldm=520 + 64)
    _case(1, 2, 517, 129, 128, "bf16", True, "document", (False, False), seed=14, ldm=132)
    _case(2, 1, 5, 7, 64, "f16", False, "rows", (True, False), seed=15)


def test_mask_long_rows_sampled():
    """B=1 H=4 N=4096 D=128, one document mask for all heads; forward on
    sampled rows (every tile boundary plus 512 seeded rows), no backward."""
    N = 4096
    rows = inputs.sample_rows(N, seed=3)
    _case(1, 4, N, N, 128, "bf16", False, "document", (False, False), seed=16, backward=False,
          rows=rows)


def test_all_hidden_mask_gives_empty_rows():
    dev = torch.device("cuda")
    B, H, N, D = 1, 2, 130, 64
    inp = inputs.make_inputs(B, H, N, N, D, dtype="bf16", seed=17, with_dO=True)
    q, k, v, do = (inp[x].to(dev) for x in ("q", "k", "v", "do"))
    mask = torch.full((N, N + 2), -math.inf, device=dev)[:, :N]   # rows padded to 132
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    fa.fa_fwd_mask(q, k, v, o, lse, mask)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty((fa.fa_bwd_workspace_bytes(B, H, N, N, D),), dtype=torch.uint8, device=dev)
    fa.fa_bwd_mask(q, k, v, o, lse, do, dq, dk, dv, ws, mask)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    assert torch.all(o == 0) and torch.all(lse == -math.inf)
    assert torch.all(dq == 0) and torch.all(dk == 0) and torch.all(dv == 0)


def test_zero_mask_equals_plain_attention():
    dev = torch.device("cuda")
    inp = inputs.make_inputs(2, 2, 384, 384, 128, dtype="bf16", seed=18)
    q, k, v = (inp[x].to(dev) for x in ("q", "k", "v"))
    o1, l1 = fa.attention_forward(q, k, v, causal=True)
    o2, l2 = torch.empty_like(q), torch.empty_like(l1)
    fa.fa_fwd_mask(q, k, v, o2, l2, torch.zeros((384, 384), device=dev), causal=True)
    torch.cuda.synchronize()
    # same result up to rounding (the plain path exponentiates a quarter of
    # the scores on the FMA pipe; the mask path uses MUFU throughout)
    assert float((o1.float() - o2.float()).abs().max()) <= 2e-2
    assert float((l1 - l2).abs().max()) <= 1e-3


def _host_flags(mask):
    """The tile summary recomputed on the host: 1 where a 128 x 128 tile of a
    plane has an entry above -inf."""
    m = mask.detach().cpu().double().numpy()
    if m.ndim == 2:
        m = m[None, None]
    P = m.shape[0] * m.shape[1]
    m = m.reshape(P, m.shape[2], m.shape[3])
    nq, nk = -(-m.shape[1] // 128), -(-m.shape[2] // 128)
    out = np.zeros((P, nq, nk), dtype=np.uint8)
    for pl in range(P):
        for a in range(nq):
            for b in range(nk):
                out[pl, a, b] = np.any(m[pl, a * 128:(a + 1) * 128, b * 128:(b + 1) * 128] > -np.inf)
    return out


@pytest.mark.parametrize("kind,planes", [("document", (1, 1)), ("window", (2, 1)), ("random", (1, 3)),
                                         ("rows", (2, 2))])
def test_tile_flags_match_the_mask(kind, planes):
    m = inputs.make_mask(kind, 700, 900, seed=21, planes=planes)
    mdev = (m._base if m._base is not None else m).cuda()[..., :900]
    flags = fa.mask_tile_flags(mdev)
    torch.cuda.synchronize()
    assert np.array_equal(flags.cpu().numpy(), _host_flags(m))


@pytest.mark.parametrize("kind", ["document", "window", "rows"])
@pytest.mark.parametrize("causal", [False, True])
def test_tile_skipping_parity(kind, causal):
    # with the summary, tiles that are entirely -inf are skipped; results as the oracle
    _case(1, 2, 1100, 1100, 64, "bf16", causal, kind, (False, False), seed=22, use_flags=True)
    _case(2, 2, 700, 900, 128, "f16", False, kind, (True, False), seed=23, use_flags=True)


def test_tile_skipping_long_document_mask():
    N = 4096
    rows = inputs.sample_rows(N, seed=4)
    _case(1, 4, N, N, 128, "bf16", False, "document", (False, False), seed=24, backward=False,
          rows=rows, use_flags=True)
