"""Pins for the float64 oracle (CPU only).

The oracle is trusted only because it agrees with things other than itself:

* a library routine for the same operation (torch's scaled_dot_product_attention
  and its autograd, float64, CPU math path);
* closed forms the pages' definitions fix: uniform scores give the mean of the
  visible V rows and LSE = ln(#visible); a dominant one-hot key returns that
  key's value row; a single key returns its value row;
* brute force in pure Python on tiny inputs;
* the online (tiled) form of the slides: any tiling and any tile order give the
  same answer (FlashAttention case-study slides, "Online softmax: divide once,
  at the end"; merge associativity from "Mastering FlashAttention: The
  Algebraic Foundation");
* central finite differences of the oracle's own forward for its backward.

The last test plants plausible mistakes in copies of the oracle source and
checks that every one of them fails at least one pin.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import online

RNG = np.random.default_rng(20241204)


# --------------------------------------------------------------------------
# helpers (independent of the oracle's code)
# --------------------------------------------------------------------------

def visible_mask(Nq, Nk, causal, bias_row=None):
    """Boolean [Nq, Nk]: which keys a query may see (bottom-right causal)."""
    m = np.ones((Nq, Nk), dtype=bool)
    if causal:
        i = np.arange(Nq)[:, None]
        j = np.arange(Nk)[None, :]
        m &= j <= i + (Nk - Nq)
    if bias_row is not None:
        m &= np.isfinite(bias_row)[None, :]
    return m


def torch_sdpa(q, k, v, bias, causal, scale):
    """torch's SDPA in float64 with an explicit additive float mask."""
    B, H, Nq, D = q.shape
    Nk = k.shape[2]
    mask = np.zeros((B, 1, Nq, Nk))
    if causal:
        mask[:, :, ~visible_mask(Nq, Nk, True)] = -np.inf
    if bias is not None:
        mask = mask + bias[:, None, None, :]
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True)
                  for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=torch.tensor(mask), scale=scale)
    return out, (tq, tk, tv)


def rand_case(B, H, Nq, Nk, D, causal, with_bias, std=1.0, finite_bias=True):
    q = RNG.standard_normal((B, H, Nq, D)) * std
    k = RNG.standard_normal((B, H, Nk, D)) * std
    v = RNG.standard_normal((B, H, Nk, D))
    bias = None
    if with_bias:
        bias = RNG.standard_normal((B, Nk)) if finite_bias else np.zeros((B, Nk))
        for b in range(B):
            cols = RNG.choice(Nk, size=max(1, Nk // 5), replace=False)
            bias[b, cols] = -np.inf
        if causal:   # keep every row non-empty for the library comparison
            bias[:, 0] = 0.0
    return q, k, v, bias


# --------------------------------------------------------------------------
# pins, written as functions of an oracle object so that planted mistakes
# can be run through exactly the same checks
# --------------------------------------------------------------------------

def pin_library(orc):
    """Agreement with torch SDPA (float64) for O, several shapes and masks."""
    worst = 0.0
    for (Nq, Nk, D, causal, wb, std) in [(9, 13, 5, False, False, 1.0),
                                          (9, 13, 5, True, False, 1.0),
                                          (11, 11, 8, True, True, 1.0),
                                          (7, 16, 4, False, True, 1.0),
                                          (6, 10, 3, False, False, 12.0)]:
        q, k, v, bias = rand_case(2, 3, Nq, Nk, D, causal, wb, std)
        scale = 1.0 / math.sqrt(D) if std == 1.0 else 7.0
        o, _ = orc.fwd(q, k, v, bias, causal, scale)
        ref, _ = torch_sdpa(q, k, v, bias, causal, scale)
        worst = max(worst, float(np.abs(o - ref.detach().numpy()).max()))
    return worst <= 1e-12, worst


def pin_uniform(orc):
    """Q = 0: every visible score is equal, so O_i = mean of visible V_j and
    LSE_i = ln(#visible keys); also exercises causal alignment for Nq < Nk,
    Nq = Nk, Nq > Nk (rows with no visible key: O = 0, LSE = -inf)."""
    worst = 0.0
    for (Nq, Nk, causal, wb) in [(8, 8, True, False), (5, 12, True, False),
                                 (12, 5, True, False), (9, 9, False, True),
                                 (10, 14, True, True)]:
        B, H, D = 2, 2, 6
        q = np.zeros((B, H, Nq, D))
        k = RNG.standard_normal((B, H, Nk, D))
        v = RNG.standard_normal((B, H, Nk, D))
        bias = None
        if wb:
            bias = np.zeros((B, Nk))
            for b in range(B):
                bias[b, RNG.choice(Nk, size=3, replace=False)] = -np.inf
        o, lse = orc.fwd(q, k, v, bias, causal, 0.37)
        for b in range(B):
            vis = visible_mask(Nq, Nk, causal, None if bias is None else bias[b])
            cnt = vis.sum(axis=1)
            for h in range(H):
                for i in range(Nq):
                    if cnt[i] == 0:
                        exp_o = np.zeros(D)
                        if lse[b, h, i] != -np.inf:
                            return False, float("inf")
                    else:
                        exp_o = v[b, h][vis[i]].mean(axis=0)
                        worst = max(worst, abs(lse[b, h, i] - math.log(cnt[i])))
                    worst = max(worst, float(np.abs(o[b, h, i] - exp_o).max()))
    return worst <= 1e-12, worst


def pin_one_hot(orc):
    """Q_i = c e_i, K_j = c e_j with c^2 * scale = 30: key i dominates row i by
    30 nats, so O_i - V_i = sum_{j != i} P_ij (V_j - V_i) is at most
    (N - 1) e^-30 * 2 max|V| in size."""
    N, D = 12, 16
    scale = 1.0 / math.sqrt(D)
    c = math.sqrt(30.0 / scale)
    q = np.zeros((1, 2, N, D))
    k = np.zeros((1, 2, N, D))
    perm = RNG.permutation(D)[:N]
    for i in range(N):
        q[0, :, i, perm[i]] = c
        k[0, :, i, perm[i]] = c
    v = RNG.uniform(-1, 1, (1, 2, N, D))
    o, lse = orc.fwd(q, k, v, None, False, scale)
    err = float(np.abs(o - v).max())
    lse_err = float(np.abs(lse - (30.0 + np.log1p((N - 1) * math.exp(-30.0)))).max())
    ok = err <= 2.0 * (N - 1) * math.exp(-30.0) * float(np.abs(v).max()) + 1e-15 \
        and lse_err <= 1e-12
    return ok, max(err, lse_err)


def pin_shift_invariance(orc):
    """Adding a constant c to every score leaves O unchanged and moves LSE by
    exactly c; with c = -1000 or +700 the unshifted exponentials would
    underflow or overflow in float64, so this also checks that the maximum is
    subtracted before exponentiating (the overflow concern of the algebra
    digest, "Mastering FlashAttention")."""
    q, k, v, _ = rand_case(2, 2, 9, 11, 4, True, False)
    o0, l0 = orc.fwd(q, k, v, np.zeros((2, 11)), True, 0.5)
    worst = 0.0
    for c in (-1000.0, 700.0):
        o1, l1 = orc.fwd(q, k, v, np.full((2, 11), c), True, 0.5)
        if not (np.all(np.isfinite(o1)) and np.all(np.isfinite(l1))):
            return False, float("inf")
        worst = max(worst, float(np.abs(o1 - o0).max()),
                    float(np.abs((l1 - c) - l0).max()) / 1000.0)
    return worst <= 1e-12, worst


def pin_single_key(orc):
    """Nk = 1: O_i = V_0 and LSE_i = scale * q_i . k_0 + bias_0."""
    q, k, v, _ = rand_case(2, 2, 7, 1, 5, False, False)
    bias = RNG.standard_normal((2, 1))
    o, lse = orc.fwd(q, k, v, bias, False, 0.3)
    want_lse = 0.3 * np.einsum("bhid,bhjd->bhi", q, k) + bias[:, None, :]
    err = max(float(np.abs(o - v).max()), float(np.abs(lse - want_lse).max()))
    return err <= 1e-12, err


def _brute(q, k, v, bias, causal, scale):
    """Pure-Python loops with math.exp, no numpy arithmetic."""
    B, H, Nq, D = q.shape
    Nk = k.shape[2]
    O = np.zeros((B, H, Nq, D))
    L = np.zeros((B, H, Nq))
    for b in range(B):
        for h in range(H):
            for i in range(Nq):
                ws, idx = [], []
                for j in range(Nk):
                    if causal and j > i + (Nk - Nq):
                        continue
                    s = scale * sum(float(q[b, h, i, d]) * float(k[b, h, j, d])
                                    for d in range(D))
                    if bias is not None:
                        s += float(bias[b, j])
                    if s == -math.inf:
                        continue
                    ws.append(s)
                    idx.append(j)
                if not ws:
                    L[b, h, i] = -math.inf
                    continue
                mx = max(ws)
                e = [math.exp(s - mx) for s in ws]
                tot = sum(e)
                for d in range(D):
                    O[b, h, i, d] = sum(e[t] * float(v[b, h, idx[t], d])
                                        for t in range(len(e))) / tot
                L[b, h, i] = mx + math.log(tot)
    return O, L


def pin_brute(orc):
    worst = 0.0
    for (Nq, Nk, causal, wb) in [(4, 6, True, True), (6, 4, True, False),
                                 (5, 5, False, True)]:
        q, k, v, bias = rand_case(1, 2, Nq, Nk, 3, causal, wb)
        o, lse = orc.fwd(q, k, v, bias, causal, 0.55)
        O, L = _brute(q, k, v, bias, causal, 0.55)
        fin = np.isfinite(L)
        if not np.array_equal(fin, np.isfinite(lse)):
            return False, float("inf")
        worst = max(worst, float(np.abs(o - O).max()),
                    float(np.abs(lse[fin] - L[fin]).max()) if fin.any() else 0.0)
    return worst <= 1e-12, worst


def pin_online(orc):
    """Two-pass oracle == online running-state form for random tilings and
    random tile orders (fully masked tiles included)."""
    worst = 0.0
    for trial in range(12):
        Nq = int(RNG.integers(1, 40))
        Nk = int(RNG.integers(1, 200))
        D = int(RNG.integers(1, 9))
        causal = bool(trial % 2)
        q = RNG.standard_normal((1, 1, Nq, D)) * (1 + 3 * (trial % 3))
        k = RNG.standard_normal((1, 1, Nk, D))
        v = RNG.standard_normal((1, 1, Nk, D))
        bias = None
        if trial % 4 == 3:
            bias = np.where(RNG.random((1, Nk)) < 0.3, -np.inf, RNG.standard_normal((1, Nk)))
        sizes = []
        left = Nk
        while left:
            t = int(RNG.integers(1, min(64, left) + 1))
            sizes.append(t)
            left -= t
        order = RNG.permutation(len(sizes))
        o, lse = orc.fwd(q, k, v, bias, causal, 0.4)
        o2, lse2 = online.fwd_online(q[0, 0], k[0, 0], v[0, 0],
                                     None if bias is None else bias[0], causal, 0.4,
                                     sizes, order)
        fin = np.isfinite(lse2)
        if not np.array_equal(fin, np.isfinite(lse[0, 0])):
            return False, float("inf")
        scale_o = max(1.0, float(np.abs(o2).max()))
        worst = max(worst, float(np.abs(o[0, 0] - o2).max()) / scale_o)
        if fin.any():
            worst = max(worst, float(np.abs(lse[0, 0][fin] - lse2[fin]).max()
                                     / max(1.0, np.abs(lse2[fin]).max())))
    return worst <= 1e-12, worst


def _loss(orc, q, k, v, do, bias, causal, scale):
    o, _ = orc.fwd(q, k, v, bias, causal, scale)
    return float((o * do).sum())


def pin_finite_differences(orc):
    """Central differences (h = 1e-6) of L = sum(O * dO) against the oracle's
    analytic backward, relative to the largest gradient entry."""
    worst = 0.0
    for (Nq, Nk, D, causal, wb) in [(5, 5, 3, True, False), (7, 5, 5, False, True),
                                    (5, 7, 3, True, True)]:
        q, k, v, bias = rand_case(1, 2, Nq, Nk, D, causal, wb)
        do = RNG.standard_normal(q.shape)
        scale = 0.45
        dq, dk, dv = orc.bwd(q, k, v, do, bias, causal, scale)
        for x, g in ((q, dq), (k, dk), (v, dv)):
            num = np.zeros_like(x)
            h = 1e-6
            for idx in np.ndindex(x.shape):
                old = x[idx]
                x[idx] = old + h
                lp = _loss(orc, q, k, v, do, bias, causal, scale)
                x[idx] = old - h
                lm = _loss(orc, q, k, v, do, bias, causal, scale)
                x[idx] = old
                num[idx] = (lp - lm) / (2 * h)
            num = num.reshape(g.shape)
            denom = max(float(np.abs(num).max()), 1e-30)
            worst = max(worst, float(np.abs(num - g).max()) / denom)
    return worst <= 1e-6, worst


def pin_autograd(orc):
    """Oracle backward == torch autograd through float64 SDPA."""
    worst = 0.0
    for (Nq, Nk, D, causal, wb) in [(9, 12, 6, True, False), (10, 10, 8, False, True),
                                    (8, 13, 4, True, True)]:
        q, k, v, bias = rand_case(2, 2, Nq, Nk, D, causal, wb)
        do = RNG.standard_normal(q.shape)
        scale = 1.0 / math.sqrt(D)
        dq, dk, dv = orc.bwd(q, k, v, do, bias, causal, scale)
        out, (tq, tk, tv) = torch_sdpa(q, k, v, bias, causal, scale)
        out.backward(torch.tensor(do))
        for g, t in ((dq, tq), (dk, tk), (dv, tv)):
            ref = t.grad.numpy().reshape(g.shape)
            worst = max(worst, float(np.abs(g - ref).max()) / max(1e-30, float(np.abs(ref).max())))
    return worst <= 1e-10, worst


# ---- the general additive mask [B or 1, H or 1, Nq, Nk] ----------------------

def rand_mask(shape, frac_masked=0.25, std=1.0):
    """Finite N(0, std^2) entries with a random share set to -inf; column 0 of
    every row stays finite so that no row is empty."""
    m = RNG.standard_normal(shape) * std
    m[RNG.random(shape) < frac_masked] = -np.inf
    m[..., 0] = RNG.standard_normal(shape[:-1])
    return m


def pin_mask_library(orc):
    """General mask: O == torch SDPA (float64) with the same additive float
    mask, for full, head-broadcast and batch-broadcast shapes, also combined
    with causal and a key bias."""
    worst = 0.0
    for (Nq, Nk, D, mshape, causal, wb) in [(9, 13, 5, (2, 3), False, False),
                                            (9, 13, 5, (1, 3), False, True),
                                            (11, 11, 8, (2, 1), True, False),
                                            (7, 16, 4, (1, 1), False, False)]:
        q, k, v, bias = rand_case(2, 3, Nq, Nk, D, causal, wb)
        m = rand_mask(mshape + (Nq, Nk))
        if causal:
            m[..., :, 0] = 0.0
        scale = 1.0 / math.sqrt(D)
        o, _ = orc.fwd(q, k, v, bias, causal, scale, mask=m)
        full = np.broadcast_to(m, (2, 3, Nq, Nk)).copy()
        if causal:
            full[:, :, ~visible_mask(Nq, Nk, True)] = -np.inf
        if bias is not None:
            full = full + bias[:, None, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(
            *(torch.tensor(x) for x in (q, k, v)), attn_mask=torch.tensor(full), scale=scale)
        worst = max(worst, float(np.abs(o - ref.numpy()).max()))
    return worst <= 1e-12, worst


def pin_mask_row_shift(orc):
    """Adding c_i to every entry of mask row i leaves O unchanged and adds c_i
    to LSE_i (softmax is shift invariant per row); a mask applied to the wrong
    axis or scaled would break this."""
    q, k, v, _ = rand_case(2, 2, 10, 14, 6, False, False)
    m = rand_mask((2, 2, 10, 14))
    c = RNG.uniform(-5, 5, size=(2, 2, 10, 1))
    o0, l0 = orc.fwd(q, k, v, None, False, 0.4, mask=m)
    o1, l1 = orc.fwd(q, k, v, None, False, 0.4, mask=m + c)
    err = max(float(np.abs(o1 - o0).max()), float(np.abs(l1 - (l0 + c[..., 0])).max()))
    return err <= 1e-11, err


def pin_mask_prefix_mean(orc):
    """Q = 0 and a 0/-inf mask: O_i is the mean of the V rows the mask leaves
    visible to row i and LSE_i = ln(#visible) (exact row/column indexing)."""
    B, H, Nq, Nk, D = 1, 2, 12, 9, 4
    q = np.zeros((B, H, Nq, D))
    _, k, v, _ = rand_case(B, H, Nq, Nk, D, False, False)
    vis = RNG.random((B, H, Nq, Nk)) < 0.5
    vis[..., RNG.integers(0, Nk, size=(B, H, Nq))[..., None] == np.arange(Nk)] = True
    m = np.where(vis, 0.0, -np.inf)
    o, lse = orc.fwd(q, k, v, None, False, 1.0, mask=m)
    err = 0.0
    for h in range(H):
        for i in range(Nq):
            sel = vis[0, h, i]
            want = v[0, h, sel].mean(axis=0)
            err = max(err, float(np.abs(o[0, h, i] - want).max()),
                      abs(float(lse[0, h, i]) - math.log(int(sel.sum()))))
    return err <= 1e-12, err


def pin_mask_causal_equivalence(orc):
    """A 0/-inf mask holding the bottom-right causal pattern gives the causal
    result (Nq != Nk both ways), forward and backward."""
    err = 0.0
    for (Nq, Nk) in [(7, 12), (12, 7)]:
        q, k, v, _ = rand_case(1, 2, Nq, Nk, 5, True, False)
        do = RNG.standard_normal(q.shape)
        m = np.where(visible_mask(Nq, Nk, True), 0.0, -np.inf)
        o0, l0 = orc.fwd(q, k, v, None, True, 0.5)
        o1, l1 = orc.fwd(q, k, v, None, False, 0.5, mask=m)
        g0 = orc.bwd(q, k, v, do, None, True, 0.5)
        g1 = orc.bwd(q, k, v, do, None, False, 0.5, mask=m)
        both = np.isfinite(l0)
        empty_ok = bool(np.all(np.isneginf(l1[~both]))) and bool(np.all(np.isneginf(l0[~both])))
        err = max(err, float(np.abs(o1 - o0).max()), float(np.abs(l1[both] - l0[both]).max()),
                  0.0 if empty_ok else 1.0,
                  *(float(np.abs(a - b).max()) for a, b in zip(g0, g1)))
    return err <= 1e-12, err


def pin_mask_autograd(orc):
    """Backward with a general mask == torch autograd through float64 SDPA."""
    q, k, v, _ = rand_case(2, 2, 9, 11, 6, False, False)
    m = rand_mask((1, 2, 9, 11))
    do = RNG.standard_normal(q.shape)
    dq, dk, dv = orc.bwd(q, k, v, do, None, False, 0.35, mask=m)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.tensor(m),
                                                           scale=0.35)
    out.backward(torch.tensor(do))
    worst = 0.0
    for g, t in ((dq, tq), (dk, tk), (dv, tv)):
        ref = t.grad.numpy().reshape(g.shape)
        worst = max(worst, float(np.abs(g - ref).max()) / max(1e-30, float(np.abs(ref).max())))
    return worst <= 1e-10, worst


PINS = [pin_library, pin_uniform, pin_one_hot, pin_shift_invariance,
        pin_single_key, pin_brute,
        pin_online, pin_finite_differences, pin_autograd,
        pin_mask_library, pin_mask_row_shift, pin_mask_prefix_mean,
        pin_mask_causal_equivalence, pin_mask_autograd]


@pytest.fixture(scope="module")
def orc():
    oracle.build()
    return oracle.Oracle(oracle._load())


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(orc, pin):
    ok, err = pin(orc)
    assert ok, f"{pin.__name__}: error {err}"


def test_rows_subset_matches_full(orc):
    q, k, v, bias = rand_case(2, 3, 37, 29, 8, True, True)
    o, lse = orc.fwd(q, k, v, bias, True, 0.3)
    rows = np.array([0, 5, 36, 17])
    o2, lse2 = orc.fwd(q, k, v, bias, True, 0.3, rows=rows)
    assert np.array_equal(o[:, :, rows], o2)
    assert np.array_equal(lse[:, :, rows], lse2)


def test_bwd_subset_of_heads(orc):
    q, k, v, _ = rand_case(2, 3, 6, 6, 4, True, False)
    do = RNG.standard_normal(q.shape)
    full = orc.bwd(q, k, v, do, None, True, 0.5)
    part = orc.bwd(q, k, v, do, None, True, 0.5, bh_list=[4, 1])
    for a, b in zip(full, part):
        assert np.array_equal(a[[4, 1]], b)


def test_bwd_row_sample_is_a_partition(orc):
    """Row-sampled backward: the dQ rows are exact and the dK, dV shares of
    disjoint row sets add up to the full gradient."""
    q, k, v, bias = rand_case(1, 2, 9, 11, 4, True, True)
    do = RNG.standard_normal(q.shape)
    full = orc.bwd(q, k, v, do, bias, True, 0.5)
    a = orc.bwd(q, k, v, do, bias, True, 0.5, rows=[0, 3, 4, 8])
    b = orc.bwd(q, k, v, do, bias, True, 0.5, rows=[1, 2, 5, 6, 7])
    assert np.allclose(a[0][:, [0, 3, 4, 8]], full[0][:, [0, 3, 4, 8]], rtol=0, atol=1e-14)
    for t in (1, 2):
        assert np.allclose(a[t] + b[t], full[t], rtol=1e-13, atol=1e-14)


def test_merge_monoid():
    """(+) is associative and commutative with identity (-inf, 0, 0)."""
    rows, D = 6, 4

    def rand_state(masked=False):
        s = RNG.standard_normal((rows, 5)) * 4
        if masked:
            s[:3] = -np.inf
        return online.tile_state(s, RNG.standard_normal((5, D)))

    a, b, c = rand_state(), rand_state(True), rand_state()
    e = online.identity_state(rows, D)

    def close(x, y):
        return all(np.allclose(p, q, rtol=1e-13, atol=1e-13) for p, q in zip(x, y))

    assert close(online.merge(online.merge(a, b), c), online.merge(a, online.merge(b, c)))
    assert close(online.merge(a, b), online.merge(b, a))
    assert close(online.merge(a, e), a) and close(online.merge(e, b), b)


def test_alpha_identity():
    """e^(s - m_old) e^(m_old - m_new) = e^(s - m_new), the slides' correction."""
    s, m_old, m_new = RNG.standard_normal(3) * 5
    assert math.isclose(math.exp(s - m_old) * math.exp(m_old - m_new),
                        math.exp(s - m_new), rel_tol=1e-14)


def test_golden_llama_shapes():
    """The slides' Llama-3-8B figures: d/h = d_k, S,P are n/d_k = 64x larger
    than Q,K,V,O, and 4 h n^2 d_k is about 1.1 TFLOP; the metric's FLOP formula
    reproduces them."""
    import json
    import os
    from exact_attention_112_b200 import metrics
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "llama3_8b_layer.json")))
    assert g["d_model"] // g["heads"] == g["d_k"]
    assert (g["n"] * g["n"]) // (g["n"] * g["d_k"]) == g["S_and_P_size_over_QKVO_size"]
    f = metrics.fwd_flops(1, g["heads"], g["n"], g["n"], g["d_k"], causal=False)
    assert abs(f - g["attention_gemm_flop_per_layer"]) <= g["attention_gemm_flop_rel_tol"] * f
    assert metrics.fwd_flops(1, 32, 8192, 8192, 128, True) == f / 2
    assert metrics.bwd_flops(1, 32, 8192, 8192, 128, True) == 2.5 * f / 2


# --------------------------------------------------------------------------
# planted mistakes: each must fail at least one pin
# --------------------------------------------------------------------------

MUTANTS = {
    "causal_off_by_one": ("return j <= i + (Nk - Nq);", "return j < i + (Nk - Nq);"),
    "causal_top_left": ("return j <= i + (Nk - Nq);", "return j <= i;"),
    "dropped_scale": ("s = scale * dot;", "s = dot;"),
    "dropped_bias": ("if (bias_b) s += bias_b[j];", ""),
    "exp_sign": ("exp(p_row[j] - m)", "exp(m - p_row[j])"),
    "no_normalise": ("for (long j = 0; j < Nk; ++j) p_row[j] /= l;", ""),
    "lse_no_log": ("return m + log(l);", "return m + l;"),
    "no_max_shift": ("double m = -INFINITY;\n    for (long j = 0; j < Nk; ++j) {\n        double s;",
                     "double m = 0.0;\n    for (long j = 0; j < Nk; ++j) {\n        double s;"),
    "v_replaced_by_k": ("o_i[d] += p_row[j] * vh[j * D + d];", "o_i[d] += p_row[j] * kh[j * D + d];"),
    "k_index": ("dot += qi[d] * kh[j * D + d];", "dot += qi[d] * kh[d * Nk + j];"),
    "bwd_no_rowterm": ("double ds = p[j] * (dp[j] - Di);", "double ds = p[j] * dp[j];"),
    "bwd_dk_unscaled": ("dkh[j * D + d] += scale * ds * qh[i * D + d];",
                        "dkh[j * D + d] += ds * qh[i * D + d];"),
    "bwd_dv_uses_ds": ("dvh[j * D + d] += p[j] * doh[i * D + d];",
                       "dvh[j * D + d] += ds * doh[i * D + d];"),
    "bwd_dq_uses_v": ("dqh[i * D + d] += scale * ds * kh[j * D + d];",
                      "dqh[i * D + d] += scale * ds * vh[j * D + d];"),
    "mask_dropped": ("if (mask_bh) s += mask_bh[i * Nk + j];", ""),
    "mask_scaled": ("if (mask_bh) s += mask_bh[i * Nk + j];",
                    "if (mask_bh) s += scale * mask_bh[i * Nk + j];"),
    "mask_rows_reversed": ("if (mask_bh) s += mask_bh[i * Nk + j];",
                           "if (mask_bh) s += mask_bh[(Nq - 1 - i) * Nk + j];"),
    "mask_head_stride_ignored": ("(bh % H) * mask_hstride", "0 * mask_hstride"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    before, after = MUTANTS[name]
    src = oracle.source_text()
    assert src.count(before) >= 1, f"mutation anchor missing: {name}"
    mutant = oracle.build_variant(src.replace(before, after), name)
    failed = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                ok, _ = pin(mutant)
        except Exception:
            ok = False
        if not ok:
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name} passed every pin"
