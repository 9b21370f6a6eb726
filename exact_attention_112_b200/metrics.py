"""Work and traffic counts used to turn timings into TFLOP/s and GB/s.

FLOPs follow the FlashAttention case-study slides (nmj0.github.io, "The same
computation at real size"): the two GEMMs of one head cost 4 * n^2 * d_k
FLOP (2 * n^2 * d_k each), i.e. 4 * B * H * Nq * Nk * D for a batch; causal
masking halves it (the convention the headline metric uses).  The backward pass
is counted as 2.5x the forward (five GEMMs of the same size instead of two).
"""
from __future__ import annotations


def fwd_flops(B, H, Nq, Nk, D, causal):
    f = 4.0 * B * H * Nq * Nk * D
    return f / 2.0 if causal else f


def bwd_flops(B, H, Nq, Nk, D, causal):
    return 2.5 * fwd_flops(B, H, Nq, Nk, D, causal)


def fwd_bytes(B, H, Nq, Nk, D, elem=2, bias=False):
    """Algorithmic HBM bytes of one forward: read Q, K, V once, write O once,
    write the fp32 LSE, read the fp32 key bias if present."""
    b = elem * B * H * D * (2 * Nq + 2 * Nk) + 4 * B * H * Nq
    if bias:
        b += 4 * B * Nk
    return b


def bwd_bytes(B, H, Nq, Nk, D, elem=2):
    """Algorithmic HBM bytes of one backward: read Q, K, V, O, dO and LSE; write
    dQ, dK, dV; the row term D_i is written and read once (fp32)."""
    reads = elem * B * H * D * (3 * Nq + 2 * Nk) + 4 * B * H * Nq
    writes = elem * B * H * D * (Nq + 2 * Nk)
    rowterm = 2 * 4 * B * H * Nq
    return reads + writes + rowterm
