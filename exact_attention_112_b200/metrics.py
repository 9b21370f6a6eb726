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


def kernel_bytes(name, B, H, Nq, Nk, D, elem=2, out_elem=2, bias=False, splits=1):
    """Algorithmic HBM bytes of one launch of a library kernel (every input
    byte read once, every output byte written once), or None for a kernel this
    table does not know.  elem is the byte size of Q, K, V (and dO), out_elem
    that of O and the gradients; LSE, the row term D_i and split-KV partials
    are fp32."""
    BH = B * H
    qkv = elem * BH * D * (Nq + 2 * Nk)
    rows = BH * Nq
    if name == "fa_fwd_kernel":
        return qkv + out_elem * BH * Nq * D + 4 * rows + (4 * B * Nk if bias else 0)
    if name == "fa_fwd_split_kernel":
        return qkv + splits * rows * (4 * D + 4) + (4 * B * Nk if bias else 0)
    if name == "fa_fwd_combine_kernel":
        return splits * rows * (4 * D + 4) + out_elem * rows * D + 4 * rows
    if name == "fa_bwd_pre_kernel":
        return 2 * out_elem * rows * D + 4 * rows
    if name == "fa_bwd_dkdv_kernel":
        return qkv + elem * rows * D + 8 * rows + 2 * out_elem * BH * Nk * D + (4 * B * Nk if bias else 0)
    if name == "fa_bwd_dq_kernel":
        return qkv + elem * rows * D + 8 * rows + out_elem * rows * D + (4 * B * Nk if bias else 0)
    return None
