"""C-ABI checks that need no GPU: the library loads, exports every function
include/fa.h declares, and rejects bad arguments synchronously (before any
CUDA call) with the documented status codes."""
import ctypes
import os
import re
import subprocess

import pytest

import exact_attention_112_b200 as fa
from exact_attention_112_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    _build.build()
    return fa.lib()


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert {"fa_fwd", "fa_bwd", "fa_bwd_workspace_bytes", "fa_status_string",
            "fa_device_status"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", fa.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r" T (\w+)$", out, flags=re.M))
    for n in names:
        assert n in exported, f"{n} declared in fa.h but not exported"
        assert hasattr(L, n)


def test_status_strings(L):
    for code in range(6):
        s = fa.fa_status_string(code)
        assert s and s.startswith("FA_")
    assert "unknown" in fa.fa_status_string(99)


def _fwd(L, q=1, k=1, v=1, o=1, lse=1, B=1, H=1, Nq=128, Nk=128, D=64, causal=0,
         scale=0.125, dtype=0, bias=None):
    P = lambda x: None if x is None else ctypes.c_void_p(16 * x if x else 0)
    return L.fa_fwd(P(q), P(k), P(v), P(o), P(lse), B, H, Nq, Nk, D, causal,
                    ctypes.c_float(scale), dtype, P(bias), None)


def test_fwd_argument_errors_are_synchronous(L):
    assert _fwd(L, D=96) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(L, D=256) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(L, dtype=7) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(L, B=0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, H=-1) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, Nk=-3) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, causal=2) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, scale=0.0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, scale=float("nan")) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, scale=float("inf")) == fa.FA_ERR_INVALID_ARG
    assert _fwd(L, q=0) == fa.FA_ERR_INVALID_ARG          # null pointer
    assert _fwd(L, lse=0) == fa.FA_ERR_INVALID_ARG
    # misaligned (not a multiple of 16 bytes)
    assert L.fa_fwd(ctypes.c_void_p(24), ctypes.c_void_p(32), ctypes.c_void_p(48),
                    ctypes.c_void_p(64), ctypes.c_void_p(80), 1, 1, 128, 128, 64, 0,
                    ctypes.c_float(0.1), 0, None, None) == fa.FA_ERR_INVALID_ARG
    # index overflow guard
    assert _fwd(L, B=1 << 16, H=1 << 16) == fa.FA_ERR_INVALID_ARG


def test_fwd_empty_query_is_a_noop(L):
    # Nq == 0: nothing to compute, no CUDA call, even with null pointers
    assert _fwd(L, q=None, k=None, v=None, o=None, lse=None, Nq=0) == fa.FA_OK


def test_workspace_size(L):
    B, H, N, D = 2, 32, 4096, 128
    ws = fa.fa_bwd_workspace_bytes(B, H, N, N, D)
    rows = B * H * N
    assert ws >= rows * 4
    assert ws < rows * 4 + 4096
    assert fa.fa_bwd_workspace_bytes(1, 1, 256, 256, 96) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(fa, "_lib", None)
    monkeypatch.setattr(fa, "library_path", lambda: str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        fa.lib()


def _bwd(L, dq=1, dk=1, ws=1, ws_bytes=1 << 20, B=1, H=1, Nq=128, Nk=128, D=64, causal=0,
         scale=0.125, dtype=0, q=1):
    P = lambda x: None if x is None else ctypes.c_void_p(16 * x if x else 0)
    return L.fa_bwd(P(q), P(2), P(3), P(4), P(5), P(6), P(dq), P(dk), P(9), B, H, Nq, Nk, D,
                    causal, ctypes.c_float(scale), dtype, None, P(ws), ctypes.c_size_t(ws_bytes), None)


def test_bwd_argument_errors_are_synchronous(L):
    assert _bwd(L, D=96) == fa.FA_ERR_UNSUPPORTED
    assert _bwd(L, B=0) == fa.FA_ERR_INVALID_ARG
    assert _bwd(L, causal=3) == fa.FA_ERR_INVALID_ARG
    assert _bwd(L, scale=-1.0) == fa.FA_ERR_INVALID_ARG
    assert _bwd(L, dq=0) == fa.FA_ERR_INVALID_ARG          # null dQ with queries present
    assert _bwd(L, dk=0) == fa.FA_ERR_INVALID_ARG          # null dK with keys present
    assert _bwd(L, ws=0) == fa.FA_ERR_WORKSPACE            # no workspace
    need = fa.fa_bwd_workspace_bytes(1, 1, 128, 128, 64)
    assert _bwd(L, ws_bytes=need - 1) == fa.FA_ERR_WORKSPACE
    # misaligned q
    assert L.fa_bwd(ctypes.c_void_p(24), *[ctypes.c_void_p(16 * i) for i in range(2, 10)], 1, 1, 128,
                    128, 64, 0, ctypes.c_float(0.1), 0, None, ctypes.c_void_p(16),
                    ctypes.c_size_t(1 << 20), None) == fa.FA_ERR_INVALID_ARG


def _split(L, num_splits=4, ws=1, ws_bytes=1 << 30, Nq=16, Nk=4096, D=128, k=1):
    P = lambda x: None if x is None else ctypes.c_void_p(16 * x if x else 0)
    return L.fa_fwd_splitkv(P(1), P(k), P(3), P(4), P(5), 1, 2, Nq, Nk, D, 0, ctypes.c_float(0.1),
                            1, None, num_splits, P(ws), ctypes.c_size_t(ws_bytes), None)


def test_splitkv_argument_errors_are_synchronous(L):
    assert _split(L, num_splits=0) == fa.FA_ERR_INVALID_ARG
    assert _split(L, num_splits=257) == fa.FA_ERR_INVALID_ARG
    assert _split(L, D=80) == fa.FA_ERR_UNSUPPORTED
    assert _split(L, k=0) == fa.FA_ERR_INVALID_ARG
    assert _split(L, ws=0) == fa.FA_ERR_WORKSPACE
    need = fa.fa_fwd_splitkv_workspace_bytes(1, 2, 16, 4096, 128, 4)
    assert _split(L, ws_bytes=need - 1) == fa.FA_ERR_WORKSPACE
    assert _split(L, Nq=0, k=None, ws=None) == fa.FA_OK      # nothing to do, no CUDA call


def test_splitkv_workspace_size(L):
    # partial O (fp32) and partial LSE per row and split, each 256-byte aligned, + slack
    rows = 1 * 2 * 16 * 4
    need = fa.fa_fwd_splitkv_workspace_bytes(1, 2, 16, 4096, 128, 4)
    assert need >= rows * 128 * 4 + rows * 4
    assert need <= rows * 128 * 4 + rows * 4 + 3 * 256
    assert fa.fa_fwd_splitkv_workspace_bytes(1, 2, 16, 4096, 128, 0) == 0
    assert fa.fa_fwd_splitkv_workspace_bytes(1, 2, 16, 4096, 96, 4) == 0


def test_noalloc_rejects_too_many_rows_before_any_cuda_call(L):
    P = lambda x: ctypes.c_void_p(16 * x)
    rows = fa.FA_BWD_NOALLOC_MAX_ROWS
    assert L.fa_bwd_noalloc(*[P(i) for i in range(1, 10)], 1, 1, rows + 1, 128, 64, 0,
                            ctypes.c_float(0.1), 0, None, None) == fa.FA_ERR_WORKSPACE


def test_noalloc_limit_matches_header_and_accepts_the_limit(L):
    """The Python constant is read from include/fa.h; exactly MAX_ROWS rows is
    not refused for size (an invalid dtype stops it at validation instead),
    and argument errors come before the size check."""
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    m = re.search(r"^#define\s+FA_BWD_NOALLOC_MAX_ROWS\s+(\d+)\s*$", text, flags=re.M)
    assert m and int(m.group(1)) == fa.FA_BWD_NOALLOC_MAX_ROWS
    P = lambda x: ctypes.c_void_p(16 * x)
    rows = fa.FA_BWD_NOALLOC_MAX_ROWS

    def call(B, H, Nq, dtype=0, D=64, ptrs=True):
        args = [P(i) for i in range(1, 10)] if ptrs else [None] * 9
        return L.fa_bwd_noalloc(*args, B, H, Nq, 128, D, 0, ctypes.c_float(0.1), dtype, None, None)

    assert call(1, 1, rows, dtype=7) == fa.FA_ERR_UNSUPPORTED
    assert call(1, 16, rows // 16, D=96) == fa.FA_ERR_UNSUPPORTED
    assert call(1, 1, rows + 1, dtype=7) == fa.FA_ERR_UNSUPPORTED   # argument errors first
    assert call(0, 1, rows + 1) == fa.FA_ERR_INVALID_ARG
    assert call(1, 1, rows + 1) == fa.FA_ERR_WORKSPACE
    assert call(4, 8, rows // 32 + 1) == fa.FA_ERR_WORKSPACE


# ---- the Python binding checks every tensor before taking its pointer ----

def _host(shape, dtype="bf16"):
    import torch
    dt = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[dtype]
    return torch.zeros(shape, dtype=dt)


def _fwd_args(B=2, H=3, Nq=40, Nk=56, D=64):
    return dict(q=_host((B, H, Nq, D)), k=_host((B, H, Nk, D)), v=_host((B, H, Nk, D)),
                o=_host((B, H, Nq, D)), lse=_host((B, H, Nq), "f32"))


def _expect_invalid(fn, match, **kw):
    with pytest.raises(fa.FaError, match=match) as e:
        fn(**kw)
    assert e.value.status == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("name,bad,match", [
    ("o", (2, 3, 39, 64), "o must have shape"),
    ("o", (2, 3, 40, 128), "o must have shape"),
    ("lse", (2, 3, 41), "lse must have shape"),
    ("v", (2, 3, 55, 64), "v must have shape"),
    ("k", (2, 4, 56, 64), "k must be"),
    ("k", (2, 3, 56, 32), "k must be"),
])
def test_binding_rejects_misshaped_forward_tensors(L, name, bad, match):
    kw = _fwd_args()
    kw[name] = _host(bad, "f32" if name == "lse" else "bf16")
    _expect_invalid(fa.fa_fwd, match, **kw)


def test_binding_rejects_wrong_dtypes_layout_and_device(L):
    kw = _fwd_args()
    kw["v"] = _host((2, 3, 56, 64), "f16")
    _expect_invalid(fa.fa_fwd, "v must be torch.bfloat16", **kw)
    kw = _fwd_args()
    kw["lse"] = _host((2, 3, 40), "bf16")
    _expect_invalid(fa.fa_fwd, "lse must be torch.float32", **kw)
    kw = _fwd_args()
    kw["key_bias"] = _host((2, 55), "f32")
    _expect_invalid(fa.fa_fwd, "key_bias must have shape", **kw)
    kw = _fwd_args()
    kw["key_bias"] = _host((2, 56), "bf16")
    _expect_invalid(fa.fa_fwd, "key_bias must be torch.float32", **kw)
    kw = _fwd_args()
    kw["o"] = _host((2, 3, 64, 40)).transpose(2, 3)       # right shape, wrong layout
    _expect_invalid(fa.fa_fwd, "contiguous", **kw)
    kw = _fwd_args()                                       # everything right but on the host
    _expect_invalid(fa.fa_fwd, "CUDA device", **kw)
    kw = _fwd_args()
    kw["q"] = _host((2, 3, 40, 64), "f32")
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd(**kw)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED


@pytest.mark.parametrize("fn", ["fa_bwd", "fa_bwd_noalloc"])
@pytest.mark.parametrize("name,bad", [("dq", (2, 3, 40, 32)), ("dk", (2, 3, 40, 64)),
                                      ("dv", (2, 3, 57, 64)), ("dO", (2, 3, 40, 128)),
                                      ("o", (1, 3, 40, 64))])
def test_binding_rejects_misshaped_backward_tensors(L, fn, name, bad):
    kw = _fwd_args()
    kw.update(dO=_host((2, 3, 40, 64)), dq=_host((2, 3, 40, 64)), dk=_host((2, 3, 56, 64)),
              dv=_host((2, 3, 56, 64)))
    if fn == "fa_bwd":
        kw["workspace"] = _host((fa.fa_bwd_workspace_bytes(2, 3, 40, 56, 64),), "f32")
    kw[name] = _host(bad)
    _expect_invalid(getattr(fa, fn), f"{name} must have shape", **kw)


def test_binding_rejects_missing_outputs_and_host_workspace(L):
    kw = _fwd_args()
    kw.update(dO=_host((2, 3, 40, 64)), dq=None, dk=_host((2, 3, 56, 64)),
              dv=_host((2, 3, 56, 64)), workspace=_host((4096,), "f32"))
    _expect_invalid(fa.fa_bwd, "dq is required", **kw)
    kw = _fwd_args()
    kw["num_splits"] = 4
    kw["workspace"] = _host((16,), "f32")
    kw["o"] = _host((2, 3, 40, 32))
    _expect_invalid(fa.fa_fwd_splitkv, "o must have shape", **kw)


def _fp8(L, D=128, qd=1.0, kd=1.0, vd=1.0, Nq=16, q=1):
    P = lambda x: None if x is None else ctypes.c_void_p(16 * x if x else 0)
    f = ctypes.c_float
    return L.fa_fwd_fp8(P(q), P(2), P(3), P(4), P(5), 1, 2, Nq, 64, D, 0, f(0.1), f(qd), f(kd), f(vd),
                        None, None)


def test_fp8_argument_errors_are_synchronous(L):
    assert _fp8(L, D=64) == fa.FA_ERR_UNSUPPORTED
    assert _fp8(L, D=96) == fa.FA_ERR_UNSUPPORTED
    for bad in (0.0, -2.0, float("nan"), float("inf")):
        assert _fp8(L, qd=bad) == fa.FA_ERR_INVALID_ARG
        assert _fp8(L, kd=bad) == fa.FA_ERR_INVALID_ARG
        assert _fp8(L, vd=bad) == fa.FA_ERR_INVALID_ARG
    assert _fp8(L, qd=1e30, kd=1e30) == fa.FA_ERR_INVALID_ARG      # scale * descales overflows
    assert _fp8(L, q=0) == fa.FA_ERR_INVALID_ARG
    assert _fp8(L, Nq=0, q=None) == fa.FA_OK


def test_fp8_binding_checks_types(L):
    import torch
    q = torch.zeros((1, 2, 8, 128), dtype=torch.float8_e4m3fn)
    o = torch.zeros((1, 2, 8, 128), dtype=torch.bfloat16)
    lse = torch.zeros((1, 2, 8), dtype=torch.float32)
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd_fp8(q.to(torch.bfloat16), q, q, o, lse)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    _expect_invalid(fa.fa_fwd_fp8, "o must be torch.bfloat16",
                    q=q, k=q, v=q, o=o.to(torch.float16), lse=lse)
    _expect_invalid(fa.fa_fwd_fp8, "v must be torch.float8_e4m3fn",
                    q=q, k=q, v=q.to(torch.bfloat16), o=o, lse=lse)
    _expect_invalid(fa.fa_fwd_fp8, "CUDA device", q=q, k=q, v=q, o=o, lse=lse)


def _varlen(L, cu=1, H=2, tq=100, tk=100, mq=64, mk=64, D=64, dtype=1):
    P = lambda x: None if x is None else ctypes.c_void_p(16 * x if x else 0)
    return L.fa_fwd_varlen(P(1), P(2), P(3), P(4), P(5), P(cu), P(cu), 3, H, tq, tk, mq, mk, D, 0,
                           ctypes.c_float(0.1), dtype, None)


def test_varlen_argument_errors_are_synchronous(L):
    assert _varlen(L, cu=0) == fa.FA_ERR_INVALID_ARG             # no sequence table
    assert _varlen(L, D=96) == fa.FA_ERR_UNSUPPORTED
    assert _varlen(L, dtype=5) == fa.FA_ERR_UNSUPPORTED
    assert _varlen(L, tq=-1) == fa.FA_ERR_INVALID_ARG
    assert _varlen(L, H=0) == fa.FA_ERR_INVALID_ARG
    assert _varlen(L, mq=-1) == fa.FA_ERR_INVALID_ARG
    assert L.fa_fwd_varlen(*[ctypes.c_void_p(16 * i) for i in range(1, 6)], ctypes.c_void_p(18),
                           ctypes.c_void_p(32), 3, 2, 100, 100, 64, 64, 64, 0, ctypes.c_float(0.1), 1,
                           None) == fa.FA_ERR_INVALID_ARG        # misaligned int32 table
    assert _varlen(L, tq=0) == fa.FA_OK                          # nothing to do, no CUDA call


def test_varlen_binding_checks_tables(L):
    import torch
    q = torch.zeros((2, 10, 64), dtype=torch.bfloat16)
    cu = torch.tensor([0, 4, 10], dtype=torch.int32)
    lse = torch.zeros((2, 10), dtype=torch.float32)
    _expect_invalid(fa.fa_fwd_varlen, "cu_seqlens_q must be a contiguous int32",
                    q=q, k=q, v=q, o=q, lse=lse, cu_seqlens_q=cu.long(), cu_seqlens_k=cu,
                    max_seqlen_q=6, max_seqlen_k=6)
    _expect_invalid(fa.fa_fwd_varlen, "must be on",
                    q=q, k=q, v=q, o=q, lse=lse, cu_seqlens_q=cu, cu_seqlens_k=cu,
                    max_seqlen_q=6, max_seqlen_k=6)
    _expect_invalid(fa.fa_fwd_varlen, "packed q and k must be 3-D",
                    q=q[None], k=q, v=q, o=q, lse=lse, cu_seqlens_q=cu, cu_seqlens_k=cu,
                    max_seqlen_q=6, max_seqlen_k=6)


def test_mask_tile_flags_arguments(L):
    P = lambda x: None if x is None else ctypes.c_void_p(16 * x if x else 0)
    assert fa.fa_mask_tile_flags_bytes(2, 3, 300, 129) == 2 * 3 * 3 * 2
    assert fa.fa_mask_tile_flags_bytes(0, 1, 10, 10) == 0
    call = lambda mask=1, Bm=1, Hm=1, Nq=300, Nk=200, ldm=200, flags=2, nbytes=1 << 20: \
        L.fa_mask_tile_flags(P(mask), Bm, Hm, Nq, Nk, ldm, P(flags), nbytes, None)
    assert call(mask=0) == fa.FA_ERR_INVALID_ARG
    assert call(ldm=198) == fa.FA_ERR_INVALID_ARG          # not a multiple of 4
    assert call(ldm=196) == fa.FA_ERR_INVALID_ARG          # shorter than Nk
    assert call(flags=0) == fa.FA_ERR_INVALID_ARG
    assert call(nbytes=5) == fa.FA_ERR_INVALID_ARG         # 3 x 2 tiles need 6 bytes
    assert call(Bm=0) == fa.FA_ERR_INVALID_ARG
    assert call(Nq=0, mask=None, flags=None) == fa.FA_OK   # no tile: nothing to do


def test_splitkv_num_splits_choice():
    # host arithmetic only (an explicit SM count touches no device)
    import exact_attention_112_b200 as fa
    # 8 units of 256 rows over 512 key tiles on 148 SMs: 18 splits of 29 tiles
    # fill 144 SMs in one wave (16 splits would leave 20 SMs idle)
    assert fa.fa_splitkv_num_splits(1, 8, 256, 65536, 148) == 18
    assert fa.fa_splitkv_num_splits(1, 8, 1, 65536, 148) == 18
    # enough units already: no split
    assert fa.fa_splitkv_num_splits(1, 32, 8192, 8192, 148) == 1
    # a single key tile cannot be split
    assert fa.fa_splitkv_num_splits(1, 1, 1, 100, 148) == 1
    # invalid sizes
    assert fa.fa_splitkv_num_splits(0, 8, 256, 65536, 148) == 1
    assert fa.fa_splitkv_num_splits(1, 8, 256, 65536, -1) == 1
    # every split holds key tiles, and the waves fit the SM count
    for B, H, Nq, Nk in [(1, 1, 1, 1000), (2, 4, 64, 20000), (1, 16, 512, 131072), (3, 5, 300, 7777)]:
        s = fa.fa_splitkv_num_splits(B, H, Nq, Nk, 148)
        tiles = (Nk + 127) // 128
        per = -(-tiles // s)
        assert 1 <= s <= min(256, tiles) and -(-tiles // per) == s
