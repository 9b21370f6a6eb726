"""The input recipe and the work counts, pinned to the figures the survey of
the pages fixes (host only).

FLOPs: 4*B*H*Nq*Nk*D per forward, halved when causal ("The same computation at
real size" slide: 4*h*n^2*d_k for one Llama-3-8B layer), backward 2.5x.
"""
import math

import numpy as np
import pytest
import torch

from exact_attention_112_b200 import inputs, metrics


def test_llama_layer_flops_match_the_slide():
    # one non-causal Llama-3-8B layer: 4 * 32 * 8192^2 * 128 = 1.0995e12 (~1.1 TFLOP)
    dense = metrics.fwd_flops(1, 32, 8192, 8192, 128, False)
    assert dense == 4 * 32 * 8192 ** 2 * 128
    assert abs(dense / 1e12 - 1.1) < 0.01
    assert metrics.fwd_flops(1, 32, 8192, 8192, 128, True) == pytest.approx(5.50e11, rel=1e-3)


@pytest.mark.parametrize("cfg,flops", [
    (("tiny", {}), 1.68e7),
    (("llama", {}), 5.50e11),
    (("stress", {}), 2.75e11),
    (("sweep", {"N": 512, "causal": False}), 6.87e10),
    (("sweep", {"N": 16384, "causal": False}), 2.20e12),
    (("sweep", {"N": 32768, "causal": False}), 8.80e12),
])
def test_config_flops(cfg, flops):
    name, over = cfg
    w = inputs.workload(name, **over)
    f = metrics.fwd_flops(w["B"], w["H"], w["Nq"], w["Nk"], w["D"], w["causal"])
    assert f == pytest.approx(flops, rel=2e-3)


def test_backward_config_flops():
    w = inputs.workload("bwd")
    f = metrics.bwd_flops(w["B"], w["H"], w["Nq"], w["Nk"], w["D"], w["causal"])
    assert f == pytest.approx(6.87e11, rel=2e-3)
    assert f == 2.5 * metrics.fwd_flops(w["B"], w["H"], w["Nq"], w["Nk"], w["D"], w["causal"])


def test_llama_forward_bytes():
    # Q, K, V, O: 4 x 64 MiB of 16-bit values, plus 1 MiB of fp32 LSE
    b = metrics.fwd_bytes(1, 32, 8192, 8192, 128)
    assert b == 4 * 64 * 2 ** 20 + 2 ** 20


def test_sweep_batch_rule():
    # B = max(1, 16384 // N): N = 32768 runs B = 1
    for n, b in [(512, 32), (1024, 16), (8192, 2), (16384, 1), (32768, 1)]:
        w = inputs.workload("sweep", N=n)
        assert (w["B"], w["Nq"], w["Nk"]) == (b, n, n)


def test_stress_bias_masks_205_distinct_keys_per_batch():
    w = inputs.workload("stress")
    inp = inputs.make_inputs(2, 1, 8, w["Nk"], 64, dtype="bf16", seed=w["seed"],
                             bias_frac=w["bias_frac"])
    bias = inp["key_bias"].numpy()
    assert bias.shape == (2, 2048)
    for b in range(2):
        assert int(np.isneginf(bias[b]).sum()) == round(0.1 * 2048) == 205
        assert np.all(bias[b][np.isfinite(bias[b])] == 0.0)
    assert not np.array_equal(np.isneginf(bias[0]), np.isneginf(bias[1]))


def test_inputs_are_seeded_and_rounded_once():
    a = inputs.make_inputs(1, 2, 33, 17, 64, dtype="bf16", seed=5, with_dO=True)
    b = inputs.make_inputs(1, 2, 33, 17, 64, dtype="bf16", seed=5, with_dO=True)
    c = inputs.make_inputs(1, 2, 33, 17, 64, dtype="bf16", seed=6, with_dO=True)
    for key in ("q", "k", "v", "do"):
        assert a[key].dtype == torch.bfloat16
        assert torch.equal(a[key], b[key])
    assert not torch.equal(a["q"], c["q"])
    # the oracle receives exactly the rounded values
    q64 = inputs.to_f64(a["q"])
    assert np.array_equal(q64, a["q"].to(torch.float64).numpy())
    assert np.array_equal(q64.astype(np.float32), q64)


def test_sample_rows_cover_every_tile_boundary():
    rows = inputs.sample_rows(1000, seed=3)
    for t in range(0, 1000, 128):
        assert t in rows and min(t + 127, 999) in rows
    assert rows[0] == 0 and rows[-1] == 999
    assert np.all(np.diff(rows) > 0)


def test_kernel_bytes_add_up_to_the_pass_totals():
    # the forward kernel's bytes are the forward's; the backward's three kernels
    # read Q, K, V, dO twice (once per recompute kernel) and O once, and write
    # dQ, dK, dV once
    B, H, N, D = 1, 32, 8192, 128
    assert metrics.kernel_bytes("fa_fwd_kernel", B, H, N, N, D) == metrics.fwd_bytes(B, H, N, N, D)
    t = 64 * 2 ** 20                  # one [1, 32, 8192, 128] 16-bit tensor
    rows = 2 ** 20                    # one fp32 value per query row
    assert metrics.kernel_bytes("fa_bwd_pre_kernel", B, H, N, N, D) == 2 * t + rows
    assert metrics.kernel_bytes("fa_bwd_dkdv_kernel", B, H, N, N, D) == 6 * t + 2 * rows
    assert metrics.kernel_bytes("fa_bwd_dq_kernel", B, H, N, N, D) == 5 * t + 2 * rows
    # fp8 inputs, bf16 output
    assert metrics.kernel_bytes("fa_fwd_kernel", B, H, N, N, D, elem=1) == 3 * t // 2 + t + rows
    # split-KV partials: fp32 O_s and LSE_s per split
    assert metrics.kernel_bytes("fa_fwd_split_kernel", 1, 8, 256, 65536, 128, splits=16) == \
        2 * (8 * 256 * 128 + 2 * 8 * 65536 * 128) + 16 * 8 * 256 * (4 * 128 + 4)
    assert metrics.kernel_bytes("fa_unknown_kernel", B, H, N, N, D) is None


def test_roofline_picks_the_binding_bound():
    import bench
    # Llama forward: ~2000 FLOP/byte, far above the ridge (~239) -> tensor
    w = inputs.workload("llama")
    f = metrics.fwd_flops(w["B"], w["H"], w["Nq"], w["Nk"], w["D"], True)
    nb = metrics.kernel_bytes("fa_fwd_kernel", w["B"], w["H"], w["Nq"], w["Nk"], w["D"])
    ms = 0.47
    kd = {"algorithmic_tflops": f / (ms * 1e-3) / 1e12, "algorithmic_gbs": nb / (ms * 1e-3) / 1e9,
          "algorithmic_bytes": nb}
    r = bench.pick_roofline(kd, 1590.0, 6650.0)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["frac"] == pytest.approx(f / (ms * 1e-3) / 1e12 / 1590.0)
    assert r["flop_per_byte"] == pytest.approx(f / nb)
    # sequence sweep at N = 512, causal: ~128 FLOP/byte, below the ridge -> HBM
    w = inputs.workload("sweep", N=512)
    f = metrics.fwd_flops(w["B"], w["H"], w["Nq"], w["Nk"], w["D"], True)
    nb = metrics.kernel_bytes("fa_fwd_kernel", w["B"], w["H"], w["Nq"], w["Nk"], w["D"])
    ms = 0.08
    kd = {"algorithmic_tflops": f / (ms * 1e-3) / 1e12, "algorithmic_gbs": nb / (ms * 1e-3) / 1e9,
          "algorithmic_bytes": nb}
    r = bench.pick_roofline(kd, 1590.0, 6650.0)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6650.0
    assert r["achieved"] == pytest.approx(nb / 0.08e-3 / 1e9)
    assert r["ridge_flop_per_byte"] == pytest.approx(1590e12 / 6650e9)


def test_traffic_records_are_consistent():
    """profiles/traffic.json: every entry names an existing ncu summary and holds
    read + write = bytes_per_launch; the headline's dominant kernel (dK/dV on the
    Llama workload) has a record for the current sources, so the headline bench
    line reports `traffic`."""
    import json
    import os
    import bench
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    t = json.load(open(os.path.join(root, "profiles", "traffic.json")))
    for key, ent in t.items():
        kernel, _, workload = key.partition(":")
        assert kernel in bench.KERNEL_SOURCE and workload, key
        assert ent["read_bytes"] + ent["write_bytes"] == ent["bytes_per_launch"], key
        src = ent["source"].split(" ")[0]
        assert src.startswith("profiles/") and os.path.exists(os.path.join(root, src)), (key, src)
    w = bench.workload_cfg(bench.parse_args([]))
    assert bench.load_traffic("fa_bwd_dkdv_kernel", w) == t["fa_bwd_dkdv_kernel:llama"]["bytes_per_launch"]
