"""The benchmark's accounting (CPU): executed FLOPs, algorithmic bytes and launches per
step, checked against the closed forms they are defined by."""
import math

import bench
from piecewise_attention_diffusion_b200 import synth

W = synth.workloads()


def test_video_forward_flops_closed_form():
    w = W["video_pisa"]
    # 40 heads x 128 query blocks x (16 exact tiles of 4 B^2 d + the Taylor tail
    # B (4 d (M - k) + 2 d^2)), B = d = 128, M = 128, k = 16
    per_block = 16 * 4 * 128 ** 2 * 128 + 128 * (4 * 128 * 112 + 2 * 128 ** 2)
    assert bench.forward_flops(w, 16, "pisa") == 40 * 128 * per_block
    assert math.isclose(bench.forward_flops(w, 16, "pisa") / 1e9, 746.25, rel_tol=1e-4)
    # keep-or-drop drops the tail; the per-block mode computes every block as a tile
    assert bench.forward_flops(w, 16, "keep_or_drop") == 40 * 128 * 16 * 4 * 128 ** 2 * 128
    assert bench.forward_flops(w, 16, "pisa_block") == 40 * 128 * 128 * 4 * 128 ** 2 * 128


def test_fixed_mask_flops_use_the_row_lengths():
    w = W["multimodal_dit"]
    rows = [18, 18] + [11] * 16   # any lengths: the count is their sum
    want = 8 * 16 * sum(rows) * 4 * 64 ** 2 * 64
    assert bench.forward_flops(w, 0, "keep_or_drop", rows) == want


def test_forward_bytes_closed_form():
    w = W["video_pisa"]
    qkvo = 4 * 40 * 16384 * 128 * 2
    stats = 40 * (2 * 128 * 128 + 128 * 128) * 4
    assert bench.forward_bytes(w, "pisa") == qkvo + stats == 678952960
    assert bench.forward_bytes(w, "keep_or_drop") == qkvo


def test_launches_and_steps_per_workload():
    # routed PISA: 3 precompute + 2 route (pooling, scoring) + validation, statistics
    # conversion, forward: the eight kernels of the step's ncu launch list
    assert bench.launches_per_step(W["video_pisa"]) == 8
    assert bench.launches_per_step(W["sweep_L4096_d125_keep_or_drop"]) == 7
    # a fixed keep-or-drop mask needs neither statistics nor routing
    assert not bench.needs_precompute(W["multimodal_dit"])
    assert bench.launches_per_step(W["multimodal_dit"]) == 2
    # PISA over the fixed mask needs the statistics, not the routing
    assert bench.needs_precompute(W["multimodal_pisa"])
    assert bench.launches_per_step(W["multimodal_pisa"]) == 6
    assert bench._steps_done(W["multimodal_dit"]) == "attended"
    assert bench._steps_done(W["video_pisa"]) == "precomputed, routed and attended"


def test_density_to_top_k():
    assert W["video_pisa"].top_k() == 16      # 12.5% of 128
    assert W["image_pisa"].top_k() == 5       # 15% of 32, rounded up
    assert W["sweep_L32768_d125_pisa"].top_k() == 32
    assert W["sweep_L4096_d1000_pisa"].top_k() == 32


def test_l2_rule_per_workload():
    """Inputs that fit twice in L2 (126 MB) are timed with a flush before every step;
    the headline workload's inputs are far larger than L2."""
    assert bench.input_bytes(W["video_pisa"]) == 3 * 40 * 16384 * 128 * 2
    assert not bench.needs_flush(W["video_pisa"])
    assert not bench.needs_flush(W["sweep_L32768_d125_pisa"])
    for small in ("tiny_pisa", "multimodal_dit", "image_pisa", "sweep_L4096_d125_pisa"):
        assert bench.needs_flush(W[small]), small
    assert bench.config_of(W["image_pisa"], 1)["l2"].startswith("L2 flushed")


def test_both_arms_name_the_workload_alike():
    """The reference arm and this arm build their config from one function."""
    for name in ("video_pisa", "multimodal_dit", "text_image_pisa"):
        c = bench.config_of(W[name], 1)
        assert c["workload"] == name and "l2" in c and "lists" in c
    assert set(bench.SWEEP_WORKLOADS) <= set(W)
