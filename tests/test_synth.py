"""The seeded input generators (CPU): determinism, head independence, and the padded
workloads' layout (real rows identical to the unpadded draw, pad rows replaced)."""
import dataclasses

import torch

from piecewise_attention_diffusion_b200 import synth


def test_same_seed_same_bytes_and_heads_are_independent():
    w = synth.workloads()["tiny_pisa"]
    a = synth.make_qkv(w, seed=3)
    b = synth.make_qkv(w, seed=3)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    # a sampled head holds exactly the bytes the full draw has for it
    one = synth.make_qkv(w, seed=3, heads=[1])
    for full, part in zip(a, one):
        assert torch.equal(full.reshape(2, w.seq_len, w.head_dim)[1], part[0])


def test_padding_replaces_only_the_pad_rows():
    w = synth.workloads()["multimodal_dit_padded"]
    small = dataclasses.replace(w, batch=1, heads=2)
    plain = dataclasses.replace(small, key_valid=())
    pq, pk, pv = synth.make_qkv(small, seed=0)
    uq, uk, uv = synth.make_qkv(plain, seed=0)
    B = w.block
    valid = small.valid_tokens()
    assert valid[:2] == [64, 13] and sum(valid) == 77 + 1024
    for got, ref in ((pq, uq), (pk, uk), (pv, uv)):
        for j, n in enumerate(valid):
            rows = slice(j * B, j * B + n)
            assert torch.equal(got[..., rows, :], ref[..., rows, :])
            if n < B:
                pad = slice(j * B + n, (j + 1) * B)
                assert not torch.equal(got[..., pad, :], ref[..., pad, :])


def test_text_image_workload_layout():
    w = synth.workloads()["text_image_pisa"]
    v = w.valid_tokens()
    assert len(v) == w.n_blocks == 34
    assert v[0] == 77 and v[-1] == 1 and all(n == 128 for n in v[1:-1])
    assert w.top_k() == 6      # ceil(0.15 * 34)
