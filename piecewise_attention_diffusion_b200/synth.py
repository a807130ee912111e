"""Seeded synthetic inputs for block-sparse / piecewise attention.

This module only draws random tensors with the shapes and value structure of the
workloads (token layout, smooth spatial fields, noise levels). It holds none of the
attention arithmetic, so both the fp64 oracle and the CUDA path can be fed from it.

All tensors are generated on the CPU as fp32 from ``torch.Generator().manual_seed``
and then rounded to bf16 (round-to-nearest-even). Callers that need the exact
values the GPU sees upcast the bf16 tensors.

Workloads (sizes named after what they are):
  * tiny_pisa          batch 1, 2 heads, L=512, d=64, block 64
  * multimodal_dit     batch 8, 16 heads, L=1152 (77 text tokens padded to 128 +
                       32x32 image patches), d=64, block 64; every position is a
                       real N(0,1) token (no token mask)
  * multimodal_pisa    the same shape and fixed mask as the exact set of PISA
  * multimodal_dit_padded, multimodal_pisa_padded   the same with the 51 pad tokens
                       marked (real tokens per block 64, 13, 64, ...)
  * text_image_pisa    batch 1, 24 heads, L=4352: 77 text tokens padded to a 128-block,
                       a 64x64 latent (32 blocks), a timestep token padded to a
                       128-block; d=128, block 128, routed PISA at 15% density
  * image_pisa_block, video_pisa_block   the per-block first-order form of PISA
  * image_pisa         batch 1, 24 heads, L=4096 (64x64 latent), d=128, block 128
  * video_pisa         batch 1, 40 heads, L=16384 (16 frames x 32x32), d=128, block 128
  * sweep_L{L}         batch 1, 24 heads, L in {4096..32768}, d=128, block 128

Token padding: a workload with ``key_valid`` marks the leading real tokens of each
block; the pad rows of k and v are filled with large noise (4 x N(0,1)) and those of q
with N(0,1), from a generator of their own, so that any leak of a pad key into a result
shows, and the real rows are the same draws as in the unpadded workload.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    seq_len: int
    head_dim: int
    block: int
    mode: str                    # "pisa", "pisa_block" or "keep_or_drop"
    density: float | None = None  # fraction of KV blocks computed exactly (routing)
    k_top: int | None = None      # explicit top-k (overrides density)
    generator: str = "iid"        # iid | block_centres | field2d_hot | field3d
    grid: tuple = ()              # spatial token grid for the field generators
    mask: dict = field(default_factory=dict)  # fixed multimodal mask descriptor
    key_valid: tuple = ()         # real tokens per block (empty: no padding)

    @property
    def n_blocks(self) -> int:
        return self.seq_len // self.block

    def valid_tokens(self) -> list | None:
        """Real tokens per block as a list of M ints, or None without padding."""
        return list(self.key_valid) if self.key_valid else None

    def top_k(self) -> int:
        """Blocks per query block computed exactly: k = max(1, ceil(density*M))."""
        if self.k_top is not None:
            return self.k_top
        m = self.n_blocks
        return max(1, math.ceil(self.density * m - 1e-9))


def workloads() -> dict:
    w = {}
    w["tiny_pisa"] = Workload("tiny_pisa", 1, 2, 512, 64, 64, "pisa", k_top=2,
                              generator="block_centres")
    # 77 text tokens padded to 128 = 2 blocks of 64; 32x32 patches in 8x8 tiles
    # give a 4x4 grid of 64-token image blocks; 3x3 window, image block 0 global.
    w["multimodal_dit"] = Workload(
        "multimodal_dit", 8, 16, 1152, 64, 64, "keep_or_drop", generator="iid",
        mask=dict(n_text_blocks=2, grid_h=4, grid_w=4, radius=1, global_stride=16,
                  global_rows_full=0))
    # the same fixed pattern as the selection of PISA: the blocks it drops enter through
    # the Taylor tail (zeroth order per block, first order through Hbar)
    w["multimodal_pisa"] = dataclasses.replace(w["multimodal_dit"], name="multimodal_pisa",
                                               mode="pisa")
    # 77 text tokens: block 0 full, block 1 with 13 real tokens and 51 pad tokens
    for n in ("multimodal_dit", "multimodal_pisa"):
        w[n + "_padded"] = dataclasses.replace(w[n], name=n + "_padded",
                                               key_valid=(64, 13) + (64,) * 16)
    # text block (77 of 128 real), 32 latent blocks, timestep block (1 of 128 real)
    w["text_image_pisa"] = Workload("text_image_pisa", 1, 24, 4352, 128, 128, "pisa",
                                    density=0.15, generator="block_centres",
                                    key_valid=(77,) + (128,) * 32 + (1,))
    w["image_pisa"] = Workload("image_pisa", 1, 24, 4096, 128, 128, "pisa", density=0.15,
                               generator="field2d_hot", grid=(64, 64))
    w["video_pisa"] = Workload("video_pisa", 1, 40, 16384, 128, 128, "pisa", density=0.125,
                               generator="field3d", grid=(16, 32, 32))
    # the per-block first-order form of PISA (every block a tile: dense tensor work)
    w["image_pisa_block"] = dataclasses.replace(w["image_pisa"], name="image_pisa_block",
                                                mode="pisa_block")
    w["video_pisa_block"] = dataclasses.replace(w["video_pisa"], name="video_pisa_block",
                                                mode="pisa_block")
    for L in (4096, 8192, 16384, 32768):
        for dens in (1.0, 0.25, 0.125):
            for mode in ("keep_or_drop", "pisa"):
                tag = f"sweep_L{L}_d{int(dens * 1000)}_{mode}"
                w[tag] = Workload(tag, 1, 24, L, 128, 128, mode, density=dens,
                                  generator="field3d", grid=(L // 1024, 32, 32))
    return w


def _smooth_field(gen: torch.Generator, dims: tuple, channels: int, n_terms: int = 4,
                  max_freq: int = 2) -> torch.Tensor:
    """Sum of a few low-frequency cosines per channel on a raster-ordered grid.

    f_c(x) = sum_r a_{c,r} cos(2*pi * <omega_{c,r}, x / dims> + phi_{c,r}), integer
    |omega| <= max_freq per axis, phi ~ U[0, 2pi), a ~ N(0,1); each channel is then
    normalised to zero mean and unit variance. Returns [prod(dims), channels] fp32.
    """
    axes = [torch.arange(n, dtype=torch.float32) / n for n in dims]
    mesh = torch.meshgrid(*axes, indexing="ij")
    coords = torch.stack([m.reshape(-1) for m in mesh], dim=1)           # [T, ndim]
    omega = torch.randint(-max_freq, max_freq + 1, (channels, n_terms, len(dims)),
                          generator=gen).to(torch.float32)
    phi = torch.rand(channels, n_terms, generator=gen) * (2 * math.pi)
    amp = torch.randn(channels, n_terms, generator=gen)
    out = torch.zeros(coords.shape[0], channels)
    for r in range(n_terms):
        arg = 2 * math.pi * coords @ omega[:, r, :].T + phi[:, r]        # [T, C]
        out += amp[:, r] * torch.cos(arg)
    out -= out.mean(dim=0, keepdim=True)
    std = out.std(dim=0, keepdim=True)
    out /= torch.where(std > 1e-6, std, torch.ones_like(std))
    return out


def make_qkv(w: Workload, seed: int = 0, heads: list | None = None) -> tuple:
    """Return (q, k, v) bf16 tensors of shape [batch, heads, L, d] on the CPU.

    ``heads`` restricts generation to a subset of (flattened batch*head) indices; the
    values for a head do not depend on which other heads are generated, so a sampled
    oracle run sees exactly the bytes the full GPU run sees.
    """
    BH = w.batch * w.heads
    sel = list(range(BH)) if heads is None else list(heads)
    L, d, B = w.seq_len, w.head_dim, w.block
    qs, ks, vs = [], [], []
    for bh in sel:
        g = torch.Generator().manual_seed(seed * 1_000_003 + bh * 7919 + 17)
        q = torch.randn(L, d, generator=g)
        if w.generator == "iid":
            k = torch.randn(L, d, generator=g)
            v = torch.randn(L, d, generator=g)
        elif w.generator == "block_centres":
            centres = torch.randn(L // B, 1, d, generator=g)
            k = (centres + 0.5 * torch.randn(L // B, B, d, generator=g)).reshape(L, d)
            v = torch.randn(L, d, generator=g)
        elif w.generator == "field2d_hot":
            k = _smooth_field(g, w.grid, d) + 0.3 * torch.randn(L, d, generator=g)
            hot = torch.randperm(L // B, generator=g)[:4]
            kb = k.view(L // B, B, d)
            kb[hot] *= 3.0
            v = _smooth_field(g, w.grid, d) + 0.3 * torch.randn(L, d, generator=g)
        elif w.generator == "field3d":
            k = _smooth_field(g, w.grid, d) + 0.3 * torch.randn(L, d, generator=g)
            v = _smooth_field(g, w.grid, d) + 0.3 * torch.randn(L, d, generator=g)
        else:
            raise ValueError(f"unknown generator {w.generator}")
        if w.key_valid:
            gp = torch.Generator().manual_seed(seed * 1_000_003 + bh * 7919 + 29)
            for j, n in enumerate(w.key_valid):
                if n < B:
                    for x, amp in ((q, 1.0), (k, 4.0), (v, 4.0)):
                        x[j * B + n:(j + 1) * B] = amp * torch.randn(B - n, d, generator=gp)
        qs.append(q)
        ks.append(k)
        vs.append(v)
    shape = (len(sel), L, d) if heads is not None else (w.batch, w.heads, L, d)

    def pack(xs):
        return torch.stack(xs).reshape(shape).to(torch.bfloat16)

    return pack(qs), pack(ks), pack(vs)
