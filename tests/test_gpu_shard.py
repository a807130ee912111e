"""Head shards on one GPU: what each rank of a head-sharded run computes is what the
whole run computes for those heads. Each shard is run here in turn, as the rank owning it
would run it (no kernels wait on one another).

Per block the statistics are the same bits (one CTA computes a block whatever the grid);
H-bar and M_j sum over blocks in an order set by the grid, so they agree to rounding; with
the whole run's statistics and block lists, routing and the forward of a shard are
bit-identical to the whole run's rows of those heads."""
import dataclasses
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from piecewise_attention_diffusion_b200 import bsattn as b, synth  # noqa: E402
from piecewise_attention_diffusion_b200.shard import head_range, shard_of  # noqa: E402

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("name,batch,heads,world", [("image_pisa", 1, 24, 3),
                                                    ("image_pisa", 2, 5, 3),
                                                    ("tiny_pisa", 1, 2, 2)])
def test_head_shards_compute_the_whole_runs_heads(name, batch, heads, world):
    w = dataclasses.replace(synth.workloads()[name], batch=batch, heads=heads)
    BH, M, L, d, kk = batch * heads, w.n_blocks, w.seq_len, w.head_dim, w.top_k()
    qd, kd, vd = (x.to(DEV) for x in synth.make_qkv(w))
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    stats = b.precompute(kd, vd, w.block, status=st)
    rp, ci, _ = b.route(qd, stats["kbar"], stats["Mnorm"], w.block, kk, 1.0, status=st)
    O, _ = b.forward(qd, kd, vd, w.block, rp, ci, 1, b.MODE_PISA, stats=stats, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    Of = O.reshape(BH, L, d)
    for r in range(world):
        h0, h1 = head_range(BH, world, r)
        qs, ks, vs = (shard_of(x, world, r) for x in (qd, kd, vd))
        # the shard's own statistics
        own = b.precompute(ks, vs, w.block, status=st)
        sub = {key: stats[key][h0:h1] for key in ("kbar", "vsum", "Hbar", "Mnorm")}
        torch.cuda.synchronize()
        assert torch.equal(own["kbar"], sub["kbar"]) and torch.equal(own["vsum"], sub["vsum"])
        hmax = sub["Hbar"].abs().max().item()
        torch.testing.assert_close(own["Hbar"], sub["Hbar"], rtol=1e-5, atol=1e-6 * hmax)
        torch.testing.assert_close(own["Mnorm"], sub["Mnorm"], rtol=1e-5, atol=0.0)
        # routing and the forward on the whole run's statistics and lists
        srp, sci, _ = b.route(qs, sub["kbar"], sub["Mnorm"], w.block, kk, 1.0, status=st)
        assert torch.equal(srp, rp[h0 * (M + 1):h1 * (M + 1)] - h0 * M * kk)
        assert torch.equal(sci, ci[h0 * M * kk:h1 * M * kk])
        Os, _ = b.forward(qs, ks, vs, w.block, srp, sci, 1, b.MODE_PISA, stats=sub, status=st)
        torch.cuda.synchronize()
        assert st.item() == 0
        assert torch.equal(Os.reshape(h1 - h0, L, d), Of[h0:h1]), (name, r)
