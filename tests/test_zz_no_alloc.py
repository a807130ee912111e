"""bsa_forward_noalloc: the forward entry point for callers that cannot allocate.

Callers that are not allowed to call cudaMalloc (a memory pool that owns the device, a
serving loop that cannot afford cudaMalloc's implicit synchronisation, a runtime with a
fixed memory budget) use bsa_forward_noalloc, whose scratch is a device array built into
the library. These tests call it through the C ABI twice in a row, with different
shapes and modes so that the second call starts from the first call's leftover scratch,
and check each result against bsa_forward (which takes a caller-allocated workspace)
within the parity tolerance. They also check that a shape needing more scratch than the
built-in array is refused before anything is launched, and that keep-or-drop, which needs
only a flag word of scratch, runs on a shape whose PISA scratch would not fit.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle as orc
from piecewise_attention_diffusion_b200 import bsattn as b
from piecewise_attention_diffusion_b200 import synth
from tests._util import assert_close_out, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(workload, heads, mode, seed):
    w = synth.workloads()[workload]
    q, k, v = synth.make_qkv(w, seed=seed, heads=heads)
    q, k, v = (x.reshape(1, len(heads), w.seq_len, w.head_dim).to(DEV) for x in (q, k, v))
    stats = b.precompute(k, v, w.block)
    rp, ci, _ = b.route(q, stats["kbar"], stats["Mnorm"], w.block, w.top_k(), 1.0)
    return w, q, k, v, stats, rp, ci


def _run_both(w, q, k, v, stats, rp, ci, mode):
    st_ref = torch.zeros(1, dtype=torch.int32, device=DEV)
    ref, ref_lse = b.forward(q, k, v, w.block, rp, ci, 1, mode, stats=stats, want_lse=True,
                             status=st_ref)
    O = torch.full_like(q, 3.0)
    lse = torch.full((q.shape[0] * q.shape[1], q.shape[2]), 5.0, dtype=torch.float32,
                     device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    b.bsa_forward_noalloc(q, k, v, w.block, rp, ci, 1, mode, stats["kbar"], stats["vsum"],
                          stats["Hbar"], 0.0, O, lse, st)
    torch.cuda.synchronize()
    assert st_ref.item() == 0 and st.item() == 0
    assert_close_out(O.reshape(-1, w.head_dim), f64(ref).reshape(-1, w.head_dim),
                     f"{w.name} noalloc vs bsa_forward")
    np.testing.assert_allclose(f64(lse), f64(ref_lse), atol=2e-3, rtol=1e-4)
    return O


def test_noalloc_matches_forward_on_two_calls_in_a_row(cuda_ok):
    # call 1: PISA on 4 heads of the video workload (about 0.4 MB of scratch)
    w1 = _case("video_pisa", [0, 1, 2, 3], b.MODE_PISA, 0)
    _run_both(*w1, b.MODE_PISA)
    # call 2: another shape and mode over the scratch the first call left behind
    w2 = _case("tiny_pisa", [0, 1], b.MODE_KEEP_OR_DROP, 7)
    O2 = _run_both(*w2, b.MODE_KEEP_OR_DROP)
    # and the second call's result is also the oracle's
    w, q, k, v, stats, rp, ci = w2
    M = w.n_blocks
    rp_h, ci_h = rp.cpu().numpy(), ci.cpu().numpy()
    for h in range(2):
        hrp, hci = orc.head_csr(rp_h, ci_h, h, M, True)
        qf, kf, vf = (f64(x[0, h]) for x in (q, k, v))
        want, _ = orc.keep_or_drop_head(qf, kf, vf, hrp, hci, w.block, 1 / math.sqrt(w.head_dim))
        assert_close_out(O2[0, h], want, f"oracle head {h}")


def test_noalloc_pisa_after_keep_or_drop(cuda_ok):
    # the reverse order: a small call first, then a PISA call that needs the full scratch
    _run_both(*_case("tiny_pisa", [0, 1], b.MODE_KEEP_OR_DROP, 3), b.MODE_KEEP_OR_DROP)
    _run_both(*_case("image_pisa", [4, 5, 6], b.MODE_PISA, 0), b.MODE_PISA)


def test_noalloc_refuses_shapes_beyond_its_scratch(cuda_ok):
    # PISA on 256 heads of L = 32768, d = 128 needs about 40 MB > 16 MiB. Refused on the
    # host before any pointer is used or any kernel launched.
    p = ctypes.c_void_p(1 << 20)
    rc = b.lib().bsa_forward_noalloc(p, p, p, 1, 256, 32768, 128, 128, None, p, p, 16, 1,
                                     b.MODE_PISA, p, p, p, 0.0, p, None, None, None)
    assert rc == b.ERR_SCRATCH_LIMIT
    assert b.status_string(rc) == "BSA_ERR_SCRATCH_LIMIT"
    need = b.bsa_workspace_bytes(b.CALL_FORWARD, 1, 256, 32768, 128, 128)
    assert need > b.NOALLOC_SCRATCH_BYTES


def test_noalloc_keep_or_drop_runs_where_pisa_scratch_would_not_fit(cuda_ok):
    """1024 heads of L = 256, d = 128: bsa_forward's workspace (the bf16 PISA statistics,
    padded to 128 blocks per head) is about 34 MB, more than the built-in array. In
    keep-or-drop mode bsa_forward_noalloc needs only the flag word and runs, matching
    bsa_forward; the same call in PISA mode is refused with BSA_ERR_SCRATCH_LIMIT."""
    Bt, H, L, d, block = 1, 1024, 256, 128, 128
    assert b.bsa_workspace_bytes(b.CALL_FORWARD, Bt, H, L, d, block) > b.NOALLOC_SCRATCH_BYTES
    g = torch.Generator().manual_seed(12)
    q, k, v = (torch.randn(Bt, H, L, d, generator=g).to(torch.bfloat16).to(DEV)
               for _ in range(3))
    rp = torch.tensor([0, 1, 3], dtype=torch.int32, device=DEV)   # one list for every head
    ci = torch.tensor([1, 0, 1], dtype=torch.int32, device=DEV)
    st_ref = torch.zeros(1, dtype=torch.int32, device=DEV)
    ref, _ = b.forward(q, k, v, block, rp, ci, 0, b.MODE_KEEP_OR_DROP, status=st_ref)
    O = torch.full_like(q, 3.0)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    b.bsa_forward_noalloc(q, k, v, block, rp, ci, 0, b.MODE_KEEP_OR_DROP, None, None, None,
                          0.0, O, None, st)
    torch.cuda.synchronize()
    assert st_ref.item() == 0 and st.item() == 0
    assert_close_out(O.reshape(-1, d), f64(ref).reshape(-1, d), "noalloc vs bsa_forward")
    with pytest.raises(b.BsaError) as e:
        f = torch.zeros(Bt * H, L // block, d, dtype=torch.float32, device=DEV)
        h = torch.zeros(Bt * H, d, d, dtype=torch.float32, device=DEV)
        b.bsa_forward_noalloc(q, k, v, block, rp, ci, 0, b.MODE_PISA, f, f, h, 0.0, O, None, st)
    assert e.value.code == b.ERR_SCRATCH_LIMIT


def test_noalloc_keep_or_drop_with_two_blocks_per_tile(cuda_ok):
    """Block 64: every 128-row tile runs the merged lists of two query blocks, each row
    masking the key blocks its own block does not select. Pairs of rows whose lists
    overlap, nest and are disjoint, per head; bsa_forward_noalloc against bsa_forward and
    against the oracle."""
    Bt, H, L, d, block = 1, 2, 512, 64, 64
    M = L // block
    g = torch.Generator().manual_seed(13)
    q, k, v = (torch.randn(Bt, H, L, d, generator=g).to(torch.bfloat16).to(DEV)
               for _ in range(3))
    lists = [[0, 1, 2], [1, 2, 3],          # overlap
             [0, 2, 4, 6], [2, 4],          # nested
             [0, 1], [5, 7],                # disjoint
             [7], [0, 3, 6, 7]]
    rows = [lists, list(reversed(lists))]   # head 1: the same lists, other pairs
    rp, ci = [], []
    for h in range(H):
        base = h * sum(len(r) for r in rows[h])
        rp.append(np.cumsum([0] + [len(r) for r in rows[h]]) + base)
        ci.extend(c for r in rows[h] for c in sorted(r))
    rp = torch.tensor(np.concatenate(rp), dtype=torch.int32, device=DEV)
    ci = torch.tensor(ci, dtype=torch.int32, device=DEV)
    st_ref = torch.zeros(1, dtype=torch.int32, device=DEV)
    ref, _ = b.forward(q, k, v, block, rp, ci, 1, b.MODE_KEEP_OR_DROP, status=st_ref)
    O = torch.full_like(q, 3.0)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    b.bsa_forward_noalloc(q, k, v, block, rp, ci, 1, b.MODE_KEEP_OR_DROP, None, None, None,
                          0.0, O, None, st)
    torch.cuda.synchronize()
    assert st_ref.item() == 0 and st.item() == 0
    assert_close_out(O.reshape(-1, d), f64(ref).reshape(-1, d), "noalloc vs bsa_forward")
    rp_h, ci_h = rp.cpu().numpy(), ci.cpu().numpy()
    for h in range(H):
        hrp, hci = orc.head_csr(rp_h, ci_h, h, M, 1)
        want, _ = orc.keep_or_drop_head(f64(q[0, h].cpu()), f64(k[0, h].cpu()),
                                        f64(v[0, h].cpu()), hrp, hci, block, 1 / math.sqrt(d))
        assert_close_out(O[0, h], want, f"noalloc block-64 head {h} vs oracle")
