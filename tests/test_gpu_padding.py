"""GPU parity with token-level key padding, through the C ABI, against the fp64 oracle.

A DiT packs variable-length text (77 tokens) and a single timestep token into whole
blocks; ``key_valid`` gives each block's leading real tokens. Pad keys must never reach
a softmax, a centroid, a value sum or H_j; pooled queries average real rows only; every
padded block is computed exactly (the routing forces it into every list, and the PISA
forward refuses a list without it). The pad rows of k and v hold large noise, so a leak
shows as a large error rather than a small one.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
from piecewise_attention_diffusion_b200 import bsattn as b
from piecewise_attention_diffusion_b200 import synth
from tests._util import assert_close_out, f64, rows_agree_up_to_ties

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _need_gpu(cuda_ok):
    yield


def _status():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def _kv(valid):
    return torch.tensor(valid, dtype=torch.int32, device=DEV)


def _heads(x, heads):
    """[batch, heads, L, d] -> [len(heads), L, d] for flattened (batch, head) indices."""
    BH = x.shape[0] * x.shape[1]
    return x.reshape(BH, x.shape[2], x.shape[3])[heads]


# d = 64 (the statistics kernel with its head dimension zero-padded to 128) and d = 128; the
# second and the last case carry a one-token (timestep) block
PRE_CASES = [
    ("multimodal_dit_padded", [0, 77, 127]),
    ("text_image_pisa", [0, 9, 23]),
    ("pad64_d128", [0, 1]),
]


def _workload(name):
    if name == "pad64_d128":
        # block 64, d = 128; blocks with 1, 13, 63 and 64 real tokens
        return synth.Workload(name, 1, 2, 512, 128, 64, "pisa", k_top=4,
                              generator="block_centres",
                              key_valid=(64, 13, 64, 64, 1, 64, 63, 64))
    if name == "pad128_d64":
        return synth.Workload(name, 1, 2, 1024, 64, 128, "pisa", k_top=3,
                              generator="block_centres",
                              key_valid=(77, 128, 128, 128, 128, 128, 128, 1))
    return synth.workloads()[name]


@pytest.mark.parametrize("name,heads", PRE_CASES)
def test_precompute_statistics_over_real_tokens(name, heads):
    w = _workload(name)
    q, k, v = synth.make_qkv(w)
    valid = w.valid_tokens()
    st = _status()
    out = b.precompute(k.to(DEV), v.to(DEV), w.block, want_blocks=True, status=st,
                       key_valid=_kv(valid))
    torch.cuda.synchronize()
    assert st.item() == 0, b.status_string(st.item())
    kh, vh = f64(_heads(k, heads)), f64(_heads(v, heads))
    for n, h in enumerate(heads):
        kbar, vsum, H, Hbar, Mn = orc.precompute_head(kh[n], vh[n], w.block, valid)
        np.testing.assert_allclose(f64(out["kbar"][h]), kbar, rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(f64(out["vsum"][h]), vsum, rtol=1e-5, atol=1e-4)
        sH = np.abs(H).max() * math.sqrt(w.block)
        np.testing.assert_allclose(f64(out["Hblk"][h]), H, atol=2e-5 * sH)
        np.testing.assert_allclose(f64(out["Hbar"][h]), Hbar, atol=2e-5 * sH)
        np.testing.assert_allclose(f64(out["Mnorm"][h]), Mn, rtol=1e-4, atol=1e-4 * Mn.max())


@pytest.mark.parametrize("name,heads", [("text_image_pisa", [0, 9, 23]),
                                        ("pad64_d128", [0, 1]), ("pad128_d64", [0, 1])])
def test_route_pools_real_queries_and_forces_padded_blocks(name, heads):
    w = _workload(name)
    q, k, v = synth.make_qkv(w)
    valid = w.valid_tokens()
    M, kk = w.n_blocks, w.top_k()
    forced = [j for j in range(M) if valid[j] < w.block]
    scale = 1 / math.sqrt(w.head_dim)
    qh, kh, vh = (f64(_heads(x, heads)) for x in (q, k, v))
    stats = [orc.precompute_head(kh[n], vh[n], w.block, valid) for n in range(len(heads))]
    kbar = np.stack([s_[0] for s_ in stats])
    Mn = np.stack([s_[4] for s_ in stats])
    st = _status()
    qd = _heads(q, heads).reshape(1, len(heads), w.seq_len, w.head_dim).to(DEV)
    rp, ci, sc = b.route(qd, torch.from_numpy(kbar).float().to(DEV),
                         torch.from_numpy(Mn).float().to(DEV), w.block, kk, 1.0, 0.0,
                         want_scores=True, status=st, key_valid=_kv(valid))
    torch.cuda.synchronize()
    assert st.item() == 0, b.status_string(st.item())
    gci = ci.cpu().numpy().reshape(len(heads), M, kk)
    for n in range(len(heads)):
        orp, oci, osc = orc.route_head(qh[n], kbar[n], Mn[n], w.block, kk, 1.0, scale, valid)
        np.testing.assert_allclose(f64(sc[n]), osc, rtol=2e-4, atol=1e-6)
        for i in range(M):
            g = gci[n, i]
            assert (np.diff(g) > 0).all()
            assert set(forced) <= set(g.tolist()), (n, i, g)
            assert rows_agree_up_to_ties(g, oci[i * kk:(i + 1) * kk], osc[i], kk, forced), \
                (n, i, g)


@pytest.mark.parametrize("name", ["text_image_pisa", "pad64_d128", "pad128_d64"])
@pytest.mark.parametrize("mode", [b.MODE_KEEP_OR_DROP, b.MODE_PISA, b.MODE_PISA_BLOCK])
def test_forward_masks_pad_keys(name, mode):
    """Oracle lists and statistics (so the forward alone is checked); padded query rows
    are compared too: they attend like any other row."""
    w = _workload(name)
    q, k, v = synth.make_qkv(w, seed=2)
    valid = w.valid_tokens()
    M, kk, BH = w.n_blocks, w.top_k(), w.batch * w.heads
    heads = [0, BH - 1]
    scale = 1 / math.sqrt(w.head_dim)
    kf, vf, qf = (f64(x).reshape(BH, w.seq_len, w.head_dim) for x in (k, v, q))
    pre = [orc.precompute_head(kf[h], vf[h], w.block, valid) for h in range(BH)]
    kbar, vsum, H, Hbar, Mn = (np.stack([p_[n] for p_ in pre]) for n in range(5))
    rp, ci, _ = orc.route(f64(q), kbar, Mn, w.block, kk, 1.0, scale, valid)
    grp = torch.from_numpy(rp).to(DEV)
    gci = torch.from_numpy(ci).to(DEV)
    f = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(DEV, torch.float32)
    stats = dict(kbar=f(kbar), vsum=f(vsum), Hbar=f(Hbar)) if mode == b.MODE_PISA else None
    st = _status()
    O, lse = b.forward(q.to(DEV), k.to(DEV), v.to(DEV), w.block, grp, gci, 1, mode,
                       stats=stats, want_lse=True, status=st, key_valid=_kv(valid))
    torch.cuda.synchronize()
    assert st.item() == 0, b.status_string(st.item())
    Og = O.reshape(BH, w.seq_len, w.head_dim)
    lg = f64(lse.reshape(BH, w.seq_len))
    for h in heads:
        hrp, hci = orc.head_csr(rp, ci, h, M, 1)
        if mode == b.MODE_KEEP_OR_DROP:
            want, wl = orc.keep_or_drop_head(qf[h], kf[h], vf[h], hrp, hci, w.block, scale,
                                             key_valid=valid)
        else:
            want, wl = orc.pisa_head(qf[h], kf[h], vf[h], hrp, hci, w.block, scale, kbar[h],
                                     vsum[h], Hbar[h], key_valid=valid,
                                     Hblocks=H[h] if mode == b.MODE_PISA_BLOCK else None)
        mx, rl = assert_close_out(Og[h], want, f"{name} mode {mode} head {h}")
        print(f"[padding] {name} mode={mode} head {h} max-abs {mx:.2e} rel-L2 {rl:.2e}")
        tol = 2e-3
        if mode == b.MODE_PISA:
            # centroid scores use kbar rounded to bf16 (unit roundoff 2^-8)
            tol = tol + (scale * np.abs(qf[h]) @ np.abs(kbar[h]).T * 2.0 ** -8).max(axis=1)
        assert (np.abs(lg[h] - wl) <= tol).all()


def test_forward_pisa_over_the_padded_multimodal_mask_per_block_mode():
    """The fixed multimodal pattern (text blocks in every row, so the padded text block
    is exact everywhere) with the per-block first-order tail."""
    w = synth.workloads()["multimodal_pisa_padded"]
    q, k, v = synth.make_qkv(w, seed=1)
    valid = w.valid_tokens()
    keep = orc.mask_dense(**w.mask)
    rp, ci = orc.dense_to_csr(keep)
    BH = w.batch * w.heads
    heads = [3, 100]
    scale = 1 / math.sqrt(w.head_dim)
    kf, vf, qf = (f64(x).reshape(BH, w.seq_len, w.head_dim) for x in (k, v, q))
    st = _status()
    O, _ = b.forward(q.to(DEV), k.to(DEV), v.to(DEV), w.block, torch.from_numpy(rp).to(DEV),
                     torch.from_numpy(ci).to(DEV), 0, b.MODE_PISA_BLOCK, status=st,
                     key_valid=_kv(valid))
    torch.cuda.synchronize()
    assert st.item() == 0, b.status_string(st.item())
    Og = O.reshape(BH, w.seq_len, w.head_dim)
    for h in heads:
        kbar, vsum, H, Hbar, _ = orc.precompute_head(kf[h], vf[h], w.block, valid)
        want, _ = orc.pisa_head(qf[h], kf[h], vf[h], rp, ci, w.block, scale, kbar, vsum, Hbar,
                                Hblocks=H, key_valid=valid)
        assert_close_out(Og[h], want, f"multimodal per-block head {h}")


def test_all_real_counts_equal_no_padding():
    """key_valid filled with B gives the same bytes as no key_valid, in every call."""
    w = synth.Workload("full_counts", 1, 2, 1024, 128, 128, "pisa", k_top=3,
                       generator="block_centres")
    q, k, v = (x.to(DEV) for x in synth.make_qkv(w, seed=6))
    kv = _kv([w.block] * w.n_blocks)
    res = []
    for key_valid in (None, kv):
        st = _status()
        s_ = b.precompute(k, v, w.block, status=st, key_valid=key_valid)
        rp, ci, _ = b.route(q, s_["kbar"], s_["Mnorm"], w.block, 3, 1.0, status=st,
                            key_valid=key_valid)
        O, lse = b.forward(q, k, v, w.block, rp, ci, 1, b.MODE_PISA, stats=s_, want_lse=True,
                           status=st, key_valid=key_valid)
        torch.cuda.synchronize()
        assert st.item() == 0
        res.append((s_["kbar"], s_["Hbar"], ci, O, lse))
    for a, c in zip(*res):
        assert torch.equal(a, c)


# ------------------------------------------------------------------------- errors
def test_pisa_forward_reports_a_list_without_a_padded_block():
    w = _workload("pad64_d128")
    q, k, v = (x.to(DEV) for x in synth.make_qkv(w))
    M = w.n_blocks
    # every row keeps blocks 0 and 2 only: the padded blocks 1, 4 and 6 are missing
    rp = torch.arange(M + 1, dtype=torch.int32, device=DEV) * 2
    ci = torch.tensor([0, 2] * M, dtype=torch.int32, device=DEV)
    f32 = dict(dtype=torch.float32, device=DEV)
    stats = dict(kbar=torch.zeros(2, M, w.head_dim, **f32),
                 vsum=torch.zeros(2, M, w.head_dim, **f32),
                 Hbar=torch.zeros(2, w.head_dim, w.head_dim, **f32))
    for mode, st_ in ((b.MODE_PISA, stats), (b.MODE_PISA_BLOCK, None)):
        st = _status()
        O = torch.full_like(q, 7.0)
        b.forward(q, k, v, w.block, rp, ci, 0, mode, stats=st_, status=st, out=O,
                  key_valid=_kv(w.valid_tokens()))
        torch.cuda.synchronize()
        assert st.item() == b.ERR_BAD_PADDING, b.status_string(st.item())
        assert (O == 7.0).all()
    # keep-or-drop accepts the same lists: dropping a padded block is its choice
    st = _status()
    b.forward(q, k, v, w.block, rp, ci, 0, b.MODE_KEEP_OR_DROP, status=st,
              key_valid=_kv(w.valid_tokens()))
    torch.cuda.synchronize()
    assert st.item() == 0


def test_route_reports_more_padded_blocks_than_k_top():
    w = _workload("pad64_d128")     # three padded blocks
    q, k, v = (x.to(DEV) for x in synth.make_qkv(w))
    kv = _kv(w.valid_tokens())
    st = _status()
    s_ = b.precompute(k, v, w.block, status=st, key_valid=kv)
    torch.cuda.synchronize()
    assert st.item() == 0
    rp, ci, _ = b.route(q, s_["kbar"], s_["Mnorm"], w.block, 2, 1.0, status=st, key_valid=kv)
    torch.cuda.synchronize()
    assert st.item() == b.ERR_BAD_PADDING
    # the lists are still well formed: ascending, in range
    g = ci.cpu().numpy().reshape(-1, 2)
    assert (np.diff(g, axis=1) > 0).all() and (g >= 0).all() and (g < w.n_blocks).all()


@pytest.mark.parametrize("bad", [0, -3, 65])
def test_out_of_range_counts_report_bad_padding(bad):
    w = _workload("pad64_d128")
    q, k, v = (x.to(DEV) for x in synth.make_qkv(w))
    valid = list(w.valid_tokens())
    valid[3] = bad
    kv = _kv(valid)
    st = _status()
    s_ = b.precompute(k, v, w.block, status=st, key_valid=kv)
    torch.cuda.synchronize()
    assert st.item() == b.ERR_BAD_PADDING
    st = _status()
    b.route(q, s_["kbar"], s_["Mnorm"], w.block, 5, 1.0, status=st, key_valid=kv)
    torch.cuda.synchronize()
    assert st.item() == b.ERR_BAD_PADDING
