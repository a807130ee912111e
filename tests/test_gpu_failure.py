"""Failure detection on the GPU without a fault: every wait in the library's kernels is
bounded; a wait that runs out makes the kernel report BSA_ERR_TIMEOUT and return, and
the context stays usable. One self-test kernel waits on an mbarrier that nothing
completes, with a short limit; the other runs the attention kernel itself with its waits
limited to a few ns, which drives its abort, drain and TMEM-release path."""
import math
import time

import numpy as np
import pytest
import torch

import oracle as orc
from piecewise_attention_diffusion_b200 import bsattn as b
from piecewise_attention_diffusion_b200 import synth
from tests._util import assert_close_out, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu(cuda_ok):
    yield


def test_bounded_wait_runs_out_reports_timeout_and_the_context_stays_usable():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    b.bsa_selftest_wait_timeout(50_000_000, st)   # 50 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert st.item() == b.ERR_TIMEOUT
    assert 0.04 < elapsed < 5.0
    # the same context then runs the path and matches the oracle
    w = synth.workloads()["tiny_pisa"]
    q, k, v = synth.make_qkv(w)
    M = w.n_blocks
    rp = np.arange(0, M * 2 + 1, 2, dtype=np.int32)
    ci = np.tile(np.array([0, 3], dtype=np.int32), M)
    st.zero_()
    O, _ = b.forward(q.cuda(), k.cuda(), v.cuda(), w.block,
                     torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda(), 0,
                     b.MODE_KEEP_OR_DROP, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    for h in range(w.heads):
        want, _ = orc.keep_or_drop_head(f64(q[0, h]), f64(k[0, h]), f64(v[0, h]), rp, ci,
                                        w.block, 1 / math.sqrt(w.head_dim))
        assert_close_out(O[0, h], want, f"head {h}")


def test_selftest_rejects_bad_arguments():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(b.BsaError):
        b.bsa_selftest_wait_timeout(0, st)
    with pytest.raises(b.BsaError):
        b.bsa_selftest_wait_timeout(20_000_000_000, st)


@pytest.mark.parametrize("d,block", [(128, 128), (64, 64)])
@pytest.mark.parametrize("mode", [b.MODE_KEEP_OR_DROP, b.MODE_PISA])
def test_forward_abort_path_drains_frees_tmem_and_reports_timeout(mode, d, block):
    """The attention kernel itself, with every bounded wait limited to a few ns: a wait
    runs out while TMA copies and MMAs are in flight, and the kernel's own abort path runs
    (abort flag, producer drains its copies, the MMA thread waits for its issued MMAs, TMEM
    freed). The call reports BSA_ERR_TIMEOUT; then, on the same context, the normal
    forward matches the oracle. Limits of 1 us and 20 us end the same way or complete.
    Head dim 128 runs the single-warpgroup kernel; head dim 64 (blocks of 64, two to a
    step) the kernel whose row softmax is split between two warpgroups, which agree on
    leaving through their named barrier."""
    w = synth.Workload("abort", 1, 8, 8192, d, block, "pisa", k_top=64, generator="iid")
    q, k, v = synth.make_qkv(w, seed=21)
    BH, M = w.batch * w.heads, w.n_blocks
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ci = torch.arange(M, dtype=torch.int32, device="cuda").repeat(BH * M)
    # every head's row_ptr holds M + 1 absolute offsets
    rp = torch.cat([torch.arange(h * M * M, (h + 1) * M * M + 1, M, dtype=torch.int32,
                                 device="cuda") for h in range(BH)])
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    stats = b.precompute(kd, vd, w.block, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ws = b.workspace(b.CALL_FORWARD, w.batch, w.heads, w.seq_len, w.head_dim, w.block)
    O = torch.empty_like(qd)
    for wait_ns in (1, 1_000, 20_000):
        st.zero_()
        t0 = time.perf_counter()
        b.bsa_selftest_forward_timeout(qd, kd, vd, w.block, rp, ci, mode, stats["kbar"],
                                       stats["vsum"], stats["Hbar"], O, ws, wait_ns, st)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
        code = st.item()
        print(f"[abort] mode={mode} d={d} wait_ns={wait_ns} status={b.status_string(code)} "
              f"{elapsed * 1e3:.2f} ms")
        assert elapsed < 5.0
        if wait_ns == 1:
            assert code == b.ERR_TIMEOUT
        else:
            assert code in (b.OK, b.ERR_TIMEOUT)
    # the same context runs the normal forward correctly
    st.zero_()
    O, _ = b.forward(qd, kd, vd, w.block, rp, ci, 1, mode,
                     stats=stats if mode == b.MODE_PISA else None, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    scale = 1 / math.sqrt(w.head_dim)
    rp_h, ci_h = rp.cpu().numpy(), ci.cpu().numpy()
    blocks = [0, 31, M - 1]
    rows = np.concatenate([np.arange(i * w.block, (i + 1) * w.block) for i in blocks])
    for h in (0, BH - 1):
        hrp, hci = orc.head_csr(rp_h, ci_h, h, M, 1)
        qf, kf, vf = f64(q[0, h]), f64(k[0, h]), f64(v[0, h])
        if mode == b.MODE_PISA:
            kbar, vsum, _, Hbar, _ = orc.precompute_head(kf, vf, w.block)
            want, _ = orc.pisa_head(qf, kf, vf, hrp, hci, w.block, scale, kbar, vsum, Hbar,
                                    qblocks=blocks)
        else:
            want, _ = orc.keep_or_drop_head(qf, kf, vf, hrp, hci, w.block, scale, qblocks=blocks)
        assert_close_out(O[0, h, rows], want, f"head {h}")


def test_forward_selftest_rejects_bad_arguments():
    w = synth.workloads()["tiny_pisa"]
    q, k, v = (x.cuda() for x in synth.make_qkv(w))
    M = w.n_blocks
    rp = torch.cat([torch.arange(h * M * M, (h + 1) * M * M + 1, M, dtype=torch.int32,
                                 device="cuda") for h in range(2)])
    ci = torch.arange(M, dtype=torch.int32, device="cuda").repeat(2 * M)
    ws = b.workspace(b.CALL_FORWARD, 1, 2, w.seq_len, w.head_dim, w.block)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    O = torch.empty_like(q)
    for bad in (0, 20_000_000_000):
        with pytest.raises(b.BsaError):
            b.bsa_selftest_forward_timeout(q, k, v, w.block, rp, ci, b.MODE_KEEP_OR_DROP, None,
                                           None, None, O, ws, bad, st)
