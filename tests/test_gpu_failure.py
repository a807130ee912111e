"""Failure detection on the GPU without a fault: every wait in the library's kernels is
bounded; a wait that runs out makes the kernel report BSA_ERR_TIMEOUT and return, and
the context stays usable. The self-test kernel waits on an mbarrier that nothing
completes, with a short limit."""
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
