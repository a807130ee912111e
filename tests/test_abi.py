"""CPU checks of the C ABI: the library loads, exports every symbol the header
declares, and its host-side validation rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

from piecewise_attention_diffusion_b200 import bsattn as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "bsattn.h")) as f:
        src = f.read()
    return re.findall(r"BSA_API\s+[\w\s\*]+?\b(bsa_\w+)\s*\(", src)


def test_header_declarations_match_binding():
    assert tuple(_declared()) == b.EXPORTS


def test_library_exports_every_declared_symbol():
    so = ctypes.CDLL(b.LIB_PATH)
    for name in _declared():
        assert hasattr(so, name), name


def test_header_status_and_mode_values_match_binding():
    with open(os.path.join(ROOT, "include", "bsattn.h")) as f:
        src = f.read()
    codes = dict((n, int(v)) for n, v in re.findall(r"\b(BSA_(?:OK|ERR_\w+))\s*=\s*(\d+)", src))
    assert codes == {"BSA_OK": b.OK, "BSA_ERR_INVALID_ARG": b.ERR_INVALID_ARG,
                     "BSA_ERR_UNSUPPORTED": b.ERR_UNSUPPORTED, "BSA_ERR_CUDA": b.ERR_CUDA,
                     "BSA_ERR_BAD_CSR": b.ERR_BAD_CSR, "BSA_ERR_TIMEOUT": b.ERR_TIMEOUT,
                     "BSA_ERR_WORKSPACE": b.ERR_WORKSPACE, "BSA_ERR_CAPACITY": b.ERR_CAPACITY,
                     "BSA_ERR_SCRATCH_LIMIT": b.ERR_SCRATCH_LIMIT,
                     "BSA_ERR_BAD_PADDING": b.ERR_BAD_PADDING}
    modes = dict((n, int(v)) for n, v in re.findall(r"\b(BSA_MODE_\w+)\s*=\s*(\d+)", src))
    assert modes == {"BSA_MODE_KEEP_OR_DROP": b.MODE_KEEP_OR_DROP, "BSA_MODE_PISA": b.MODE_PISA,
                     "BSA_MODE_PISA_BLOCK": b.MODE_PISA_BLOCK}
    for code in codes.values():
        assert b.status_string(code) != "BSA_UNKNOWN_STATUS"


def test_status_strings_and_version():
    assert b.bsa_version() >= 100
    assert b.status_string(b.OK) == "BSA_OK"
    assert b.status_string(b.ERR_BAD_CSR) == "BSA_ERR_BAD_CSR"
    assert b.status_string(99) == "BSA_UNKNOWN_STATUS"


def test_mask_blocks_and_invalid_descriptors():
    assert b.bsa_mask_blocks(dict(n_text_blocks=2, grid_h=4, grid_w=4, radius=1,
                                  global_stride=16)) == 18
    assert b.bsa_mask_blocks(dict(n_text_blocks=1, grid_h=1, grid_w=8, radius=2,
                                  global_stride=4)) == 9
    assert b.bsa_mask_blocks(dict(n_text_blocks=-1, grid_h=1, grid_w=8, radius=2,
                                  global_stride=4)) == -1
    assert b.bsa_mask_blocks(dict(n_text_blocks=1, grid_h=0, grid_w=8, radius=2,
                                  global_stride=4)) == -1
    assert b.bsa_mask_blocks(dict(n_text_blocks=0, grid_h=64, grid_w=64, radius=1,
                                  global_stride=0)) == -1      # M > 2048


def test_workspace_sizes():
    # routing: one fp32 column sum of d per 32-row segment of Q
    assert b.bsa_workspace_bytes(b.CALL_ROUTE, 1, 40, 16384, 128, 128) == 40 * 512 * 128 * 4
    assert b.bsa_workspace_bytes(b.CALL_ROUTE, 8, 16, 1152, 64, 64) == 128 * 36 * 64 * 4
    assert b.bsa_workspace_bytes(b.CALL_PRECOMPUTE, 1, 40, 16384, 128, 128) > 0
    assert b.bsa_workspace_bytes(b.CALL_FORWARD, 1, 40, 16384, 128, 128) > 0
    assert b.bsa_workspace_bytes(b.CALL_FORWARD, 1, 4, 1000, 128, 128) == 0   # L % block
    assert b.bsa_workspace_bytes(b.CALL_FORWARD, 1, 4, 1024, 96, 128) == 0    # d


def _fake(n=1 << 20):
    # A 16-byte aligned host address; validation rejects the calls below before any
    # pointer is dereferenced or any CUDA call is made.
    return ctypes.c_void_p(1 << 20)


@pytest.mark.parametrize("d,block,L,want", [
    (96, 128, 1024, b.ERR_UNSUPPORTED), (128, 32, 1024, b.ERR_UNSUPPORTED),
    (128, 128, 1000, b.ERR_UNSUPPORTED), (128, 128, 0, b.ERR_INVALID_ARG),
    (64, 64, 64 * 4096, b.ERR_UNSUPPORTED)])
def test_forward_rejects_unsupported_shapes(d, block, L, want):
    p = _fake()
    rc = b.lib().bsa_forward(p, p, p, 1, 2, L, d, block, None, p, p, 8, 0, 0, None, None, None,
                             0.0, p, None, p, 1 << 20, None, None)
    assert rc == want


def test_forward_rejects_bad_arguments():
    p = _fake()
    mis = ctypes.c_void_p((1 << 20) + 2)
    f = b.lib().bsa_forward
    common = (1, 2, 256, 64, 64)
    # misaligned Q
    assert f(mis, p, p, *common, None, p, p, 8, 0, 0, None, None, None, 0.0, p, None, p, 1 << 20,
             None, None) == b.ERR_INVALID_ARG
    # PISA without statistics
    assert f(p, p, p, *common, None, p, p, 8, 0, 1, None, None, None, 0.0, p, None, p, 1 << 20,
             None, None) == b.ERR_INVALID_ARG
    # bad mode / csr flag / negative scale / negative nnz
    assert f(p, p, p, *common, None, p, p, 8, 0, 7, None, None, None, 0.0, p, None, p, 1 << 20,
             None, None) == b.ERR_INVALID_ARG
    assert f(p, p, p, *common, None, p, p, 8, 3, 0, None, None, None, 0.0, p, None, p, 1 << 20,
             None, None) == b.ERR_INVALID_ARG
    assert f(p, p, p, *common, None, p, p, 8, 0, 0, None, None, None, -1.0, p, None, p, 1 << 20,
             None, None) == b.ERR_INVALID_ARG
    assert f(p, p, p, *common, None, p, p, -1, 0, 0, None, None, None, 0.0, p, None, p, 1 << 20,
             None, None) == b.ERR_INVALID_ARG
    # missing / short workspace
    assert f(p, p, p, *common, None, p, p, 8, 0, 0, None, None, None, 0.0, p, None, None, 0,
             None, None) == b.ERR_WORKSPACE
    assert f(p, p, p, *common, None, p, p, 8, 0, 0, None, None, None, 0.0, p, None, p, 8,
             None, None) == b.ERR_WORKSPACE


def test_route_and_precompute_reject_bad_arguments():
    p = _fake()
    r = b.lib().bsa_route
    assert r(p, p, p, 1, 2, 512, 64, 64, None, 0, 1.0, 0.0, p, p, None, p, 1 << 20, None, None) == \
        b.ERR_INVALID_ARG                                      # k_top 0
    assert r(p, p, p, 1, 2, 512, 64, 64, None, 9, 1.0, 0.0, p, p, None, p, 1 << 20, None, None) == \
        b.ERR_INVALID_ARG                                      # k_top > M
    assert r(p, p, p, 1, 2, 512, 64, 64, None, 2, -1.0, 0.0, p, p, None, p, 1 << 20, None, None) == \
        b.ERR_INVALID_ARG                                      # lambda < 0
    assert r(p, p, p, 1, 2, 512, 64, 64, None, 2, 1.0, 0.0, p, p, None, p, 64, None, None) == \
        b.ERR_WORKSPACE                                        # workspace too small
    assert r(p, p, p, 1, 2, 512, 64, 64, None, 2, 1.0, 0.0, p, p, None, None, 0, None, None) == \
        b.ERR_WORKSPACE                                        # no workspace
    odd = ctypes.c_void_p((1 << 20) + 2)                       # key_valid not 4-aligned
    assert r(p, p, p, 1, 2, 512, 64, 64, odd, 2, 1.0, 0.0, p, p, None, p, 1 << 20, None, None) == \
        b.ERR_INVALID_ARG
    pc = b.lib().bsa_precompute
    assert pc(p, p, 1, 2, 512, 64, 64, None, p, p, p, p, None, None, 0, None, None) == \
        b.ERR_WORKSPACE
    assert pc(p, None, 1, 2, 512, 64, 64, None, p, p, p, p, None, p, 1 << 30, None, None) == \
        b.ERR_INVALID_ARG
    assert pc(p, p, 1, 2, 512, 64, 64, odd, p, p, p, p, None, p, 1 << 30, None, None) == \
        b.ERR_INVALID_ARG


def test_noalloc_rejects_misaligned_key_valid():
    p = _fake()
    odd = ctypes.c_void_p((1 << 20) + 2)
    rc = b.lib().bsa_forward_noalloc(p, p, p, 1, 2, 512, 64, 64, odd, p, p, 16, 0, 0, None, None,
                                     None, 0.0, p, None, None, None)
    assert rc == b.ERR_INVALID_ARG


def test_build_mask_rejects_bad_arguments():
    d = b.MaskDesc(2, 4, 4, 1, 16, 0)
    p = _fake()
    assert b.lib().bsa_build_mask(ctypes.byref(d), None, p, 324, None, None) == \
        b.ERR_INVALID_ARG
    bad = b.MaskDesc(2, 4, 0, 1, 16, 0)
    assert b.lib().bsa_build_mask(ctypes.byref(bad), p, p, 324, None, None) == \
        b.ERR_INVALID_ARG


def test_binding_refuses_host_tensors():
    """There is no CPU path: every wrapper refuses tensors that are not on a CUDA device
    before anything is launched."""
    import torch
    q = torch.zeros(1, 2, 256, 64, dtype=torch.bfloat16)
    f32 = dict(dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        b.forward(q, q, q, 64, torch.zeros(5, dtype=torch.int32),
                  torch.zeros(8, dtype=torch.int32), 0, b.MODE_KEEP_OR_DROP, ws=q)
    with pytest.raises(ValueError, match="CUDA"):
        b.bsa_route(q, torch.zeros(2, 4, 64, **f32), torch.zeros(2, 4, **f32), 64, 2, 1.0, 0.0,
                    torch.zeros(10, dtype=torch.int32), torch.zeros(16, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA"):
        b.bsa_precompute(q, q, 64, torch.zeros(2, 4, 64, **f32), torch.zeros(2, 4, 64, **f32),
                         torch.zeros(2, 64, 64, **f32), torch.zeros(2, 4, **f32))
