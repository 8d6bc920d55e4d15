"""mdr_route_noalloc: the route step for callers that cannot allocate device
memory (their memory is all reserved by their own pool, or their plugin
interface passes only inputs and outputs).  It must give exactly what
mdr_route gives, call after call, although every call reuses the same
built-in scratch array.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

from tests import parity_util as U
from workloads import AR, SCALING_32K, scaling, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _reference_route(w, inp):
    """Index and route through the existing entry points (with a workspace)."""
    import torch
    from learned_product_hash_b200 import mdr
    cfg = mdr.make_config(w)
    q, k, v, cb = U.to_device(inp, w)
    idx = mdr.Index.empty(cfg)
    ws = mdr.workspace(cfg)
    mdr.mdr_build_index(cfg, k, cb, idx, ws)
    rt = mdr.RouteOut.empty(cfg, debug=True)
    mdr.mdr_route(cfg, q, cb, idx, rt, ws)
    torch.cuda.synchronize()
    return cfg, q, cb, idx, rt


def test_noalloc_route_matches_route_on_consecutive_calls():
    import torch
    from learned_product_hash_b200 import mdr
    # two different problems back to back: stale scratch from the first call
    # must not leak into the second
    for w, seed in [(scaling(4096), 0), (AR.with_(B=16), 1), (scaling(4096), 2)]:
        inp = make_inputs(w, seed)
        cfg, q, cb, idx, rt = _reference_route(w, inp)
        for _ in range(2):
            sel = torch.full_like(rt.sel, -7)
            ncand = torch.full_like(rt.ncand, -7)
            mdr.mdr_route_noalloc(cfg, q, cb, idx, sel, ncand)
            torch.cuda.synchronize()
            assert torch.equal(sel, rt.sel), w.name
            assert torch.equal(ncand, rt.ncand), w.name


def test_noalloc_route_at_the_benchmark_size():
    import torch
    from learned_product_hash_b200 import mdr
    inp = make_inputs(SCALING_32K, 0)
    cfg, q, cb, idx, rt = _reference_route(SCALING_32K, inp)
    sel = torch.empty_like(rt.sel)
    mdr.mdr_route_noalloc(cfg, q, cb, idx, sel)
    torch.cuda.synchronize()
    assert torch.equal(sel, rt.sel)


def test_noalloc_route_allocates_no_device_memory():
    """After its first call on the device, further calls leave the device's
    free memory unchanged: the scratch is the library's own array."""
    import torch
    from learned_product_hash_b200 import mdr
    w = scaling(4096)
    cfg, q, cb, idx, rt = _reference_route(w, make_inputs(w, 4))
    sel = torch.empty_like(rt.sel)
    ncand = torch.empty_like(rt.ncand)
    mdr.mdr_route_noalloc(cfg, q, cb, idx, sel, ncand)          # first call: address lookup
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        mdr.mdr_route_noalloc(cfg, q, cb, idx, sel, ncand)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.equal(sel, rt.sel) and torch.equal(ncand, rt.ncand)
    # a normal route never writes -1 in a row's last entry (the query block
    # itself); a call whose summary step failed on the device does
    assert (sel[..., -1] >= 0).all()


def test_noalloc_route_rejects_sizes_beyond_its_scratch():
    from learned_product_hash_b200 import mdr
    big = mdr.make_config(scaling(131072).with_(B=4))        # 4*8*2048 routes * 544 B > 32 MiB
    fake = ctypes.c_void_p(0x10000)                          # never touched: rejected first
    idx = mdr.mdr_index(*([0x10000] * 6))
    s = mdr.lib().mdr_route_noalloc(ctypes.byref(big), fake, fake, ctypes.byref(idx), fake, None, None)
    assert s == mdr.MDR_ERR_WORKSPACE
