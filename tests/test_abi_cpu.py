"""The C-ABI library without a GPU: it loads, exports every entry point that
include/mdr.h declares, and its host-side argument checks answer correctly
before anything is enqueued."""
import ctypes
import os
import re

import pytest

from learned_product_hash_b200 import mdr
from workloads import ALL, TINY, SCALING_32K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^\s*(?:mdr_status|int32_t|const char\*)\s+(mdr_\w+)\s*\(", src, re.M)
    return names


def test_library_exports_every_declared_symbol():
    L = mdr.lib()
    declared = _declared()
    assert len(declared) >= 11
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) == set(mdr.EXPORTED) | (set(declared) - set(mdr.EXPORTED))
    assert mdr.mdr_abi_version() == 1


@pytest.mark.parametrize("name", sorted(ALL))
def test_workload_configs_are_supported(name):
    cfg = mdr.make_config(ALL[name])
    assert mdr.mdr_check_config(cfg) == mdr.MDR_OK
    assert mdr.mdr_workspace_bytes(cfg) > 0
    assert mdr.mdr_host_workspace_bytes(cfg) > mdr.mdr_workspace_bytes(cfg)


BAD = [
    (dict(S=100), mdr.MDR_ERR_INVALID_ARG),             # S % block != 0
    (dict(Hq=3, Hkv=2), mdr.MDR_ERR_INVALID_ARG),       # Hq % Hkv != 0
    (dict(L=0), mdr.MDR_ERR_INVALID_ARG),               # own block must be local
    (dict(probes=9), mdr.MDR_ERR_INVALID_ARG),          # probes > K
    (dict(cap=0), mdr.MDR_ERR_INVALID_ARG),
    (dict(R=-1), mdr.MDR_ERR_INVALID_ARG),
    (dict(rope_base=1.0), mdr.MDR_ERR_INVALID_ARG),
    (dict(dtype=7), mdr.MDR_ERR_INVALID_ARG),
    (dict(D=48), mdr.MDR_ERR_UNSUPPORTED),
    (dict(block=8, S=96), mdr.MDR_ERR_UNSUPPORTED),
    (dict(K=200, probes=2), mdr.MDR_ERR_UNSUPPORTED),
    (dict(R=33), mdr.MDR_ERR_UNSUPPORTED),
    (dict(P=3, D=32), mdr.MDR_ERR_INVALID_ARG),         # D % P != 0
]


@pytest.mark.parametrize("change,expect", BAD)
def test_bad_configs_rejected(change, expect):
    cfg = mdr.make_config(TINY.with_(**change))
    assert mdr.mdr_check_config(cfg) == expect


def test_bf16_needs_tensor_core_tiles():
    cfg = mdr.make_config(TINY.with_(dtype="bf16"))       # block 16, D 32
    assert mdr.mdr_check_config(cfg) == mdr.MDR_ERR_UNSUPPORTED
    assert mdr.mdr_check_config(mdr.make_config(SCALING_32K)) == mdr.MDR_OK


def test_entry_points_check_arguments_before_any_gpu_work():
    L = mdr.lib()
    cfg = mdr.make_config(TINY)
    n = mdr.mdr_workspace_bytes(cfg)
    idx = mdr.mdr_index()
    rt = mdr.mdr_route_out()
    fake = ctypes.c_void_p(0x10000)            # never dereferenced: checks fail first
    # null inputs
    assert L.mdr_forward(ctypes.byref(cfg), None, fake, fake, fake, ctypes.byref(idx), ctypes.byref(rt),
                         fake, fake, n, None) == mdr.MDR_ERR_INVALID_ARG
    # missing index buffers
    rt.sel = 0x10000
    assert L.mdr_forward(ctypes.byref(cfg), fake, fake, fake, fake, ctypes.byref(idx), ctypes.byref(rt),
                         fake, fake, n, None) == mdr.MDR_ERR_INVALID_ARG
    idx = mdr.mdr_index(*([0x10000] * 6))
    # workspace too small, then misaligned
    assert L.mdr_forward(ctypes.byref(cfg), fake, fake, fake, fake, ctypes.byref(idx), ctypes.byref(rt),
                         fake, fake, n - 1, None) == mdr.MDR_ERR_WORKSPACE
    assert L.mdr_forward(ctypes.byref(cfg), fake, fake, fake, fake, ctypes.byref(idx), ctypes.byref(rt),
                         fake, ctypes.c_void_p(0x10010), n, None) == mdr.MDR_ERR_WORKSPACE
    # unsupported config is reported before pointers are looked at
    bad = mdr.make_config(TINY.with_(D=48))
    assert L.mdr_build_index(ctypes.byref(bad), None, None, None, None, 0, None) == mdr.MDR_ERR_UNSUPPORTED
    assert L.mdr_attend(ctypes.byref(cfg), fake, None, fake, fake, fake, fake, n, None) == mdr.MDR_ERR_INVALID_ARG
    assert L.mdr_route(ctypes.byref(cfg), fake, fake, ctypes.byref(idx), None, fake, n, None) == mdr.MDR_ERR_INVALID_ARG
    # unaligned tensors
    odd = ctypes.c_void_p(0x10004)
    assert L.mdr_attend(ctypes.byref(cfg), odd, fake, fake, fake, fake, fake, n, None) == mdr.MDR_ERR_INVALID_ARG
    assert L.mdr_read_device_status(None, None, None) == mdr.MDR_ERR_INVALID_ARG


def test_status_strings():
    for s in range(6):
        assert mdr.status_string(s)
    assert mdr.status_string(99) == "unknown status"


def test_decode_entry_points_check_arguments_before_any_gpu_work():
    L = mdr.lib()
    cfg = mdr.make_config(TINY)
    assert mdr.mdr_decode_workspace_bytes(cfg) > 0
    fake = ctypes.c_void_p(0x10000)            # 16-byte aligned, never dereferenced: checks fail first
    st = mdr.mdr_decode_state(fake, fake, fake, mdr.mdr_index(fake, fake, fake, fake, fake, fake))
    n = mdr.mdr_decode_workspace_bytes(cfg)
    step = lambda t, **kw: L.mdr_decode_step(
        ctypes.byref(kw.get("cfg", cfg)), t, fake, fake, fake, fake, ctypes.byref(kw.get("st", st)),
        fake, kw.get("sel", fake), None, kw.get("ws", ctypes.c_void_p(0x100000)), kw.get("n", n), None)
    assert step(-1) == mdr.MDR_ERR_INVALID_ARG                       # before the first position
    assert step(TINY.S) == mdr.MDR_ERR_INVALID_ARG                   # past the capacity
    assert step(0, sel=None) == mdr.MDR_ERR_INVALID_ARG              # sel is required
    assert step(0, ws=None) == mdr.MDR_ERR_WORKSPACE
    assert step(0, ws=ctypes.c_void_p(0x100010)) == mdr.MDR_ERR_WORKSPACE   # not 256-byte aligned
    nost = mdr.mdr_decode_state(None, fake, fake, mdr.mdr_index(fake, fake, fake, fake, fake, fake))
    assert step(0, st=nost) == mdr.MDR_ERR_INVALID_ARG               # state without a key cache
    bad = mdr.make_config(TINY.with_(S=100))
    assert step(0, cfg=bad) == mdr.MDR_ERR_INVALID_ARG
    pre = lambda S0, nbytes=n: L.mdr_decode_prefill(ctypes.byref(cfg), S0, fake, fake, fake, ctypes.byref(st),
                                                    ctypes.c_void_p(0x100000), nbytes, None)
    assert pre(TINY.block + 1) == mdr.MDR_ERR_INVALID_ARG             # not a whole number of blocks
    assert pre(TINY.S + TINY.block) == mdr.MDR_ERR_INVALID_ARG        # past the capacity
    assert pre(TINY.block, nbytes=n - 1) == mdr.MDR_ERR_WORKSPACE


def test_control_entry_points_check_arguments_before_any_gpu_work():
    L = mdr.lib()
    cfg = mdr.make_config(TINY)
    fake = ctypes.c_void_p(0x10000)            # never dereferenced: the checks fail first
    idx = mdr.mdr_index(fake, fake, fake, fake, fake, fake)
    rt = mdr.mdr_route_out(fake, None, None, None)
    ws, n = ctypes.c_void_p(0x100000), 1 << 30
    forced = lambda force, **kw: L.mdr_route_forced(
        ctypes.byref(kw.get("cfg", cfg)), fake, fake, ctypes.byref(idx), force, ctypes.byref(kw.get("rt", rt)),
        kw.get("ws", ws), n, None)
    assert forced(None) == mdr.MDR_ERR_INVALID_ARG                      # the forced ids are required
    assert forced(fake, rt=mdr.mdr_route_out(None, None, None, None)) == mdr.MDR_ERR_INVALID_ARG
    assert forced(fake, ws=None) == mdr.MDR_ERR_WORKSPACE
    assert forced(fake, cfg=mdr.make_config(TINY.with_(S=100))) == mdr.MDR_ERR_INVALID_ARG
    hits = lambda sel, target, counts: L.mdr_target_hits(ctypes.byref(cfg), sel, target, None, counts, None)
    assert hits(None, fake, fake) == mdr.MDR_ERR_INVALID_ARG
    assert hits(fake, None, fake) == mdr.MDR_ERR_INVALID_ARG
    assert hits(fake, fake, None) == mdr.MDR_ERR_INVALID_ARG


def test_calibration_entry_points_check_arguments_before_any_gpu_work():
    L = mdr.lib()
    n = ctypes.c_size_t(0)
    assert L.mdr_calibrate_workspace_bytes(8192, 128, 2, 64, ctypes.byref(n)) == mdr.MDR_OK and n.value > 0
    assert L.mdr_calibrate_workspace_bytes(0, 128, 2, 64, ctypes.byref(n)) == mdr.MDR_ERR_INVALID_ARG
    assert L.mdr_calibrate_workspace_bytes(10, 96, 2, 64, ctypes.byref(n)) == mdr.MDR_ERR_UNSUPPORTED
    assert L.mdr_calibrate_workspace_bytes(10, 128, 2, 129, ctypes.byref(n)) == mdr.MDR_ERR_UNSUPPORTED
    assert L.mdr_calibrate_workspace_bytes(10, 32, 8, 4, ctypes.byref(n)) == mdr.MDR_ERR_UNSUPPORTED   # P > 4
    assert L.mdr_calibrate_workspace_bytes(10, 32, 4, 4, ctypes.byref(n)) == mdr.MDR_OK                  # dsub 8
    fake = ctypes.c_void_p(0x10000)
    ws, nbytes = ctypes.c_void_p(0x100000), 1 << 30
    call = lambda rec=fake, cin=fake, cout=fake, rounds=1, ws=ws: L.mdr_calibrate_codebooks(
        rec, 100, 64, 2, 16, cin, cout, rounds, None, None, ws, nbytes, None)
    assert call(rec=None) == mdr.MDR_ERR_INVALID_ARG
    assert call(rec=ctypes.c_void_p(0x10004)) == mdr.MDR_ERR_INVALID_ARG          # not 16-byte aligned
    assert call(cout=None) == mdr.MDR_ERR_INVALID_ARG
    assert call(rounds=-1) == mdr.MDR_ERR_INVALID_ARG
    assert call(cout=ctypes.c_void_p(0x10010)) == mdr.MDR_ERR_INVALID_ARG         # overlaps the input codebooks
    assert call(ws=None) == mdr.MDR_ERR_WORKSPACE
    assert call(ws=ctypes.c_void_p(0x100010)) == mdr.MDR_ERR_WORKSPACE            # not 256-byte aligned


def test_backward_entry_point_checks_arguments_before_any_gpu_work():
    L = mdr.lib()
    cfg = mdr.make_config(TINY)
    n = mdr.mdr_backward_workspace_bytes(cfg)
    assert n > 0
    fake = ctypes.c_void_p(0x10000)
    ws = ctypes.c_void_p(0x100000)
    call = lambda cfg=cfg, dout=fake, ws=ws, nbytes=n: L.mdr_attend_backward(
        ctypes.byref(cfg), fake, fake, fake, fake, dout, fake, fake, fake, ws, nbytes, None)
    assert call(dout=None) == mdr.MDR_ERR_INVALID_ARG
    assert call(ws=None) == mdr.MDR_ERR_WORKSPACE
    assert call(ws=ctypes.c_void_p(0x100010)) == mdr.MDR_ERR_WORKSPACE       # not 256-byte aligned
    assert call(nbytes=n - 1) == mdr.MDR_ERR_WORKSPACE
    big = mdr.make_config(TINY.with_(S=30000 * 16))                           # 30,000 blocks
    nbig = mdr.mdr_backward_workspace_bytes(big)
    assert call(cfg=big, nbytes=nbig) == mdr.MDR_ERR_UNSUPPORTED


def test_backward_tensor_core_path_checks_alignment_before_any_gpu_work():
    """bf16 storage runs on the tensor cores, whose TMA loads need 16-byte
    aligned tensors: a misaligned input or gradient is refused on the host."""
    from workloads import AR
    L = mdr.lib()
    cfg = mdr.make_config(AR)
    n = mdr.mdr_backward_workspace_bytes(cfg)
    ok, bad = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10008)
    ws = ctypes.c_void_p(0x100000)
    for i in (0, 1, 2, 4, 5, 6, 7):        # q, k, v, dout, dq, dk, dv (sel may have any alignment)
        args = [ok] * 8
        args[i] = bad
        assert L.mdr_attend_backward(ctypes.byref(cfg), *args, ws, n, None) == mdr.MDR_ERR_INVALID_ARG, i
