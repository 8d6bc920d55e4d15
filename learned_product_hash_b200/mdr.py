"""Thin ctypes binding of libmdr (include/mdr.h), same names as the C ABI.

Argument marshalling only: every step of the forward runs in the CUDA kernels
behind the C ABI.  PyTorch provides device memory and the current stream.
The shared library must be built (``python -m learned_product_hash_b200.build``
or ``__graft_entry__.build()``); without it every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmdr.so")

MDR_OK, MDR_ERR_INVALID_ARG, MDR_ERR_UNSUPPORTED, MDR_ERR_WORKSPACE, MDR_ERR_CUDA, MDR_ERR_DEVICE = range(6)
MDR_F32, MDR_BF16 = 0, 1

EXPORTED = (
    "mdr_abi_version", "mdr_status_string", "mdr_check_config", "mdr_workspace_bytes",
    "mdr_build_index", "mdr_route", "mdr_attend", "mdr_forward", "mdr_host_workspace_bytes",
    "mdr_forward_host", "mdr_read_device_status", "mdr_forward_profiled", "mdr_route_noalloc",
    "mdr_decode_workspace_bytes", "mdr_decode_reset", "mdr_decode_prefill", "mdr_decode_step",
    "mdr_route_forced", "mdr_target_hits", "mdr_calibrate_workspace_bytes", "mdr_calibrate_codebooks",
    "mdr_backward_workspace_bytes", "mdr_attend_backward",
)


class MdrError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


class mdr_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "S", "Hq", "Hkv", "D", "block", "P", "K", "cap", "probes", "R", "L")] + \
               [("rope_base", ctypes.c_float), ("scale", ctypes.c_float), ("dtype", ctypes.c_int32)]


class mdr_index(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("kbar", "addr", "lists", "load", "overflow", "maxload")]


class mdr_route_out(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("sel", "qbar", "qcodes", "ncand")]


class mdr_decode_state(ctypes.Structure):
    _fields_ = [("krot", ctypes.c_void_p), ("v", ctypes.c_void_p), ("ksum", ctypes.c_void_p), ("idx", mdr_index)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmdr.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmdr.so is not built ({LIB_PATH}); run "
                              "`python -m learned_product_hash_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        cfgp = ctypes.POINTER(mdr_config)
        idxp = ctypes.POINTER(mdr_index)
        rtp = ctypes.POINTER(mdr_route_out)
        sig = {
            "mdr_abi_version": ([], ctypes.c_int32),
            "mdr_status_string": ([i32], ctypes.c_char_p),
            "mdr_check_config": ([cfgp], i32),
            "mdr_workspace_bytes": ([cfgp, ctypes.POINTER(sz)], i32),
            "mdr_build_index": ([cfgp, vp, vp, idxp, vp, sz, vp], i32),
            "mdr_route": ([cfgp, vp, vp, idxp, rtp, vp, sz, vp], i32),
            "mdr_attend": ([cfgp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
            "mdr_forward": ([cfgp, vp, vp, vp, vp, idxp, rtp, vp, vp, sz, vp], i32),
            "mdr_attend_train": ([cfgp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
            "mdr_forward_train": ([cfgp, vp, vp, vp, vp, idxp, rtp, vp, vp, vp, sz, vp], i32),
            "mdr_host_workspace_bytes": ([cfgp, ctypes.POINTER(sz)], i32),
            "mdr_forward_host": ([cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
            "mdr_read_device_status": ([vp, ctypes.POINTER(ctypes.c_int32), vp], i32),
            "mdr_forward_profiled": ([cfgp, vp, vp, vp, vp, idxp, rtp, vp, vp, sz, vp,
                                      ctypes.POINTER(vp), ctypes.c_int32], i32),
            "mdr_route_noalloc": ([cfgp, vp, vp, idxp, vp, vp, vp], i32),
            "mdr_route_forced": ([cfgp, vp, vp, idxp, vp, rtp, vp, sz, vp], i32),
            "mdr_target_hits": ([cfgp, vp, vp, vp, vp, vp], i32),
            "mdr_backward_workspace_bytes": ([cfgp, ctypes.POINTER(sz)], i32),
            "mdr_attend_backward": ([cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
            "mdr_attend_backward_saved": ([cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
            "mdr_calibrate_workspace_bytes": ([ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                               ctypes.POINTER(sz)], i32),
            "mdr_calibrate_codebooks": ([vp, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                         vp, vp, ctypes.c_int32, vp, vp, vp, sz, vp], i32),
            "mdr_decode_workspace_bytes": ([cfgp, ctypes.POINTER(sz)], i32),
            "mdr_decode_reset": ([cfgp, ctypes.POINTER(mdr_decode_state), vp], i32),
            "mdr_decode_prefill": ([cfgp, ctypes.c_int32, vp, vp, vp, ctypes.POINTER(mdr_decode_state),
                                    vp, sz, vp], i32),
            "mdr_decode_step": ([cfgp, ctypes.c_int32, vp, vp, vp, vp, ctypes.POINTER(mdr_decode_state),
                                 vp, vp, vp, vp, sz, vp], i32),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes, f.restype = args, res
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().mdr_status_string(int(s)).decode()


def _ok(status: int, what: str):
    if status != MDR_OK:
        raise MdrError(status, what)


def make_config(w) -> mdr_config:
    """mdr_config from any object with the workload fields (B, S, Hq, ...)."""
    dt = {"bf16": MDR_BF16, "f32": MDR_F32}[w.dtype] if isinstance(w.dtype, str) else int(w.dtype)
    return mdr_config(w.B, w.S, w.Hq, w.Hkv, w.D, w.block, w.P, w.K, w.cap, w.probes, w.R, w.L,
                      float(w.rope_base), float(w.scale), dt)


def mdr_abi_version() -> int:
    return lib().mdr_abi_version()


def mdr_check_config(cfg: mdr_config) -> int:
    return lib().mdr_check_config(ctypes.byref(cfg))


def mdr_workspace_bytes(cfg: mdr_config) -> int:
    n = ctypes.c_size_t(0)
    _ok(lib().mdr_workspace_bytes(ctypes.byref(cfg), ctypes.byref(n)), "mdr_workspace_bytes")
    return n.value


def mdr_host_workspace_bytes(cfg: mdr_config) -> int:
    n = ctypes.c_size_t(0)
    _ok(lib().mdr_host_workspace_bytes(ctypes.byref(cfg), ctypes.byref(n)), "mdr_host_workspace_bytes")
    return n.value


# ------------------------------------------------------------ torch helpers
def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


@dataclass
class Index:
    """Device buffers of mdr_index (torch tensors)."""
    kbar: object
    addr: object
    lists: object
    load: object
    overflow: object
    maxload: object

    @classmethod
    def empty(cls, cfg: mdr_config, device="cuda") -> "Index":
        import torch
        nb, A = cfg.S // cfg.block, cfg.K ** cfg.P
        i32 = dict(dtype=torch.int32, device=device)
        return cls(torch.empty(cfg.B, cfg.Hkv, nb, cfg.D, dtype=torch.float32, device=device),
                   torch.empty(cfg.B, cfg.Hkv, nb, **i32),
                   torch.empty(cfg.B, cfg.Hkv, A, cfg.cap, **i32),
                   torch.empty(cfg.B, cfg.Hkv, A, **i32),
                   torch.empty(cfg.B, cfg.Hkv, **i32),
                   torch.empty(cfg.B, cfg.Hkv, **i32))

    def c(self) -> mdr_index:
        return mdr_index(*(_ptr(getattr(self, f)) for f in ("kbar", "addr", "lists", "load", "overflow", "maxload")))


@dataclass
class RouteOut:
    sel: object
    qbar: object = None
    qcodes: object = None
    ncand: object = None

    @classmethod
    def empty(cls, cfg: mdr_config, device="cuda", debug=False) -> "RouteOut":
        import torch
        nb = cfg.S // cfg.block
        i32 = dict(dtype=torch.int32, device=device)
        sel = torch.empty(cfg.B, cfg.Hq, nb, cfg.R + cfg.L, **i32)
        if not debug:
            return cls(sel)
        return cls(sel, torch.empty(cfg.B, cfg.Hq, nb, cfg.D, dtype=torch.float32, device=device),
                   torch.empty(cfg.B, cfg.Hq, nb, cfg.P, cfg.probes, **i32),
                   torch.empty(cfg.B, cfg.Hq, nb, **i32))

    def c(self) -> mdr_route_out:
        return mdr_route_out(_ptr(self.sel), _ptr(self.qbar), _ptr(self.qcodes), _ptr(self.ncand))


def workspace(cfg: mdr_config, device="cuda"):
    import torch
    return torch.empty(mdr_workspace_bytes(cfg), dtype=torch.uint8, device=device)


def mdr_build_index(cfg, k, codebooks, idx: Index, ws, stream=None):
    _ok(lib().mdr_build_index(ctypes.byref(cfg), _ptr(k), _ptr(codebooks), ctypes.byref(idx.c()),
                              _ptr(ws), ws.numel(), _stream(stream)), "mdr_build_index")


def mdr_route(cfg, q, codebooks, idx: Index, rt: RouteOut, ws, stream=None):
    _ok(lib().mdr_route(ctypes.byref(cfg), _ptr(q), _ptr(codebooks), ctypes.byref(idx.c()),
                        ctypes.byref(rt.c()), _ptr(ws), ws.numel(), _stream(stream)), "mdr_route")


def mdr_attend(cfg, q, k, v, sel, out, ws, stream=None):
    _ok(lib().mdr_attend(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(sel), _ptr(out),
                         _ptr(ws), ws.numel(), _stream(stream)), "mdr_attend")


def mdr_forward(cfg, q, k, v, codebooks, idx: Index, rt: RouteOut, out, ws, stream=None):
    _ok(lib().mdr_forward(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(codebooks),
                          ctypes.byref(idx.c()), ctypes.byref(rt.c()), _ptr(out), _ptr(ws),
                          ws.numel(), _stream(stream)), "mdr_forward")


def mdr_attend_train(cfg, q, k, v, sel, out, lse, ws, stream=None):
    """mdr_attend that also writes each row's softmax normaliser lse
    (float32 [B,Hq,S], natural log) for mdr_attend_backward_saved."""
    _ok(lib().mdr_attend_train(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(sel), _ptr(out), _ptr(lse),
                               _ptr(ws), ws.numel(), _stream(stream)), "mdr_attend_train")


def mdr_forward_train(cfg, q, k, v, codebooks, idx: Index, rt: RouteOut, out, lse, ws, stream=None):
    """mdr_forward that also writes each row's softmax normaliser lse."""
    _ok(lib().mdr_forward_train(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(codebooks),
                                ctypes.byref(idx.c()), ctypes.byref(rt.c()), _ptr(out), _ptr(lse), _ptr(ws),
                                ws.numel(), _stream(stream)), "mdr_forward_train")


def mdr_forward_profiled(cfg, q, k, v, codebooks, idx: Index, rt: RouteOut, out, ws, events, stream=None):
    """events: list of torch.cuda.Event(enable_timing=True) (or None), recorded
    before K1 and after K1, K3, K4, K5."""
    for e in events:
        if e is not None and not e.cuda_event:
            e.record()          # torch creates the CUDA event on its first record
    arr = (ctypes.c_void_p * len(events))(*[None if e is None else e.cuda_event for e in events])
    _ok(lib().mdr_forward_profiled(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(codebooks),
                                   ctypes.byref(idx.c()), ctypes.byref(rt.c()), _ptr(out), _ptr(ws),
                                   ws.numel(), _stream(stream), arr, len(events)), "mdr_forward_profiled")


def mdr_forward_host(cfg, q, k, v, codebooks, out, sel=None, overflow=None, maxload=None,
                     dev_ws=None, stream=None):
    """Host buffers (torch CPU tensors, ideally pinned) in and out."""
    _ok(lib().mdr_forward_host(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(codebooks), _ptr(out),
                               _ptr(sel), _ptr(overflow), _ptr(maxload), _ptr(dev_ws), dev_ws.numel(),
                               _stream(stream)), "mdr_forward_host")


def mdr_read_device_status(ws, stream=None) -> int:
    code = ctypes.c_int32(0)
    s = lib().mdr_read_device_status(_ptr(ws), ctypes.byref(code), _stream(stream))
    if s not in (MDR_OK, MDR_ERR_DEVICE):
        raise MdrError(s, "mdr_read_device_status")
    return code.value


def mdr_route_noalloc(cfg, q, codebooks, idx: Index, sel, ncand=None, stream=None):
    """Route with the library's built-in scratch instead of a workspace (for
    callers that cannot allocate device memory); see include/mdr.h."""
    _ok(lib().mdr_route_noalloc(ctypes.byref(cfg), _ptr(q), _ptr(codebooks), ctypes.byref(idx.c()),
                                _ptr(sel), _ptr(ncand), _stream(stream)), "mdr_route_noalloc")


# ------------------------------------------------- controls and diagnostics
def mdr_route_forced(cfg, q, codebooks, idx: Index, force, rt: RouteOut, ws, stream=None):
    """mdr_route with a forced target block per route (int32 [B,Hq,nb], -1
    none); see include/mdr.h."""
    _ok(lib().mdr_route_forced(ctypes.byref(cfg), _ptr(q), _ptr(codebooks), ctypes.byref(idx.c()),
                               _ptr(force), ctypes.byref(rt.c()), _ptr(ws), ws.numel(), _stream(stream)),
        "mdr_route_forced")


def mdr_target_hits(cfg, sel, target, counts, hit=None, stream=None):
    """Per-route target hits (hit, optional) and counts[0] = routes with a
    target, counts[1] = hits (device int32 [2]); see include/mdr.h."""
    _ok(lib().mdr_target_hits(ctypes.byref(cfg), _ptr(sel), _ptr(target), _ptr(hit), _ptr(counts),
                              _stream(stream)), "mdr_target_hits")


# ------------------------------------------------------------------ backward
def mdr_backward_workspace_bytes(cfg: mdr_config) -> int:
    n = ctypes.c_size_t(0)
    _ok(lib().mdr_backward_workspace_bytes(ctypes.byref(cfg), ctypes.byref(n)), "mdr_backward_workspace_bytes")
    return n.value


def backward_workspace(cfg: mdr_config, device=None):
    import torch
    return torch.empty(mdr_backward_workspace_bytes(cfg), dtype=torch.uint8, device=device or torch.device("cuda"))


def mdr_attend_backward(cfg, q, k, v, sel, dout, dq, dk, dv, ws, stream=None):
    """dq, dk, dv (float32) of the attention output for upstream gradient
    dout, with the route sel held fixed; see include/mdr.h."""
    _ok(lib().mdr_attend_backward(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(sel), _ptr(dout),
                                  _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(), _stream(stream)),
        "mdr_attend_backward")


def mdr_attend_backward_saved(cfg, q, k, v, sel, out, lse, dout, dq, dk, dv, ws, stream=None):
    """mdr_attend_backward reusing the forward's output and row normalisers
    (from mdr_attend_train / mdr_forward_train)."""
    _ok(lib().mdr_attend_backward_saved(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(sel), _ptr(out),
                                        _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(),
                                        _stream(stream)), "mdr_attend_backward_saved")


# ------------------------------------------------------ codebook calibration
def mdr_calibrate_workspace_bytes(N: int, D: int, P: int, K: int) -> int:
    n = ctypes.c_size_t(0)
    _ok(lib().mdr_calibrate_workspace_bytes(N, D, P, K, ctypes.byref(n)), "mdr_calibrate_workspace_bytes")
    return n.value


def calibrate_workspace(N: int, D: int, P: int, K: int, device=None):
    import torch
    return torch.empty(mdr_calibrate_workspace_bytes(N, D, P, K), dtype=torch.uint8,
                       device=device or torch.device("cuda"))


def mdr_calibrate_codebooks(records, codebooks_in, codebooks_out, rounds, ws, counts=None, assign=None,
                            stream=None):
    """records: float32 [N, D] (or any contiguous [..., D]); codebooks
    float32 [P, K, D/P]; see include/mdr.h."""
    D = records.shape[-1]
    N = records.numel() // D
    P, K = codebooks_in.shape[0], codebooks_in.shape[1]
    _ok(lib().mdr_calibrate_codebooks(_ptr(records), N, D, P, K, _ptr(codebooks_in), _ptr(codebooks_out),
                                      int(rounds), _ptr(counts), _ptr(assign), _ptr(ws), ws.numel(),
                                      _stream(stream)), "mdr_calibrate_codebooks")


# ------------------------------------------------------------------ decoding
def mdr_decode_workspace_bytes(cfg: mdr_config) -> int:
    n = ctypes.c_size_t(0)
    _ok(lib().mdr_decode_workspace_bytes(ctypes.byref(cfg), ctypes.byref(n)), "mdr_decode_workspace_bytes")
    return n.value


@dataclass
class DecodeState:
    """Device buffers of mdr_decode_state (torch tensors); cfg.S is the
    capacity in tokens."""
    krot: object
    v: object
    ksum: object
    idx: Index

    @classmethod
    def empty(cls, cfg: mdr_config, device="cuda") -> "DecodeState":
        import torch
        dt = torch.bfloat16 if cfg.dtype == MDR_BF16 else torch.float32
        return cls(torch.empty(cfg.B, cfg.S, cfg.Hkv, cfg.D, dtype=dt, device=device),
                   torch.empty(cfg.B, cfg.S, cfg.Hkv, cfg.D, dtype=dt, device=device),
                   torch.empty(cfg.B, cfg.Hkv, cfg.D, dtype=torch.float32, device=device),
                   Index.empty(cfg, device))

    def c(self) -> mdr_decode_state:
        return mdr_decode_state(_ptr(self.krot), _ptr(self.v), _ptr(self.ksum), self.idx.c())


def decode_workspace(cfg: mdr_config, device="cuda"):
    import torch
    return torch.empty(mdr_decode_workspace_bytes(cfg), dtype=torch.uint8, device=device)


def mdr_decode_reset(cfg, st: DecodeState, stream=None):
    _ok(lib().mdr_decode_reset(ctypes.byref(cfg), ctypes.byref(st.c()), _stream(stream)), "mdr_decode_reset")


def mdr_decode_prefill(cfg, S0: int, k, v, codebooks, st: DecodeState, ws, stream=None):
    _ok(lib().mdr_decode_prefill(ctypes.byref(cfg), int(S0), _ptr(k), _ptr(v), _ptr(codebooks),
                                 ctypes.byref(st.c()), _ptr(ws), ws.numel(), _stream(stream)),
        "mdr_decode_prefill")


def mdr_decode_step(cfg, t: int, q_t, k_t, v_t, codebooks, st: DecodeState, out_t, sel_t, ws,
                    ncand_t=None, stream=None):
    _ok(lib().mdr_decode_step(ctypes.byref(cfg), int(t), _ptr(q_t), _ptr(k_t), _ptr(v_t), _ptr(codebooks),
                              ctypes.byref(st.c()), _ptr(out_t), _ptr(sel_t), _ptr(ncand_t), _ptr(ws),
                              ws.numel(), _stream(stream)), "mdr_decode_step")
