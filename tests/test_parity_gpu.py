"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on
seeded inputs of every workload, plus edge cases.  The bar is stated in
tests/parity_util.py."""
import numpy as np
import pytest

from oracle import mdr_oracle as O
from tests import parity_util as U
from workloads import ALL, AR, CAPACITY, LONG, SCALING_32K, TINY, make_inputs, scaling

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from learned_product_hash_b200 import mdr
    mdr.lib()


SMALL = [TINY, AR, CAPACITY, scaling(4096)]


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_forward_matches_oracle(w, seed):
    inp = make_inputs(w, seed)
    g = U.run_gpu(w, inp)
    res = U.oracle_for(w, inp)
    rep = U.compare(w, g, res, inp.codebooks, max_ties=2)
    print(f"ties {w.name} seed {seed}: {rep}")


@pytest.mark.parametrize("w", [TINY, AR.with_(B=8), CAPACITY], ids=lambda w: w.name)
def test_split_entry_points_equal_forward(w):
    """mdr_build_index + mdr_route + mdr_attend give exactly what mdr_forward gives."""
    inp = make_inputs(w, 3)
    a = U.run_gpu(w, inp, "forward")
    b = U.run_gpu(w, inp, "split")
    for key in a:
        assert np.array_equal(a[key], b[key]), key


EDGE = {
    # every block in one list: overflow nb - cap, ties everywhere resolved by index
    "zeros_f32": (TINY, dict(zero=True)),
    "zeros_bf16": (scaling(4096).with_(cap=16), dict(zero=True)),
    # every eligible block admitted: the route is the exact top-R, the output dense causal
    "dense_limit_bf16": (AR.with_(B=2, cap=6, K=4, probes=4, R=6), {}),
    "dense_limit_f32": (TINY.with_(cap=6, K=2, probes=2, R=6), {}),
    # local-only control
    "local_only": (AR.with_(B=4, R=0), {}),
    # ragged: 7 blocks, 3 query heads per KV head, block 128, D 64
    "ragged_gqa": (CAPACITY.with_(S=7 * 128, block=128, Hq=6, Hkv=2, R=3, L=3, keys="gaussian"), {}),
    # many locals, tiny capacity (heavy overflow), one probe
    "overflow_heavy": (scaling(4096).with_(cap=1, probes=1, K=4, L=4), {}),
    "fp32_d128": (TINY.with_(D=128, S=256, block=32, Hq=4, Hkv=2, K=16, cap=4, probes=3, R=3, L=2), {}),
    # more heads than one summary pass takes at once (32 for f32 D=128, 64 for
    # bf16 D=128): head groups with a ragged last group, strided row copies
    "many_heads_f32": (TINY.with_(D=128, S=128, block=32, Hq=40, Hkv=40, K=16, cap=4, probes=3, R=2, L=1), {}),
    "many_heads_bf16": (AR.with_(B=1, S=256, Hq=72, Hkv=72, D=128, keys="gaussian"), {}),
    # odd head count: token groups that do not tile the 512 summary threads
    "three_heads_bf16": (AR.with_(B=2, S=512, Hq=3, Hkv=3, D=128, block=128, keys="gaussian"), {}),
    # block 128 at D = 64, one query head per KV head: the per-head kernel
    # rotates 128-row Q tiles whose pairs share one 64-column region
    "block128_d64_bf16": (AR.with_(B=2, S=640, Hq=2, Hkv=2, block=128, keys="gaussian"), {}),
    # block 128 with grouped query heads: pairs of heads share one gather of
    # their selections' union (two and four heads per KV head, D 128 and 64)
    "union_g2_d128": (CAPACITY.with_(S=12 * 128, block=128, D=128, Hq=4, Hkv=2, K=8, cap=16, R=4, L=2), {}),
    "union_g4_long": (LONG.with_(B=2, S=24 * 128), {}),
    "union_g2_d64": (CAPACITY.with_(S=10 * 128, block=128, Hq=2, Hkv=1, K=8, cap=16, R=5, L=1), {}),
}


@pytest.mark.parametrize("name", sorted(EDGE))
def test_edge_cases(name):
    w, kw = EDGE[name]
    inp = make_inputs(w, 5, **kw)
    g = U.run_gpu(w, inp)
    res = U.oracle_for(w, inp)
    rep = U.compare(w, g, res, inp.codebooks, max_ties=2)
    print(f"ties {name}: {rep}")
    if kw.get("zero"):
        assert (g["addr"] == 0).all()
        assert (g["overflow"] == max(0, w.nb - w.cap)).all()
    if name.startswith("dense_limit"):
        assert (g["ncand"] == np.maximum(np.arange(w.nb) - w.L + 1, 0)[None, None, :]).all()


def test_bad_selection_sets_device_status():
    """mdr_attend checks every selected id against the block grid; an id that
    points past the query block is skipped and reported in the status word."""
    import torch
    from learned_product_hash_b200 import mdr
    w = TINY
    inp = make_inputs(w, 0)
    cfg = mdr.make_config(w)
    q, k, v, _ = U.to_device(inp, w)
    res = U.oracle_for(w, inp)
    sel = torch.from_numpy(res.sel.astype(np.int32)).cuda()
    sel[0, 0, 2, 0] = 5                                 # later than block 2
    out = torch.empty_like(q)
    ws = mdr.workspace(cfg)
    mdr.mdr_attend(cfg, q, k, v, sel, out, ws)
    assert mdr.mdr_read_device_status(ws) == 2
    # the other query blocks are unaffected
    rows = np.ones((1, w.S, 1), dtype=bool)
    rows[0, 32:48] = False
    U.check_out(w, out.cpu().numpy(), res.out, rows)


def test_union_attend_caller_selections():
    """Block 128, two query heads per KV head (one unit per head pair, the
    union of the pair's blocks gathered once), on selections a route never
    writes: one head of a pair with nothing selected while the other has
    blocks, both heads empty, disjoint and identical rows, ids in any order,
    and an id past its query block (skipped, status 2)."""
    import torch
    from learned_product_hash_b200 import mdr
    w = CAPACITY.with_(S=9 * 128, block=128, D=128, Hq=4, Hkv=2, K=8, cap=16, R=4, L=2)
    inp = make_inputs(w, 21)
    cfg = mdr.make_config(w)
    q, k, v, _ = U.to_device(inp, w)
    rng = np.random.default_rng(22)
    sel = np.full((w.B, w.Hq, w.nb, w.R + w.L), -1, dtype=np.int32)
    for hq in range(w.Hq):
        for j in range(w.nb):
            n = int(rng.integers(1, min(j + 1, w.R + w.L) + 1))
            sel[0, hq, j, :n] = rng.permutation(j + 1)[:n]          # distinct, any order
    sel[0, 0, 5] = -1                                              # head 0 empty, head 1 not
    sel[0, 1, 7] = -1                                              # head 1 empty, head 0 not
    sel[0, 2, 3] = -1                                              # both heads of a pair empty
    sel[0, 3, 3] = -1
    sel[0, 3, 6] = sel[0, 2, 6]                                    # identical rows
    sel[0, 2, 8, :] = [0, 2, 4, 6, 8, -1]                          # disjoint rows
    sel[0, 3, 8, :] = [1, 3, 5, 7, -1, -1]
    sel[0, 1, 4, -1] = 6                                           # later than block 4
    out = torch.empty_like(q)
    ws = mdr.workspace(cfg)
    mdr.mdr_attend(cfg, q, k, v, torch.from_numpy(sel).cuda(), out, ws)
    assert mdr.mdr_read_device_status(ws) == 2
    got = U.out_to_numpy(out, w)
    p = O.Params.of(w)
    qr, kr = O.rope(inp.q.astype(np.float64), p.rope_base), O.rope(inp.k.astype(np.float64), p.rope_base)
    jj = np.arange(w.nb)[None, None, :, None]
    clean = np.where((sel >= 0) & (sel <= jj), sel, -1)
    has = (clean >= 0).any(axis=-1)
    rows = [(0, hq, j) for hq in range(w.Hq) for j in range(w.nb) if has[0, hq, j]]
    ref = O.attend(qr, kr, inp.v.astype(np.float64), clean, w.block, p.softmax_scale, rows)
    for hq, j in ((0, 5), (1, 7), (2, 3), (3, 3)):
        assert not has[0, hq, j]
        assert (got[0, j * w.block:(j + 1) * w.block, hq] == 0).all()
    U.check_out(w, got, ref)


HOST_CASES = {
    "ar_b4": AR.with_(B=4),                                          # 6 blocks: one chunk per block
    "scaling4k": scaling(4096),                                      # 64 blocks in 8 chunks
    "overflow_heavy": scaling(4096).with_(cap=1, probes=1, K=4, L=4),  # lists overflow across chunks
    "union_g2_d128": CAPACITY.with_(S=12 * 128, block=128, D=128, Hq=4, Hkv=2, K=8, cap=16, R=4, L=2, B=2),
    "tiny_f32": TINY,
}


@pytest.mark.parametrize("name", sorted(HOST_CASES))
def test_host_entry_point_matches_device(name):
    """mdr_forward_host runs the sequence in chunks of query blocks (copies of
    one chunk overlapping the kernels and copies of the others); its out,
    sel, overflow and maxload are bit-identical to mdr_forward's."""
    import torch
    from learned_product_hash_b200 import mdr
    w = HOST_CASES[name]
    inp = make_inputs(w, 7)
    g = U.run_gpu(w, inp)
    cfg = mdr.make_config(w)
    pin = lambda x: torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x).pin_memory()
    q, k, v = pin(inp.q_store), pin(inp.k_store), pin(inp.v_store)
    cb = torch.from_numpy(inp.codebooks).pin_memory()
    out = torch.empty_like(q).pin_memory()
    sel = torch.empty(g["sel"].shape, dtype=torch.int32).pin_memory()
    ovf = torch.empty(g["overflow"].shape, dtype=torch.int32)
    mx = torch.empty(g["maxload"].shape, dtype=torch.int32)
    dws = torch.empty(mdr.mdr_host_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
    mdr.mdr_forward_host(cfg, q, k, v, cb, out, sel, ovf, mx, dws)
    assert np.array_equal(sel.numpy(), g["sel"])
    assert np.array_equal(ovf.numpy(), g["overflow"]) and np.array_equal(mx.numpy(), g["maxload"])
    got = out.view(torch.bfloat16).float().numpy() if w.dtype == "bf16" else out.numpy()
    assert np.array_equal(got, g["out"])


@pytest.mark.parametrize("w", [SCALING_32K, LONG], ids=lambda w: w.name)
def test_full_size_sampled(w):
    """The benchmark's launch at full size: routing compared everywhere,
    attention on sampled query blocks the oracle computes one by one."""
    inp = make_inputs(w, 0)
    g = U.run_gpu(w, inp)
    p = O.Params.of(w)
    res = O.forward(inp.q, inp.k, inp.v, inp.codebooks, p, attention=False)
    rows = U.sampled_rows(w, res)
    res.out = O.attend(res.qr, res.kr, res.v, res.sel, w.block, p.softmax_scale, rows)
    rep = U.compare(w, g, res, inp.codebooks, max_ties=U.full_size_tie_budget(w))
    print(f"ties {w.name}: {rep}")
    if w is LONG:
        assert rep["overflow"] > 0, "the long workload must overflow its lists"
