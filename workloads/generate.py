"""Seeded synthetic inputs for the routed-attention forward.

This module only draws random numbers and stores them; it computes no step of
the method (no rotation, no mean, no score, no routing).  The same arrays feed
the CPU oracle and the CUDA library.

Recipes (all normals are standard unless stated, drawn from numpy's
PCG64 generator seeded by (seed, workload name, tensor name) -- q, k, v in
float32, directions in float64 -- then rounded to
the storage type with round-to-nearest-even):

* gaussian -- q, k, v ~ N(0, 1) everywhere.
* planted  -- as gaussian, plus, per sequence, one planted block b* drawn
              uniformly among the blocks that are remote-eligible for the last
              query block.  Per head, a unit direction u and a unit direction
              w orthogonal to it are drawn inside the coordinates of the two
              slowest rotary pairs (pair indices D/2-2 and D/2-1 under the
              rotate-half pairing, i.e. coordinates i and i + D/2), which turn
              by under 0.07 rad over the whole 384-token sequence.  The last
              block's queries get +alpha*u and the planted block's keys get
              +alpha*(c u + sqrt(1-c^2) w).  A block mean of bs standard
              normals adds noise of squared norm D/bs on average to the planted
              alpha, so c = 0.9*(alpha^2 + D/bs)/alpha^2 makes the expected
              cosine between the block-mean query and the block-mean planted
              key 0.9 (the workload's stated alignment).
* clusters -- v, q ~ N(0, 1).  Each key block draws one of n_clusters unit
              centres (uniformly, or Zipf(s) over cluster rank when zipf_s >
              0); every key of the block is sigma*N(0, I) plus the centre,
              which lives in the coordinates of the cluster_pairs slowest
              rotary pairs (D/8 pairs by default).  With one pair the centres
              are directions in the plane of the slowest pair: that is the
              only place where a cluster survives block averaging and 128K
              positions of rotation without the generator knowing the
              rotation, and it overflows the lists of the long workload.

Codebooks: P sets of K unit vectors of dimension D/P (Gaussian, normalised),
the seeded untrained-router control.

Upstream gradients (make_grad): dL/d(out) ~ N(0, 1), rounded to the storage
type like q, k, v.

Calibration records (make_records): rows = one of n_centres unit centres
times a log-normal length, plus sigma*N(0, I); optional zero rows and exact
copies of a row (edge cases of the calibration).
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass

import numpy as np

from .configs import Workload

ALPHA_PLANTED = 4.0
PLANTED_COS = 0.9        # stated alignment of the planted mean key with the last mean query
PLANTED_PAIRS = 2        # slowest rotary pairs that carry the planted directions


def rng_for(seed: int, *tags: str) -> np.random.Generator:
    h = hashlib.sha256(("/".join(tags)).encode()).digest()
    return np.random.default_rng([int(seed), int.from_bytes(h[:8], "little")])


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    rounded = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class Inputs:
    """Values in float32 (exactly the stored numbers) and the storage arrays."""
    q: np.ndarray            # [B,S,Hq,D] float32
    k: np.ndarray            # [B,S,Hkv,D] float32
    v: np.ndarray            # [B,S,Hkv,D] float32
    codebooks: np.ndarray    # [P,K,D/P] float32
    q_store: np.ndarray      # uint16 bf16 bits or float32
    k_store: np.ndarray
    v_store: np.ndarray
    planted: np.ndarray | None = None   # [B] planted block per sequence


def _store(x64: np.ndarray, dtype: str):
    x32 = x64.astype(np.float32)
    if dtype == "bf16":
        bits = f32_to_bf16_bits(x32)
        return bf16_bits_to_f32(bits), bits
    if dtype == "f32":
        return x32, x32
    raise ValueError(dtype)


def slow_pair_coords(D: int, npairs: int = 0) -> np.ndarray:
    """Coordinates of the npairs rotary pairs with the lowest frequencies
    (npairs = 0 -> D/8 pairs)."""
    half = D // 2
    i = np.arange(half - (npairs or D // 8), half)
    return np.concatenate([i, i + half])


def _normal(r: np.random.Generator, shape) -> np.ndarray:
    """Standard normals; large tensors are drawn in float32 (they are rounded
    to float32 or bfloat16 for storage anyway)."""
    return r.standard_normal(shape, dtype=np.float32)


def _unit(r: np.random.Generator, shape) -> np.ndarray:
    x = r.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def make_codebooks(w: Workload, seed: int) -> np.ndarray:
    r = rng_for(seed, w.name, "codebooks")
    return _unit(r, (w.P, w.K, w.D // w.P)).astype(np.float32)


def make_inputs(w: Workload, seed: int, *, keys: str | None = None,
                zero: bool = False) -> Inputs:
    keys = keys or w.keys
    B, S, Hq, Hkv, D, bs = w.B, w.S, w.Hq, w.Hkv, w.D, w.block
    nb = S // bs
    planted = None
    if zero:
        q = np.zeros((B, S, Hq, D))
        k = np.zeros((B, S, Hkv, D))
        v = _normal(rng_for(seed, w.name, "v"), (B, S, Hkv, D))
    else:
        q = _normal(rng_for(seed, w.name, "q"), (B, S, Hq, D))
        v = _normal(rng_for(seed, w.name, "v"), (B, S, Hkv, D))
        if keys == "gaussian":
            k = _normal(rng_for(seed, w.name, "k"), (B, S, Hkv, D))
        elif keys == "planted":
            k = _normal(rng_for(seed, w.name, "k"), (B, S, Hkv, D))
            r = rng_for(seed, w.name, "plant")
            last_eligible = nb - 1 - w.L
            assert last_eligible >= 0, "planted recipe needs a remote-eligible block"
            planted = r.integers(0, last_eligible + 1, size=B)
            coords = slow_pair_coords(D, PLANTED_PAIRS)
            m = coords.size
            g = Hq // Hkv
            c = min(1.0, PLANTED_COS * (ALPHA_PLANTED ** 2 + D / bs) / ALPHA_PLANTED ** 2)
            for b in range(B):
                for h in range(Hkv):
                    u = _unit(r, (m,))
                    x = r.standard_normal(m)
                    x -= x.dot(u) * u
                    wv = x / np.linalg.norm(x)
                    key_dir = c * u + np.sqrt(1.0 - c * c) * wv
                    kb = k[b, planted[b] * bs:(planted[b] + 1) * bs, h]
                    kb[:, coords] += ALPHA_PLANTED * key_dir[None, :]
                    for hq in range(h * g, (h + 1) * g):
                        qb = q[b, (nb - 1) * bs:nb * bs, hq]
                        qb[:, coords] += ALPHA_PLANTED * u[None, :]
        elif keys == "clusters":
            k = _cluster_keys(w, seed)
        else:
            raise ValueError(keys)
    qv, qs_ = _store(q, w.dtype)
    kv, ks_ = _store(k, w.dtype)
    vv, vs_ = _store(v, w.dtype)
    return Inputs(q=qv, k=kv, v=vv, codebooks=make_codebooks(w, seed),
                  q_store=qs_, k_store=ks_, v_store=vs_, planted=planted)


def _cluster_keys(w: Workload, seed: int) -> np.ndarray:
    B, S, Hkv, D, bs = w.B, w.S, w.Hkv, w.D, w.block
    nb = S // bs
    r = rng_for(seed, w.name, "k")
    coords = slow_pair_coords(D, w.cluster_pairs)
    C = w.n_clusters
    centres = _unit(r, (Hkv, C, coords.size))
    if w.zipf_s > 0:
        pr = np.arange(1, C + 1, dtype=np.float64) ** (-w.zipf_s)
        pr /= pr.sum()
    else:
        pr = np.full(C, 1.0 / C)
    k = w.sigma * _normal(r, (B, S, Hkv, D))
    member = r.choice(C, size=(B, Hkv, nb), p=pr)
    for b in range(B):
        for h in range(Hkv):
            cen = centres[h, member[b, h]]            # [nb, m]
            kh = k[b, :, h]                           # view [S, D]
            kh[:, coords] += np.repeat(cen, bs, axis=0)
    return k


def make_keys(w: Workload, seed: int):
    """The keys make_inputs(w, seed) would give (gaussian or clusters
    recipe), without drawing q and v: (k as stored, widened to float32;
    k in its storage type).  Used where only the index is built."""
    if w.keys == "gaussian":
        k = _normal(rng_for(seed, w.name, "k"), (w.B, w.S, w.Hkv, w.D))
    elif w.keys == "clusters":
        k = _cluster_keys(w, seed)
    else:
        raise ValueError(f"keys-only generation does not cover the {w.keys} recipe")
    return _store(k, w.dtype)


def make_records(N: int, D: int, n_centres: int, sigma: float, seed: int, *,
                 zero_rows: int = 0, repeat_rows: int = 0) -> np.ndarray:
    """Float32 records [N, D] for codebook calibration: each row is one of
    n_centres unit centres (Gaussian, normalised; drawn uniformly per row)
    scaled by a log-normal length, plus sigma*N(0, I).  zero_rows rows (at
    seeded positions) are set to 0; repeat_rows rows are copies of row 0."""
    r = rng_for(seed, "records", str(N), str(D), str(n_centres))
    c = r.standard_normal((n_centres, D))
    c /= np.linalg.norm(c, axis=1, keepdims=True)
    which = r.integers(0, n_centres, size=N)
    length = np.exp(0.5 * r.standard_normal(N))
    x = c[which] * length[:, None] + sigma * r.standard_normal((N, D))
    x = x.astype(np.float32)
    if zero_rows:
        x[r.choice(N, size=zero_rows, replace=False)] = 0.0
    if repeat_rows:
        x[r.choice(np.arange(1, N), size=repeat_rows, replace=False)] = x[0]
    return x


def make_grad(w: Workload, seed: int):
    """Upstream gradient dL/d(out) [B,S,Hq,D] ~ N(0, 1): (as stored, widened
    to float32; in its storage type)."""
    g = _normal(rng_for(seed, w.name, "dout"), (w.B, w.S, w.Hq, w.D))
    return _store(g, w.dtype)
