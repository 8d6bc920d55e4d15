"""The five workloads of the routed-attention forward, as plain data.

Each workload fixes the shapes, the routing parameters and the recipe of its
seeded synthetic inputs.  Nothing here computes any step of the method.

Shapes follow the pages' experiments:
  * tiny        -- a six-block fp32 case small enough to check by hand;
  * ar          -- six blocks, two of five eligible remote blocks selected, the
                   shape of the associative-recall run ("Monodratic: a
                   reproducible sparse attention mixer", section "Learned
                   sparse route");
  * capacity    -- 8,192 tokens at capacity 64, the shape of the capacity run
                   (same page, section "Capacity");
  * scaling     -- 4K..32K tokens, the range of the packed timing (same page,
                   section "Finite-range scaling"), extended to 128K;
  * long        -- 128K tokens with skewed key clusters that overflow the lists.
"""
from __future__ import annotations

from dataclasses import dataclass, replace, asdict


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    S: int
    Hq: int
    Hkv: int
    D: int
    block: int
    P: int
    K: int
    cap: int
    probes: int
    R: int
    L: int
    dtype: str = "bf16"          # storage type of q, k, v and the output
    rope_base: float = 10000.0
    scale: float = 0.0           # 0 -> 1/sqrt(D)
    keys: str = "gaussian"       # gaussian | planted | clusters
    n_clusters: int = 0
    zipf_s: float = 0.0          # 0 -> clusters drawn uniformly
    sigma: float = 0.0           # per-coordinate spread around a cluster centre
    cluster_pairs: int = 0       # slowest rotary pairs the centres live in (0 -> D/8)

    @property
    def nb(self) -> int:
        return self.S // self.block

    @property
    def A(self) -> int:
        return self.K ** self.P

    @property
    def n_sel(self) -> int:
        return self.R + self.L

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    def as_dict(self) -> dict:
        return asdict(self)


TINY = Workload("tiny", B=1, S=96, Hq=1, Hkv=1, D=32, block=16, P=2, K=8,
                cap=8, probes=2, R=2, L=1, dtype="f32")

AR = Workload("ar", B=64, S=384, Hq=4, Hkv=4, D=64, block=64, P=2, K=16,
              cap=16, probes=2, R=2, L=1, keys="planted")

CAPACITY = Workload("capacity", B=1, S=8192, Hq=15, Hkv=5, D=64, block=64,
                    P=2, K=16, cap=64, probes=2, R=8, L=2, keys="clusters",
                    n_clusters=32, sigma=0.3)


def scaling(S: int) -> Workload:
    return Workload(f"scaling{S // 1024}k", B=1, S=S, Hq=8, Hkv=8, D=128,
                    block=64, P=2, K=32, cap=64, probes=4, R=8, L=2)


SCALING_32K = scaling(32768)

LONG = Workload("long", B=1, S=131072, Hq=32, Hkv=8, D=128, block=128, P=2,
                K=64, cap=64, probes=4, R=16, L=2, keys="clusters",
                n_clusters=256, zipf_s=1.1, sigma=0.3, cluster_pairs=1)

ALL = {w.name: w for w in (TINY, AR, CAPACITY, SCALING_32K, LONG)}
SCALING_SWEEP = [scaling(S) for S in (4096, 8192, 16384, 32768, 65536, 131072)]
