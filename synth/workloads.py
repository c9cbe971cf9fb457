"""Shapes, layer schedules and seeded tensors of the five synthetic workloads.

Each workload is a decode (or prefill-chunk) call over one shared global KV
cache. Layer modes are 'FULL', 'REINDEX' and 'REUSE' ("CED: Continuing Context
with a Causal Encoder and Decoder", section "What Full, Reindex, and Reuse
Share", Fig. 5). Tensors are drawn lazily and cached; every tensor has its own
counter-based stream, so a smaller variant of a workload (fewer sequences,
a shorter cache) is a prefix-free redraw, not a slice.

Value recipe (the same on every side):
  * index queries/keys: uniform integers in [-127, 127] (int8);
  * head weights: uniform integers in [1, 8] (int32, one per indexer head, per layer);
  * main queries, local K and local V: N(0,1) rounded to bf16;
  * global KV before quantisation: N(0,1) as fp32.
Query positions are the last Tq positions of the cache; each sequence's local
KV holds the rows from ``local_base`` to N-1, enough for every query's window.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Dict, List

import numpy as np

from . import normal_bf16, normal_f32, randint_i8, randint_i32


@dataclass(frozen=True)
class LayerSpec:
    mode: str            # 'FULL' | 'REINDEX' | 'REUSE'
    k: int = 0           # top-k (FULL/REINDEX)
    P: int = 0           # candidate-pool size (FULL only; 0 = no pool)
    key_set: int = -1    # which int8 key set the layer scores (FULL/REINDEX)


@dataclass(frozen=True)
class WorkloadSpec:
    name: str
    B: int
    N: int
    Tq: int
    Hq: int
    D: int
    Hi: int
    Di: int
    W: int
    layers: tuple
    description: str = ""
    replay: bool = False  # bounded replay: local KV exists only for the Tq replayed positions
    m: int = 1            # sequence compression rate: N global entries cover m * N positions

    @property
    def L(self) -> int:
        return len(self.layers)

    @property
    def n_pos(self) -> int:
        return self.m * self.N

    @property
    def local_base(self) -> int:
        if self.replay:
            return self.n_pos - self.Tq
        return max(0, self.n_pos - self.Tq - self.W + 1)

    @property
    def Lloc(self) -> int:
        return self.n_pos - self.local_base

    @property
    def n_key_sets(self) -> int:
        return 1 + max(l.key_set for l in self.layers)


def _stack20_layers(k=2048, P=8192):
    layers, ks = [], 0
    for _ in range(5):
        layers.append(LayerSpec("FULL", k=k, P=P, key_set=ks)); ks += 1
        layers.append(LayerSpec("REUSE"))
        layers.append(LayerSpec("REUSE"))
        layers.append(LayerSpec("REINDEX", k=k, key_set=ks)); ks += 1
    return tuple(layers)


def _long_layers():
    layers = [LayerSpec("FULL", k=2048, P=8192, key_set=0)]
    for i in range(19):
        layers.append(LayerSpec("REINDEX", k=1024, key_set=0) if i % 2 == 0 else LayerSpec("REUSE"))
    return tuple(layers)


def _paper_layers(k=512, P=2048):
    # [Full + 3 Reuse] then 4 x [Reindex + 3 Reuse]: 1 Full, 4 Reindex, 15 Reuse.
    layers = [LayerSpec("FULL", k=k, P=P, key_set=0)] + [LayerSpec("REUSE")] * 3
    for _ in range(4):
        layers += [LayerSpec("REINDEX", k=k, key_set=0)] + [LayerSpec("REUSE")] * 3
    return tuple(layers)


CONFIGS: Dict[str, WorkloadSpec] = {
    "tiny": WorkloadSpec(
        "tiny", B=1, N=2048, Tq=16, Hq=8, D=64, Hi=4, Di=32, W=128,
        layers=(LayerSpec("FULL", k=256, P=0, key_set=0),),
        description="1 seq, 2048 cached positions, 16 decode queries, 8 heads x 64, "
                    "indexer 4x32, top-256, SWA 128, one Full layer"),
    "decode_full": WorkloadSpec(
        "decode_full", B=32, N=32768, Tq=1, Hq=16, D=128, Hi=8, Di=64, W=512,
        layers=(LayerSpec("FULL", k=2048, P=0, key_set=0),),
        description="32 seqs x 32768 positions, 1 decode query each, 16 heads x 128, "
                    "indexer 8x64, top-2048, SWA 512, one Full layer"),
    "stack20_128k": WorkloadSpec(
        "stack20_128k", B=16, N=131072, Tq=1, Hq=16, D=128, Hi=8, Di=64, W=512,
        layers=_stack20_layers(),
        description="16 seqs x 131072 positions, 20 layers [Full,Reuse,Reuse,Reindex]x5, "
                    "pool 8192, top-2048, own keys per Full/Reindex layer, SWA 512"),
    "prefill_chunk": WorkloadSpec(
        "prefill_chunk", B=1, N=69632, Tq=4096, Hq=32, D=128, Hi=8, Di=64, W=512,
        layers=(LayerSpec("FULL", k=2048, P=0, key_set=0),),
        description="4096 new positions appended to 65536 cached, 32 heads x 128, "
                    "indexer 8x64, top-2048 under the causal triangle, SWA 512"),
    "long_1m": WorkloadSpec(
        "long_1m", B=1, N=1 << 20, Tq=64, Hq=16, D=128, Hi=8, Di=64, W=1024,
        layers=_long_layers(),
        description="1 seq x 1048576 positions, 64 decode queries, layer 1 Full "
                    "(pool 8192, top-2048), layers 2-20 alternate Reindex (top-1024) and Reuse, "
                    "one shared key set, SWA 1024"),
    "replay_prefill": WorkloadSpec(
        "replay_prefill", B=4, N=131072, Tq=512, Hq=16, D=128, Hi=8, Di=64, W=512,
        layers=_stack20_layers(), replay=True,
        description="bounded-replay prefill: the last 512 of 131072 prompt positions of 4 seqs replayed "
                    "through 20 layers [Full,Reuse,Reuse,Reindex]x5 (pool 8192, top-2048), window 512 "
                    "with references before the replayed segment cut"),
    "encoder_m2": WorkloadSpec(
        "encoder_m2", B=16, N=65536, Tq=1, Hq=16, D=128, Hi=8, Di=64, W=512,
        layers=_stack20_layers(), m=2,
        description="encoder-side CSA2 at sequence compression rate 2: 16 seqs x 131072 positions in 65536 "
                    "global entries (each the mean of two positions), 20 layers [Full,Reuse,Reuse,Reindex]x5, "
                    "pool 8192, top-2048, SWA 512 over positions"),
    "paper_schedule": WorkloadSpec(
        "paper_schedule", B=16, N=131072, Tq=1, Hq=16, D=128, Hi=8, Di=64, W=128,
        layers=_paper_layers(),
        description="16 seqs x 131072 positions, 20 layers [Full+3 Reuse]+4x[Reindex+3 Reuse], "
                    "top-512, SWA 128, pool 2048, one shared key set"),
}

# tensor-id plan: every tensor gets its own stream
_TID_KV = 1
_TID_KEYSET = 100
_TID_LAYER = 1000


@dataclass
class Workload:
    spec: WorkloadSpec
    seed: int = 0
    _cache: dict = field(default_factory=dict, repr=False)

    def __getattr__(self, item):
        # expose the spec's fields (B, N, Tq, ...) directly
        if item.startswith("_") or item in ("spec", "seed"):
            raise AttributeError(item)
        return getattr(self.spec, item)

    def _get(self, key, fn):
        if key not in self._cache:
            self._cache[key] = fn()
        return self._cache[key]

    # shared tensors -------------------------------------------------------
    def q_pos(self) -> np.ndarray:
        s = self.spec
        return self._get("q_pos", lambda: np.broadcast_to(
            np.arange(s.n_pos - s.Tq, s.n_pos, dtype=np.int32), (s.B, s.Tq)).copy())

    def local_base_arr(self) -> np.ndarray:
        s = self.spec
        return self._get("local_base", lambda: np.full((s.B,), s.local_base, dtype=np.int32))

    def kv_f32(self) -> np.ndarray:
        """Global KV before quantisation (and, at compression rate m > 1, before the
        entries are formed): [B, m * N, D] fp32 per position, N(0,1)."""
        s = self.spec
        return self._get("kv", lambda: normal_f32(self.seed, _TID_KV, (s.B, s.n_pos, s.D)))

    def ki(self, key_set: int) -> np.ndarray:
        """int8 index keys [B, N, Di]."""
        s = self.spec
        return self._get(("ki", key_set), lambda: randint_i8(
            self.seed, _TID_KEYSET + key_set, (s.B, s.N, s.Di), -127, 127))

    # per-layer tensors ----------------------------------------------------
    def qi(self, layer: int) -> np.ndarray:
        s = self.spec
        return self._get(("qi", layer), lambda: randint_i8(
            self.seed, _TID_LAYER + 16 * layer + 0, (s.B, s.Tq, s.Hi, s.Di), -127, 127))

    def w(self, layer: int) -> np.ndarray:
        s = self.spec
        return self._get(("w", layer), lambda: randint_i32(
            self.seed, _TID_LAYER + 16 * layer + 1, (s.Hi,), 1, 8))

    def q(self, layer: int) -> np.ndarray:
        """Main queries, bf16 bits [B, Tq, Hq, D]."""
        s = self.spec
        return self._get(("q", layer), lambda: normal_bf16(
            self.seed, _TID_LAYER + 16 * layer + 2, (s.B, s.Tq, s.Hq, s.D)))

    def kl(self, layer: int) -> np.ndarray:
        """Local K, bf16 bits [B, Lloc, D]."""
        s = self.spec
        return self._get(("kl", layer), lambda: normal_bf16(
            self.seed, _TID_LAYER + 16 * layer + 3, (s.B, s.Lloc, s.D)))

    def vl(self, layer: int) -> np.ndarray:
        """Local V, bf16 bits [B, Lloc, D]."""
        s = self.spec
        return self._get(("vl", layer), lambda: normal_bf16(
            self.seed, _TID_LAYER + 16 * layer + 4, (s.B, s.Lloc, s.D)))

    def drop(self, *keys):
        for k in keys:
            self._cache.pop(k, None)


def make_workload(name: str, seed: int = 0, **overrides) -> Workload:
    """The named workload, optionally with fields replaced (e.g. B=2, N=4096)."""
    spec = CONFIGS[name]
    if overrides:
        spec = dataclasses.replace(spec, **overrides)
    return Workload(spec, seed)


def layer_modes(spec: WorkloadSpec) -> List[str]:
    return [l.mode for l in spec.layers]
