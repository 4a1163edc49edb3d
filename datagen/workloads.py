"""Workload shapes of the decode-attention path and their seeded inputs.

Shapes only (no arithmetic of the method).  Each workload is one layer type at
one batch/context; ``seed`` and ``layer`` select independent streams.

Input recipe (both the CUDA path and the oracle read these bytes):
* raw shared states S, compressed rows, window rows, attention queries and
  states to quantise: Irwin-Hall(12) - 6 ~ N(0,1), rounded to bf16;
* indexer queries and bf16 indexer keys: integers uniform in [-8, 8] (bf16);
* fp4 indexer keys: E2M1 magnitude codes 0..6 with a random sign and every
  16-channel scale 2.0, so keys dequantise to integers in [-8, 8];
* compression weights: per-tap, per-channel softmax of N(0,1) logits (fp32).
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import datagen as D

DIM, IDX_DIM, WINDOW, TOPK = 512, 128, 128, 512


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str          # "c4a" (indexer + sparse) or "c128a" (dense)
    batch: int
    t: int             # context length = position of the decode query
    heads: int
    main_fmt: int = 0  # 0 bf16, 1 fp8 row, 2 fp4 g16
    index_fmt: int = 0  # 0 bf16, 2 fp4 g16
    window: int = WINDOW
    k: int = TOPK

    @property
    def stride(self) -> int:
        return 4 if self.kind == "c4a" else 128

    @property
    def taps(self) -> int:
        return 8 if self.kind == "c4a" else 128

    @property
    def n(self) -> int:
        return max(0, (self.t - self.window) // self.stride)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY_C4A = Workload("tiny c4a B=1 t=2048 H=16", "c4a", 1, 2048, 16)
C128A_B8 = Workload("c128a B=8 t=131072 H=64", "c128a", 8, 131072, 64)
C4A_B32 = Workload("c4a B=32 t=131072 H=64", "c4a", 32, 131072, 64)
STACK_C4A = Workload("stack c4a layer B=1 t=1048576 H=64", "c4a", 1, 1 << 20, 64)
STACK_C128A = Workload("stack c128a layer B=1 t=1048576 H=64", "c128a", 1, 1 << 20, 64)
Q_C4A_FP8 = Workload("c4a B=64 t=262144 fp8 main fp4 index", "c4a", 64, 262144, 64, 1, 2)
Q_C4A_FP4 = Workload("c4a B=64 t=262144 fp4 main fp4 index", "c4a", 64, 262144, 64, 2, 2)
Q_C128A_FP8 = Workload("c128a B=64 t=262144 fp8 main", "c128a", 64, 262144, 64, 1, 0)
Q_C128A_FP4 = Workload("c128a B=64 t=262144 fp4 main", "c128a", 64, 262144, 64, 2, 0)

# The 61-layer stack: layer l is c128a when l is even, c4a when l is odd
# (30 c4a + 31 c128a).
STACK_LAYERS = 61


def stack_layer_kind(layer: int) -> str:
    return "c128a" if layer % 2 == 0 else "c4a"


def keys_for(seed: int, layer: int) -> dict:
    """Stream keys of every input tensor of one layer."""
    return {
        "raw": D.stream_key(seed, D.TID_RAW_S, layer),
        "comp": D.stream_key(seed, D.TID_COMP, layer),
        "win": D.stream_key(seed, D.TID_WIN, layer),
        "q": D.stream_key(seed, D.TID_Q, layer),
        "qidx": D.stream_key(seed, D.TID_QIDX, layer),
        "kidx": D.stream_key(seed, D.TID_KIDX, layer),
        "kidx_fp4": D.stream_key(seed, D.TID_KIDX_FP4, layer),
        "states": D.stream_key(seed, D.TID_STATES, layer),
    }
