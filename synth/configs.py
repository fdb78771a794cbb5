"""The five seeded synthetic MoE-layer workloads and their input recipe.

Shapes follow the Grok-1 layer described in "How does Grok-1 use a
mixture-of-experts design?" (n4n.ai), section "The high-level architecture":
8 experts, top-2, hidden 6144, expert_dim 32768.  Every tensor is drawn from
seed 0 with its own tensor id (see ``synth.normal``):

    x        id 1   (decode workload: call i uses id 100 + i)   N(0, 1)
    w_router id 2   [E, d]                                        N(0, 0.02)
    w_gate   id 3   [E, d, f]                                     N(0, 1/sqrt(d))
    w_up     id 4   [E, d, f]                                     N(0, 1/sqrt(d))
    w_down   id 5   [E, f, d]                                     N(0, 1/sqrt(f))

The second argument of N(.,.) is the standard deviation.  bf16 workloads round
every tensor once from double to bf16; the fp32 workload rounds to fp32.
Because ids and seed are shared, the three Grok-shape workloads see the same
expert weights, and the first rows of the skewed workload's x equal the
prefill workload's x.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from . import normal

SEED = 0
TID_X, TID_WR, TID_WG, TID_WU, TID_WD = 1, 2, 3, 4, 5
TID_X_DECODE_BASE = 100


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    f: int
    E: int = 8
    top_k: int = 2
    capacity_factor: float = 1.25
    dtype: str = "bf16"            # storage / compute type of x, weights and out
    logit_bias: tuple = field(default=None)
    calls: int = 1                 # distinct x tensors (decode workload: 100)
    description: str = ""

    @property
    def storage(self) -> str:
        return "f32" if self.dtype == "f32" else "bf16"


WORKLOADS = {
    "tiny_f32": Workload(
        "tiny_f32", T=64, d=256, f=1024, capacity_factor=1.25, dtype="f32",
        description="tiny fp32 layer, T=64 d=256 f=1024 E=8 k=2 cf=1.25"),
    "mid_bf16": Workload(
        "mid_bf16", T=2048, d=1536, f=8192, capacity_factor=1.25,
        description="mid bf16 layer, T=2048 d=1536 f=8192 E=8 k=2 cf=1.25"),
    "grok_prefill": Workload(
        "grok_prefill", T=8192, d=6144, f=32768, capacity_factor=4.0,
        description="Grok-1-shape prefill, T=8192 d=6144 f=32768 E=8 k=2, no drop (cf=E/k)"),
    "grok_decode": Workload(
        "grok_decode", T=32, d=6144, f=32768, capacity_factor=4.0, calls=100,
        description="Grok-1-shape decode, T=32 d=6144 f=32768 E=8 k=2, no drop, 100 calls"),
    "grok_skew": Workload(
        "grok_skew", T=16384, d=6144, f=32768, capacity_factor=1.25,
        logit_bias=(1.5, 0.5, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0),
        description="Grok-1-shape skewed routing, T=16384 d=6144 f=32768 E=8 k=2 cf=1.25, "
                    "logit bias +[1.5,0.5,0,...]"),
}


def x_tensor_id(call: int = 0, workload: Workload | None = None) -> int:
    if workload is not None and workload.calls > 1:
        return TID_X_DECODE_BASE + call
    return TID_X


def make_x(w: Workload, call: int = 0, rows=None) -> np.ndarray:
    """x [T, d] (or only the given contiguous row range ``rows=(r0, r1)``)."""
    r0, r1 = (0, w.T) if rows is None else rows
    return normal(SEED, x_tensor_id(call, w), (r1 - r0, w.d), std=1.0, dtype=w.storage, start=r0 * w.d)


def make_router(w: Workload) -> np.ndarray:
    return normal(SEED, TID_WR, (w.E, w.d), std=0.02, dtype=w.storage)


def make_w_gate(w: Workload) -> np.ndarray:
    return normal(SEED, TID_WG, (w.E, w.d, w.f), std=1.0 / math.sqrt(w.d), dtype=w.storage)


def make_w_up(w: Workload) -> np.ndarray:
    return normal(SEED, TID_WU, (w.E, w.d, w.f), std=1.0 / math.sqrt(w.d), dtype=w.storage)


def make_w_down(w: Workload) -> np.ndarray:
    return normal(SEED, TID_WD, (w.E, w.f, w.d), std=1.0 / math.sqrt(w.f), dtype=w.storage)


def make_bias(w: Workload):
    return None if w.logit_bias is None else np.asarray(w.logit_bias, dtype=np.float32)


def scaled(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields changed (for smaller parity cases)."""
    d = dict(w.__dict__)
    d.update(changes)
    return Workload(**d)
