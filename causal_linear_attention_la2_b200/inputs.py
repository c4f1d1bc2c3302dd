"""Seeded synthetic inputs and the named workloads.

This module is shared by the tests, the benchmark and the smoke check; it
holds none of the attention arithmetic, only how inputs are drawn.  It imports
neither the CUDA binding nor the oracle, so both sides can be fed the same
tensors.

Recipe (every workload): a CPU ``torch.Generator`` seeded with ``seed`` draws,
in this order, q, k, v and dO, each ``randn`` in float32 of shape [B,H,T,d]
(q, k) or [B,H,T,e] (v, dO).  q, k and v are multiplied by d**-0.5; dO is left
N(0,1).  For bf16 workloads all four are then rounded to bf16 (round to
nearest even).  The decay of head h is computed in float64 and rounded once to
float32, and that float32 value is what both the GPU path and the oracle use.
These shapes stand in for the attention layers of the TransNormerLLM models
that the Lightning Attention-2 pages train (no dataset is involved).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


def decay_tnl(H: int) -> np.ndarray:
    """lambda_h = 1 - 2^-(5 + 8h/H), h = 0..H-1, rounded once to float32."""
    h = np.arange(H, dtype=np.float64)
    return (1.0 - np.exp2(-(5.0 + 8.0 * h / H))).astype(np.float32)


def decay_tiny(H: int) -> np.ndarray:
    """lambda_h = 1 - 2^-(5 + h) (exact in float32 for small h)."""
    h = np.arange(H, dtype=np.float64)
    return (1.0 - np.exp2(-(5.0 + h))).astype(np.float32)


def decay_ones(H: int) -> np.ndarray:
    """lambda_h = 1: plain (undecayed) causal linear attention."""
    return np.ones(H, dtype=np.float32)


_DECAYS = {"tnl": decay_tnl, "tiny": decay_tiny, "ones": decay_ones}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    d: int
    e: int
    block: int
    dtype: str  # "bf16" or "f32"
    decay: str = "tnl"
    note: str = field(default="", compare=False)

    @property
    def sequences(self) -> int:
        return self.B * self.H

    @property
    def tokens(self) -> int:
        return self.B * self.T

    def decays(self) -> np.ndarray:
        return _DECAYS[self.decay](self.H)


def sweep_workload(T: int, block: int = 128) -> Workload:
    """Length sweep at a fixed 131,072 tokens per step (B = 131072 // T, at least 1)."""
    B = max(1, 131072 // T)
    return Workload(f"sweep_T{T}_blk{block}", B, 32, T, 128, 128, block, "bf16")


SWEEP_T = (1024, 4096, 16384, 32768, 65536, 92160, 131072)

WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 2, 512, 64, 64, 64, "f32", "tiny",
                         "tiny fp32 case the oracle finishes in well under a second"),
    "tnl400m": Workload("tnl400m", 8, 16, 2048, 64, 64, 128, "bf16", "tnl",
                        "TNL-400M-shaped attention layer"),
    "long": Workload("long", 1, 16, 65536, 128, 128, 128, "bf16", "tnl",
                     "long-context layer"),
    "tnl15b": Workload("tnl15b", 2, 40, 6144, 128, 128, 128, "bf16", "tnl",
                       "TNL-15B-shaped attention layer (d_model 5120, 40 heads)"),
    "tnl15b_nodecay": Workload("tnl15b_nodecay", 2, 40, 6144, 128, 128, 128, "bf16", "ones",
                               "TNL-15B-shaped layer with lambda = 1"),
}
for _T in SWEEP_T:
    for _blk in (128, 256):
        _w = sweep_workload(_T, _blk)
        WORKLOADS[_w.name] = _w

# The launch plan of the T = 131,072 sweep point (32 sequences: a forward in
# four segments with a state pre-pass, a backward of 96 one-segment units) at
# an eighth of its length, so that a full profiler capture holds about 1.7 GB
# on the device; per-launch DRAM traffic scales to the full length by 8.
WORKLOADS["sweep_plan_T16384"] = Workload(
    "sweep_plan_T16384", 1, 32, 16384, 128, 128, 128, "bf16", "tnl",
    "profiling shape: the T = 131,072 sweep point's launch plan at 1/8 of its length")


# Decode-step shapes: one new token for each of B sequences of H heads, the
# heads of the TNL-15B and TNL-400M layers at serving batch sizes (the fp32
# states, 168 MB and 33.5 MB, are larger than or comparable to the L2).
DECODE_WORKLOADS = {
    "decode_tnl15b": Workload("decode_tnl15b", 64, 40, 1, 128, 128, 128, "bf16", "tnl",
                              "decode step, TNL-15B heads, batch 64"),
    "decode_tnl400m": Workload("decode_tnl400m", 128, 16, 1, 64, 64, 128, "bf16", "tnl",
                               "decode step, TNL-400M heads, batch 128"),
}


def make_inputs(B: int, H: int, T: int, d: int, e: int, dtype: str = "bf16",
                seed: int = 0, decay: str = "tnl"):
    """Return dict(q, k, v, do, lam) as CPU tensors (lam: float32 [H])."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    scale = float(d) ** -0.5
    q = torch.randn(B, H, T, d, generator=g, dtype=torch.float32) * scale
    k = torch.randn(B, H, T, d, generator=g, dtype=torch.float32) * scale
    v = torch.randn(B, H, T, e, generator=g, dtype=torch.float32) * scale
    do = torch.randn(B, H, T, e, generator=g, dtype=torch.float32)
    if dtype == "bf16":
        q, k, v, do = (x.to(torch.bfloat16) for x in (q, k, v, do))
    elif dtype != "f32":
        raise ValueError(f"unknown dtype {dtype!r}")
    lam = torch.from_numpy(_DECAYS[decay](H).copy())
    return {"q": q, "k": k, "v": v, "do": do, "lam": lam}


def make_workload_inputs(w: Workload, seed: int = 0):
    return make_inputs(w.B, w.H, w.T, w.d, w.e, w.dtype, seed, w.decay)
