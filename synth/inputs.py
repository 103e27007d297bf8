"""Workload shapes and seeded bfloat16 input generation.

The workloads are the ones the attention pages describe: tensors of shape
(batch, seqlen, nheads, head_dim), last dimension contiguous, filled with
i.i.d. standard-normal values (the pages' own smoke tests draw ``randn``
tensors of that layout: "flash-attn install guide for CUDA 12.8 + PyTorch
2.7" (yfxerp.com), section 3.3; "RTX 5060 flash-attention" (pptc.cn),
section 4.4).  Some workloads scale the draws by 0.5.

Recipe (fixed here; the pages only say the inputs are random):
  * generator: numpy ``Generator(PCG64(seed))``;
  * draw order: Q, K, V, dO, each ``standard_normal`` in float32 of shape
    (B, S, H, D) (K and V with Hk heads when the key/value heads are
    grouped), multiplied by the workload's input scale;
  * round every value to bfloat16 (or IEEE float16 for the float16 tests)
    with round-to-nearest-even;
  * the CUDA path receives the bf16 bit patterns; the oracle receives the
    same values widened to float64.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np


@dataclass(frozen=True)
class AttnConfig:
    """One attention workload.

    ``variants`` lists the (causal, win_left, win_right) mask settings the
    workload is run with; -1 means "unbounded" for a window side.
    """

    name: str
    B: int
    H: int
    Sq: int
    Sk: int
    D: int
    input_scale: float
    seed: int
    variants: Tuple[Tuple[int, int, int], ...]
    backward: bool = False
    desc: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def visible_pairs(self, causal: int, win_left: int, win_right: int) -> int:
        """Count of (query, key) pairs the mask keeps, per (batch, head)."""
        delta = self.Sk - self.Sq
        total = 0
        for i in range(self.Sq):
            lo = 0
            hi = self.Sk - 1
            if win_left >= 0:
                lo = max(lo, i + delta - win_left)
            if causal:
                hi = min(hi, i + delta)
            if win_right >= 0:
                hi = min(hi, i + delta + win_right)
            if hi >= lo:
                total += hi - lo + 1
        return total


CONFIGS: List[AttnConfig] = [
    AttnConfig("c1_b1h2s128d64", 1, 2, 128, 128, 64, 1.0, 1001,
               ((0, -1, -1),), False,
               "fwd, batch 1, 2 heads, S=128, D=64, N(0,1), non-causal"),
    AttnConfig("c2_b2h16s2048d128_causal", 2, 16, 2048, 2048, 128, 1.0, 1002,
               ((1, -1, -1),), False,
               "fwd, batch 2, 16 heads, S=2048, D=128, N(0,1), causal"),
    AttnConfig("c3_b1h32s8192d128", 1, 32, 8192, 8192, 128, 0.5, 1003,
               ((1, -1, -1), (0, -1, -1)), False,
               "fwd, batch 1, 32 heads, S=8192, D=128, N(0,1)*0.5, causal and non-causal"),
    AttnConfig("c4_b1h32s32768d128_window", 1, 32, 32768, 32768, 128, 0.5, 1004,
               ((1, 4096, 0), (1, -1, -1)), False,
               "fwd, batch 1, 32 heads, S=32768, D=128, N(0,1)*0.5, causal with window (4096, 0) and full causal"),
    AttnConfig("c5_b1h32s8192d128_fwdbwd", 1, 32, 8192, 8192, 128, 0.5, 1005,
               ((1, -1, -1),), True,
               "fwd+bwd, batch 1, 32 heads, S=8192, D=128, Q/K/V/dO N(0,1)*0.5, causal"),
]


def config_by_name(name: str) -> AttnConfig:
    for c in CONFIGS:
        if c.name == name or c.name.startswith(name + "_"):
            return c
    raise KeyError(name)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return the bit patterns as uint16."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounding = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return ((u + rounding) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to float32 exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to IEEE float16 (nearest, ties to even); return the bit patterns as uint16."""
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def f16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen float16 bit patterns (uint16) to float32 exactly."""
    return np.ascontiguousarray(b, dtype=np.uint16).view(np.float16).astype(np.float32)


def bits_to_f32(b: np.ndarray, fmt: str = "bf16") -> np.ndarray:
    return f16_bits_to_f32(b) if fmt == "f16" else bf16_bits_to_f32(b)


def make_inputs(B: int, Sq: int, Sk: int, H: int, D: int, seed: int,
                input_scale: float = 1.0, with_dout: bool = False, Hk: Optional[int] = None,
                fmt: str = "bf16"):
    """Draw Q, K, V (and dO) for one workload.

    Returns a dict of 16-bit bit arrays (uint16; bfloat16, or IEEE float16 when
    fmt == "f16") with keys 'q', 'k', 'v' and, if requested, 'do'; Q and dO have
    shape (B, Sq, H, D), K and V (B, Sk, Hk, D) with Hk = H unless given
    (grouped K/V heads).  The float32 draws do not depend on fmt.
    """
    if fmt not in ("bf16", "f16"):
        raise ValueError(fmt)
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {}
    Hk = H if Hk is None else Hk
    shapes = [("q", Sq, H), ("k", Sk, Hk), ("v", Sk, Hk)]
    if with_dout:
        shapes.append(("do", Sq, H))
    for name, S, heads in shapes:
        x = rng.standard_normal((B, S, heads, D), dtype=np.float32)
        if input_scale != 1.0:
            x *= np.float32(input_scale)
        out[name] = f32_to_f16_bits(x) if fmt == "f16" else f32_to_bf16_bits(x)
    return out


def packed_lengths(total: int, lo: int, hi: int, seed: int) -> Tuple[int, ...]:
    """Sequence lengths of a packed batch of exactly ``total`` tokens: lengths
    drawn log-uniformly in [lo, hi] (numpy PCG64(seed)) until the total is
    reached, the last one cut to fit.  The mix of many short and a few long
    sequences is that of a packed fine-tuning batch."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out, used = [], 0
    while used < total:
        n = int(round(math.exp(rng.uniform(math.log(lo), math.log(hi)))))
        n = min(max(n, 1), total - used)
        out.append(n)
        used += n
    return tuple(out)


def make_config_inputs(cfg: AttnConfig, with_dout: Optional[bool] = None):
    wd = cfg.backward if with_dout is None else with_dout
    return make_inputs(cfg.B, cfg.Sq, cfg.Sk, cfg.H, cfg.D, cfg.seed, cfg.input_scale, wd)


def sample_rows(cfg: AttnConfig, n: int = 4096, seed: int = 7,
                extra_rows: Tuple[int, ...] = ()) -> np.ndarray:
    """Seeded (batch, head, row) triples for sampled comparison at large sizes.

    ``n`` triples are drawn without replacement; rows 0, 1 and Sq-1 of every
    (batch, head) are always added, plus ``extra_rows`` of every head.
    Returns an int64 array of shape (m, 3), sorted and unique.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    total = cfg.B * cfg.H * cfg.Sq
    n = min(n, total)
    flat = rng.choice(total, size=n, replace=False)
    b = flat // (cfg.H * cfg.Sq)
    h = (flat // cfg.Sq) % cfg.H
    i = flat % cfg.Sq
    trip = [np.stack([b, h, i], axis=1)]
    fixed = sorted({0, 1, cfg.Sq - 1, *[r for r in extra_rows if 0 <= r < cfg.Sq]})
    for bb in range(cfg.B):
        for hh in range(cfg.H):
            trip.append(np.array([[bb, hh, r] for r in fixed], dtype=np.int64))
    t = np.concatenate(trip, axis=0).astype(np.int64)
    t = np.unique(t, axis=0)
    return t
