"""Seeded synthetic inputs for the Dust estimator workloads.

This module holds no step of the estimator: it only draws the inputs (layer
inputs X, weights W, targets, the synthetic direction u, sequence offsets)
that both the CUDA path and the CPU oracle consume, so that both see the same
bytes.  All randomness is numpy PCG64 with a fixed seed; the activation noise
itself is NOT drawn here (it is regenerated inside the kernels and inside the
oracle from the Philox specification).

Workload shapes follow the pages' setup (cnblogs Dust explainer, section
"结果：能打，但还贵": GPT-style model of width 512, 4096-token BPE vocabulary,
16k-token batches; population sweeps from 64 to 16k draws).  FineWeb and the
trained checkpoints are not available, so X ~ N(0, 1), W ~ N(0, 1/fan_in) and
uniform targets stand in for them.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal(shape, std: float = 1.0, seed: int = 0) -> np.ndarray:
    return (rng(seed).standard_normal(size=shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def targets(T: int, V: int, seed: int = 0) -> np.ndarray:
    return rng(seed).integers(0, V, size=T, dtype=np.int32)


def uniform_offsets(n_seq: int, L: int) -> np.ndarray:
    return (np.arange(n_seq + 1, dtype=np.int32) * np.int32(L)).astype(np.int32)


def offsets_from_lengths(lengths) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(np.asarray(lengths, np.int64))]).astype(np.int32)


def ragged_lengths(T: int, n_seq: int, seed: int = 0, allow_empty: bool = True) -> np.ndarray:
    """n_seq lengths summing to T (some may be 0 when allow_empty)."""
    r = rng(seed)
    if n_seq == 1:
        return np.array([T], np.int64)
    cuts = np.sort(r.integers(0 if allow_empty else 1, T + (1 if allow_empty else 0), size=n_seq - 1))
    if not allow_empty:
        cuts = np.unique(cuts)
        while len(cuts) < n_seq - 1:
            cuts = np.unique(np.concatenate([cuts, r.integers(1, T, size=n_seq - 1 - len(cuts))]))
        cuts = np.sort(cuts)
    edges = np.concatenate([[0], cuts, [T]])
    return np.diff(edges)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 to the nearest bfloat16 (ties to even); returned as float32 values."""
    b = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return (b.astype(np.uint32) << 16).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) of float32 values that are already bf16-exact."""
    return (np.ascontiguousarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


# ------------------------------------------------------------------ workloads

@dataclass(frozen=True)
class HiddenLayer:
    name: str
    d_in: int
    d_out: int
    layer: int          # Philox key word 1 for this layer's noise


@dataclass(frozen=True)
class Workload:
    """One configuration of the estimator hot path."""
    name: str
    n_seq: int
    seq_len: int
    K: int
    sigma: float = 1e-2
    gamma: float = 0.0
    dtype: str = "bf16"                     # layer-input / head-weight dtype
    hidden: tuple = ()                      # HiddenLayer entries
    head_d: int = 0                         # LM head input width (0: no head)
    V: int = 0
    Vc: int = 0
    head_layer: int = 0
    eps_scale: float = 0.01                 # synthetic-cost observation noise
    seed: int = 0
    notes: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return self.n_seq * self.seq_len


# Tiny LM-head step, fp32 (the oracle finishes it in seconds).
HEAD_SMALL = Workload("head_small_fp32", n_seq=1, seq_len=256, K=16, dtype="f32",
                      head_d=64, V=512, Vc=512, head_layer=0)

# Hidden layer scored by the toy causal suffix, fp32; gamma in {0, 0.9, 1.0}.
HIDDEN_SUFFIX = Workload("hidden_suffix_fp32", n_seq=4, seq_len=256, K=64, dtype="f32",
                         hidden=(HiddenLayer("linear256", 256, 256, 1),),
                         notes={"dh": 64, "V": 1024, "gammas": (0.0, 0.9, 1.0)})

# Pages-shaped LM head: 16 x 1024 tokens, width 512, vocab 4096 in chunks of 1024.
HEAD_PAGES = Workload("head_pages_bf16", n_seq=16, seq_len=1024, K=1024, dtype="bf16",
                      head_d=512, V=4096, Vc=1024, head_layer=2,
                      notes={"Ks": (64, 1024)})

# Estimator-only sweep over the linear shapes of an 8-layer width-512 GPT block.
HIDDEN_SWEEP = Workload("hidden_sweep_bf16", n_seq=16, seq_len=1024, K=1024, gamma=0.95,
                        dtype="bf16",
                        hidden=(HiddenLayer("qkv", 512, 1536, 3),
                                HiddenLayer("attn_out", 512, 512, 4),
                                HiddenLayer("mlp_up", 512, 2048, 5),
                                HiddenLayer("mlp_down", 2048, 512, 6)),
                        notes={"Ks": (64, 1024, 16384)})

# Scaled shape: d_model 1024, d_ff 4096, LM head V=4096, 64 x 1024 tokens, K=4096.
SCALED = Workload("scaled_d1024_ff4096_v4096", n_seq=64, seq_len=1024, K=4096, gamma=0.99,
                  dtype="bf16",
                  hidden=(HiddenLayer("mlp_up", 1024, 4096, 7),
                          HiddenLayer("mlp_down", 4096, 1024, 8)),
                  head_d=1024, V=4096, Vc=1024, head_layer=9,
                  notes={"gammas": (0.0, 0.99)})

WORKLOADS = {w.name: w for w in (HEAD_SMALL, HIDDEN_SUFFIX, HEAD_PAGES, HIDDEN_SWEEP, SCALED)}


def layer_inputs(w: Workload, layer: HiddenLayer, seed_offset: int = 0) -> dict:
    """X [T][d_in] (bf16-exact when w.dtype == 'bf16') and u [T][d_out] for one hidden layer."""
    X = normal((w.T, layer.d_in), 1.0, seed=1000 + layer.layer + seed_offset)
    if w.dtype == "bf16":
        X = bf16_round(X)
    u = normal((w.T, layer.d_out), 1.0, seed=2000 + layer.layer + seed_offset)
    return {"X": X, "u": u}


def head_inputs(w: Workload, seed_offset: int = 0) -> dict:
    """X [T][d], W [V][d] ~ N(0, 1/d) (bf16-exact when bf16), targets [T]."""
    X = normal((w.T, w.head_d), 1.0, seed=3000 + seed_offset)
    W = normal((w.V, w.head_d), 1.0 / np.sqrt(w.head_d), seed=3001 + seed_offset)
    if w.dtype == "bf16":
        X = bf16_round(X)
        W = bf16_round(W)
    y = targets(w.T, w.V, seed=3002 + seed_offset)
    return {"X": X, "W": W, "y": y}


def suffix_inputs(w: Workload, seed_offset: int = 0) -> dict:
    """Weights of the toy causal suffix behind HIDDEN_SUFFIX (all ~ N(0, 1/fan_in))."""
    layer = w.hidden[0]
    d, dh, V = layer.d_out, w.notes["dh"], w.notes["V"]
    s = 4000 + seed_offset
    return {
        "X": normal((w.T, layer.d_in), 1.0, seed=s),
        "W": normal((d, layer.d_in), 1.0 / np.sqrt(layer.d_in), seed=s + 1),
        "Wq": normal((dh, d), 1.0 / np.sqrt(d), seed=s + 2),
        "Wk": normal((dh, d), 1.0 / np.sqrt(d), seed=s + 3),
        "Wv": normal((dh, d), 1.0 / np.sqrt(d), seed=s + 4),
        "Wo": normal((d, dh), 1.0 / np.sqrt(dh), seed=s + 5),
        "Wout": normal((V, d), 1.0 / np.sqrt(d), seed=s + 6),
        "y": targets(w.T, V, seed=s + 7),
    }
