"""Seeded synthetic inputs for the BERT-style encoder forward.

This module only draws random numbers and casts them to the storage type; it
holds none of the encoder's arithmetic.  Both the float64 oracle (through the
tests and the bench's CPU leg) and the CUDA library take their inputs from
here, so the two sides always see the same values.

Draw order (fixed, PCG64 seeded generator): x, then for each layer
Wqkv, bqkv, Wo, bo, W1, b1, W2, b2, gamma1, beta1, gamma2, beta2 (the LN
parameters are drawn only in the ``ln_affine_random`` variant), then
valid_len.  Values: x ~ N(0, 1); weights ~ N(0, 0.02); biases ~ N(0, 0.02)
or exactly 0; gamma = 1, beta = 0 unless ``ln_affine_random`` (then
gamma ~ N(1, 0.1), beta ~ N(0, 0.1)); valid_len ~ U{lo..hi}.

Weight layout is [in, out] row-major (y = x @ W + b); Wqkv's columns are
Q | K | V, and within each block head h owns columns h*d .. h*d+d-1.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional

import numpy as np

LAYER_KEYS = ("w_qkv", "b_qkv", "w_o", "b_o", "ln1_g", "ln1_b",
              "w_ff1", "b_ff1", "w_ff2", "b_ff2", "ln2_g", "ln2_b")

DTYPES = {"fp32": np.float32, "fp16": np.float16}


@dataclass(frozen=True)
class EncoderShape:
    head_num: int
    size_per_head: int
    ffn_dim: int
    num_layers: int

    @property
    def hidden(self) -> int:
        return self.head_num * self.size_per_head


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: encoder structure, batch shape and value recipe."""
    name: str
    shape: EncoderShape
    batch: int
    seq: int
    dtype: str                      # "fp32" or "fp16" (storage type)
    valid_lo: int
    valid_hi: int
    zero_bias: bool = False
    ln_affine_random: bool = False
    seed: int = 0
    weight_std: float = 0.02

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def tokens(self) -> int:
        return self.batch * self.seq


BERT_BASE = EncoderShape(12, 64, 3072, 12)
BERT_LARGE = EncoderShape(16, 64, 4096, 24)
PRUNED = EncoderShape(4, 32, 512, 12)
TINY_FP32 = EncoderShape(4, 32, 512, 1)


def named_workload(kind: str, batch: int, seq: Optional[int] = None) -> Workload:
    """The synthetic workloads the encoder is measured and checked on.

    kind: "tiny-fp32" (1 layer, 4x32, FFN 512, FP32, biases 0, all tokens valid),
    "bert-base-s32" (12x64, FFN 3072, 12 layers, valid_len in [1,32]),
    "pruned-s32" (4x32, FFN 512, 12 layers, valid_len in [8,32]),
    "bert-base" (seq 128 or 96, valid_len in [64,seq]),
    "bert-large" (16x64, FFN 4096, 24 layers, seq 128 or 512, valid_len in [seq/2,seq]).
    """
    if kind == "tiny-fp32":
        return Workload("tiny-fp32-1L-h128-s32-b1", TINY_FP32, batch, 32, "fp32",
                        32, 32, zero_bias=True)
    if kind == "bert-base-s32":
        return Workload(f"bert-base-12L-h768-s32-b{batch}-fp16", BERT_BASE, batch, 32,
                        "fp16", 1, 32)
    if kind == "pruned-s32":
        return Workload(f"pruned-12L-h128-s32-b{batch}-fp16", PRUNED, batch, 32, "fp16", 8, 32)
    if kind == "bert-base":
        s = 128 if seq is None else seq
        return Workload(f"bert-base-12L-h768-s{s}-b{batch}-fp16", BERT_BASE, batch, s,
                        "fp16", 64, s)
    if kind == "bert-large":
        s = 128 if seq is None else seq
        return Workload(f"bert-large-24L-h1024-s{s}-b{batch}-fp16", BERT_LARGE, batch, s,
                        "fp16", s // 2, s)
    raise ValueError(f"unknown workload kind {kind!r}")


@dataclass
class EncoderInputs:
    """Arrays in the storage dtype (what the GPU receives)."""
    workload: Workload
    x: np.ndarray                               # [B, S, H]
    valid_len: np.ndarray                       # [B] int32
    layers: List[Dict[str, np.ndarray]] = field(default_factory=list)

    def as_float64(self):
        """The same values widened to float64 (exact: widening does not round)."""
        return (self.x.astype(np.float64), self.valid_len.copy(),
                [{k: v.astype(np.float64) for k, v in lw.items()} for lw in self.layers])


def _draw_layer(rng: np.random.Generator, sh: EncoderShape, wl: Workload, dt) -> Dict[str, np.ndarray]:
    H, F = sh.hidden, sh.ffn_dim
    std = wl.weight_std

    def bias(n):
        if wl.zero_bias:
            return np.zeros(n, dt)
        return rng.normal(0.0, std, n).astype(dt)

    lw = {}
    lw["w_qkv"] = rng.normal(0.0, std, (H, 3 * H)).astype(dt)
    lw["b_qkv"] = bias(3 * H)
    lw["w_o"] = rng.normal(0.0, std, (H, H)).astype(dt)
    lw["b_o"] = bias(H)
    lw["w_ff1"] = rng.normal(0.0, std, (H, F)).astype(dt)
    lw["b_ff1"] = bias(F)
    lw["w_ff2"] = rng.normal(0.0, std, (F, H)).astype(dt)
    lw["b_ff2"] = bias(H)
    if wl.ln_affine_random:
        lw["ln1_g"] = rng.normal(1.0, 0.1, H).astype(dt)
        lw["ln1_b"] = rng.normal(0.0, 0.1, H).astype(dt)
        lw["ln2_g"] = rng.normal(1.0, 0.1, H).astype(dt)
        lw["ln2_b"] = rng.normal(0.0, 0.1, H).astype(dt)
    else:
        lw["ln1_g"] = np.ones(H, dt)
        lw["ln1_b"] = np.zeros(H, dt)
        lw["ln2_g"] = np.ones(H, dt)
        lw["ln2_b"] = np.zeros(H, dt)
    return lw


def make_inputs(wl: Workload) -> EncoderInputs:
    """Draw x, the per-layer weights and valid_len for one workload (see module doc)."""
    dt = DTYPES[wl.dtype]
    sh = wl.shape
    rng = np.random.Generator(np.random.PCG64(wl.seed))
    x = rng.standard_normal((wl.batch, wl.seq, sh.hidden)).astype(dt)
    layers = [_draw_layer(rng, sh, wl, dt) for _ in range(sh.num_layers)]
    lo = max(0, min(wl.valid_lo, wl.seq))
    hi = max(lo, min(wl.valid_hi, wl.seq))
    valid_len = rng.integers(lo, hi + 1, size=wl.batch).astype(np.int32)
    return EncoderInputs(wl, np.ascontiguousarray(x), valid_len, layers)


def random_array(shape, dtype: str, seed: int, std: float = 1.0, mean: float = 0.0) -> np.ndarray:
    """A seeded N(mean, std) array in the storage dtype (for single-step checks)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.normal(mean, std, shape).astype(DTYPES[dtype])


def sample_sequences(batch: int, count: int, valid_len: np.ndarray, seed: int = 1) -> np.ndarray:
    """A seeded sample of sequence indices that always holds the first, the last
    and one shortest sequence; the rest are drawn without replacement."""
    must = {0, batch - 1, int(np.argmin(valid_len))}
    rng = np.random.Generator(np.random.PCG64(seed))
    rest = [i for i in rng.permutation(batch).tolist() if i not in must]
    picked = sorted(must) + rest[: max(0, count - len(must))]
    return np.array(sorted(set(picked)), dtype=np.int64)


# ------------------------------------------------------------------ decoder inputs
DECODER_LAYER_KEYS = ("w_qkv", "b_qkv", "w_o", "b_o", "ln1_g", "ln1_b",
                      "w_q2", "b_q2", "w_kv2", "b_kv2", "w_o2", "b_o2", "ln2_g", "ln2_b",
                      "w_ff1", "b_ff1", "w_ff2", "b_ff2", "ln3_g", "ln3_b")


@dataclass(frozen=True)
class DecoderWorkload:
    """One synthetic decoder workload: target tokens y [B, T, H] attending to a
    memory (an encoder output) mem [B, S, H]."""
    name: str
    shape: EncoderShape
    batch: int
    tgt_seq: int
    mem_seq: int
    dtype: str
    tgt_lo: int
    tgt_hi: int
    mem_lo: int
    mem_hi: int
    ln_affine_random: bool = False
    seed: int = 0
    weight_std: float = 0.02

    def with_(self, **kw) -> "DecoderWorkload":
        return replace(self, **kw)


@dataclass
class DecoderInputs:
    workload: DecoderWorkload
    y: np.ndarray                               # [B, T, H]
    mem: np.ndarray                             # [B, S, H]
    tgt_len: np.ndarray                         # [B] int32
    mem_len: np.ndarray                         # [B] int32
    layers: List[Dict[str, np.ndarray]] = field(default_factory=list)

    def as_float64(self):
        return (self.y.astype(np.float64), self.tgt_len.copy(), self.mem.astype(np.float64), self.mem_len.copy(),
                [{k: v.astype(np.float64) for k, v in lw.items()} for lw in self.layers])


def make_decoder_inputs(wl: DecoderWorkload) -> DecoderInputs:
    """Draw order (PCG64, seed): y, mem, then per layer w_qkv, b_qkv, w_o, b_o,
    w_q2, b_q2, w_kv2, b_kv2, w_o2, b_o2, w_ff1, b_ff1, w_ff2, b_ff2 (weights and
    biases ~ N(0, weight_std)), then (ln_affine_random) gamma ~ N(1, 0.1) and
    beta ~ N(0, 0.1) of LayerNorms 1, 2, 3 (else 1 and 0), then tgt_len ~
    U{tgt_lo..tgt_hi} and mem_len ~ U{mem_lo..mem_hi}.  y, mem ~ N(0, 1)."""
    dt = DTYPES[wl.dtype]
    sh = wl.shape
    H, F = sh.hidden, sh.ffn_dim
    std = wl.weight_std
    rng = np.random.Generator(np.random.PCG64(wl.seed))
    y = rng.standard_normal((wl.batch, wl.tgt_seq, H)).astype(dt)
    mem = rng.standard_normal((wl.batch, wl.mem_seq, H)).astype(dt)
    layers = []
    for _ in range(sh.num_layers):
        lw = {}
        for name, shp in (("w_qkv", (H, 3 * H)), ("b_qkv", (3 * H,)), ("w_o", (H, H)), ("b_o", (H,)),
                          ("w_q2", (H, H)), ("b_q2", (H,)), ("w_kv2", (H, 2 * H)), ("b_kv2", (2 * H,)),
                          ("w_o2", (H, H)), ("b_o2", (H,)), ("w_ff1", (H, F)), ("b_ff1", (F,)),
                          ("w_ff2", (F, H)), ("b_ff2", (H,))):
            lw[name] = rng.normal(0.0, std, shp).astype(dt)
        for i in (1, 2, 3):
            if wl.ln_affine_random:
                lw[f"ln{i}_g"] = rng.normal(1.0, 0.1, H).astype(dt)
                lw[f"ln{i}_b"] = rng.normal(0.0, 0.1, H).astype(dt)
            else:
                lw[f"ln{i}_g"] = np.ones(H, dt)
                lw[f"ln{i}_b"] = np.zeros(H, dt)
        layers.append(lw)
    tlo = max(0, min(wl.tgt_lo, wl.tgt_seq)); thi = max(tlo, min(wl.tgt_hi, wl.tgt_seq))
    mlo = max(0, min(wl.mem_lo, wl.mem_seq)); mhi = max(mlo, min(wl.mem_hi, wl.mem_seq))
    tgt_len = rng.integers(tlo, thi + 1, size=wl.batch).astype(np.int32)
    mem_len = rng.integers(mlo, mhi + 1, size=wl.batch).astype(np.int32)
    return DecoderInputs(wl, np.ascontiguousarray(y), np.ascontiguousarray(mem), tgt_len, mem_len, layers)
