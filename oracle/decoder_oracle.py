"""Float64 CPU oracle for the post-LN Transformer decoder forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, the graft entry's smoke check and
the bench's CPU-baseline leg may import this module.  The CUDA library never
calls it and shares no code with it.

Source page: "有钱任性：英伟达训练80亿参数量GPT-2，1475块V100 53分钟训练BERT"
(机器之心, the Faster Transformer write-up), cited as [FT].  [FT] "什么是
Faster Transformer" says the first release covers the encoder and that a
decoder follows in a later release; the page gives no decoder design.  The
reading used here is the plain post-LN Transformer decoder layer run over a
whole target sequence (every target token at once, as in training or
scoring), with the encoder's conventions (LayerNorm epsilon 1e-12, biased
variance, erf GELU, scale 1/sqrt(d), masked keys weigh exactly 0):
  1. masked self-attention over the target: query i attends to keys j with
     j <= i and j < nt (nt = clamp(tgt_len, 0, T));  H1 = LN1(y + A1 Wo + bo);
  2. cross-attention from the target to the memory (the encoder output):
     Q = H1 Wq2 + bq2, [K | V] = mem Wkv2 + bkv2, keys j < nm
     (nm = clamp(mem_len, 0, S));  H2 = LN2(H1 + A2 Wo2 + bo2);
  3. FFN:  out = LN3(H2 + GELU(H2 W1 + b1) W2 + b2).
Query rows i >= nt are computed but not meaningful; a row whose keys are all
masked (nt = 0, or nm = 0 for cross-attention) has ctx = 0.

The method is exact, so this is the definition written out.  Library
primitives: numpy matmul and exp; the LayerNorm, GELU and masked softmax of
encoder_oracle.py.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

from oracle.encoder_oracle import GELU, layer_norm


def _softmax_rows(scores: np.ndarray, limits: Sequence[int]) -> np.ndarray:
    """Row r of scores [R, K] over keys j < limits[r] (probability 0 elsewhere;
    an all-zero row when limits[r] <= 0)."""
    p = np.zeros_like(scores)
    for r, lim in enumerate(limits):
        if lim <= 0:
            continue
        s = scores[r, :lim]
        e = np.exp(s - s.max())
        p[r, :lim] = e / e.sum()
    return p


def self_attention_causal(q: np.ndarray, k: np.ndarray, v: np.ndarray, nt: int) -> np.ndarray:
    """One (sequence, head): q, k, v [T, d]; query i attends to keys j <= i, j < nt."""
    T, d = q.shape
    limits = [min(i + 1, nt) for i in range(T)]
    return _softmax_rows((q @ k.T) / math.sqrt(d), limits) @ v


def cross_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, nm: int) -> np.ndarray:
    """One (sequence, head): q [T, d] against memory keys k, v [S, d], keys j < nm."""
    T, d = q.shape
    return _softmax_rows((q @ k.T) / math.sqrt(d), [nm] * T) @ v


def _heads(x2d: np.ndarray, nh: int, d: int) -> List[np.ndarray]:
    """[R, nh*d] -> per-head [R, d] blocks (head h = columns h*d .. h*d+d-1)."""
    return [x2d[:, h * d:(h + 1) * d] for h in range(nh)]


def decoder_layer(y: np.ndarray, tgt_len: Sequence[int], mem: np.ndarray, mem_len: Sequence[int],
                  lw: Dict[str, np.ndarray], head_num: int, size_per_head: int, gelu: str = "erf") -> np.ndarray:
    """One post-LN decoder layer over y [B, T, H] with memory mem [B, S, H]."""
    B, T, H = y.shape
    S = mem.shape[1]
    nh, d = head_num, size_per_head
    out = np.empty_like(y)
    for b in range(B):
        nt = int(min(max(int(tgt_len[b]), 0), T))
        nm = int(min(max(int(mem_len[b]), 0), S))
        x = y[b]
        qkv = x @ lw["w_qkv"] + lw["b_qkv"]                          # Q | K | V columns
        qs, ks, vs = _heads(qkv[:, :H], nh, d), _heads(qkv[:, H:2 * H], nh, d), _heads(qkv[:, 2 * H:], nh, d)
        ctx = np.concatenate([self_attention_causal(qs[h], ks[h], vs[h], nt) for h in range(nh)], axis=1)
        h1 = layer_norm(x + ctx @ lw["w_o"] + lw["b_o"], lw["ln1_g"], lw["ln1_b"])
        q2 = h1 @ lw["w_q2"] + lw["b_q2"]
        kv2 = mem[b] @ lw["w_kv2"] + lw["b_kv2"]                      # K | V columns
        q2s, k2s, v2s = _heads(q2, nh, d), _heads(kv2[:, :H], nh, d), _heads(kv2[:, H:], nh, d)
        ctx2 = np.concatenate([cross_attention(q2s[h], k2s[h], v2s[h], nm) for h in range(nh)], axis=1)
        h2 = layer_norm(h1 + ctx2 @ lw["w_o2"] + lw["b_o2"], lw["ln2_g"], lw["ln2_b"])
        u = GELU[gelu](h2 @ lw["w_ff1"] + lw["b_ff1"])
        out[b] = layer_norm(h2 + u @ lw["w_ff2"] + lw["b_ff2"], lw["ln3_g"], lw["ln3_b"])
    return out


def decoder_forward(y: np.ndarray, tgt_len: Sequence[int], mem: np.ndarray, mem_len: Sequence[int],
                    layers: List[Dict[str, np.ndarray]], head_num: int, size_per_head: int,
                    seqs: Optional[Sequence[int]] = None, gelu: str = "erf") -> np.ndarray:
    """The decoder stack: Y_0 = y, Y_{l+1} = layer_l(Y_l, mem), output Y_L.  Every
    layer attends to the same memory.  ``seqs`` restricts the work to a subset
    of the batch (sequences never interact)."""
    y = np.asarray(y, dtype=np.float64)
    mem = np.asarray(mem, dtype=np.float64)
    tl, ml = np.asarray(tgt_len), np.asarray(mem_len)
    if seqs is not None:
        idx = np.asarray(list(seqs), dtype=np.int64)
        y, mem, tl, ml = y[idx], mem[idx], tl[idx], ml[idx]
    for lw in layers:
        y = decoder_layer(y, tl, mem, ml, lw, head_num, size_per_head, gelu)
    return y
