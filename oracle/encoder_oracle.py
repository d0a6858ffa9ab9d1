"""Float64 CPU oracle for the post-LN BERT encoder forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, the graft entry's smoke check and
the bench's CPU-baseline leg may import this module.  The CUDA library never
calls it and shares no code with it.

Source page: "有钱任性：英伟达训练80亿参数量GPT-2，1475块V100 53分钟训练BERT"
(机器之心, the Faster Transformer write-up), cited below as [FT] with its
section title.  The page describes the encoder forward ([FT] "什么是 Faster
Transformer"): a stack of Transformer encoder layers whose structure is set
by head_num and size_per_head, run over batch_size sequences of a maximum
length.  Its layer figure ([FT] "Faster Transformer 优化原理", figure
"BERT 中 Transformer Layer 的计算流程图") did not survive, so the per-layer
order is the plain post-LN encoder layer: QKV projection; per-head scaled
QK^T with the padding mask; softmax; PV; output projection;
bias + residual + LayerNorm; FFN with GELU; bias + residual + LayerNorm.

The method is exact (no approximation or iteration), so this oracle is the
definition written out.  Library primitives: numpy matmul, numpy exp/sqrt,
scipy.special.erf.  No blocking, fusion or reordering beyond the definition.

Readings where the page is silent (each also listed in the design notes):
  * LayerNorm epsilon = 1e-12, biased variance (divide by H).
  * GELU is the erf form 0.5*t*(1+erf(t/sqrt 2)); the tanh form (the page's
    "x*x*x" remark) is available as gelu="tanh".
  * Scores are scaled by 1/sqrt(size_per_head).
  * Masking excludes keys j >= n (weight exactly 0); n = clamp(valid_len, 0, S);
    query rows i >= n are still computed; n == 0 gives ctx = 0.
  * x is already the hidden states (no embeddings, no positional terms).
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np
from scipy.special import erf as _erf

LN_EPS = 1e-12
_SQRT2 = math.sqrt(2.0)
_SQRT_2_OVER_PI = math.sqrt(2.0 / math.pi)


def gelu_erf(t: np.ndarray) -> np.ndarray:
    """GELU(t) = t * Phi(t) = 0.5 t (1 + erf(t / sqrt 2)).

    [FT] "Faster Transformer 优化原理": GELU is the FFN activation (figure 1,
    the TensorFlow timeline of GELU).  The erf form is the exact definition.
    """
    return 0.5 * t * (1.0 + _erf(t / _SQRT2))


def gelu_tanh(t: np.ndarray) -> np.ndarray:
    """tanh approximation 0.5 t (1 + tanh(sqrt(2/pi) (t + 0.044715 t^3))).

    [FT] "Faster Transformer 优化原理": the page builds GELU from Pow/Add/Tanh
    and replaces pow(x, 3) by x*x*x, which is this form.
    """
    return 0.5 * t * (1.0 + np.tanh(_SQRT_2_OVER_PI * (t + 0.044715 * t * t * t)))


GELU = {"erf": gelu_erf, "tanh": gelu_tanh}


def layer_norm(z: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float = LN_EPS) -> np.ndarray:
    """Row-wise LayerNorm over the last axis: gamma * (z - mu) / sqrt(var + eps) + beta,
    mu = mean(z), var = mean((z - mu)^2) (biased).

    [FT] "Faster Transformer 优化原理": Layer Normalization (its TensorFlow
    timeline figure) with sums taken in higher precision and 1/sqrt.
    """
    mu = z.mean(axis=-1, keepdims=True)
    dev = z - mu
    var = (dev * dev).mean(axis=-1, keepdims=True)
    return gamma * (dev / np.sqrt(var + eps)) + beta


def softmax_masked(scores: np.ndarray, n: int) -> np.ndarray:
    """Softmax over the key axis of one score block [rows, S], keys j >= n
    excluded (probability exactly 0).  Subtracting the row max does not change
    the exact value.  n == 0 gives an all-zero block.

    [FT] "Faster Transformer 优化原理": SoftMax, with row reductions (max, sum).
    """
    p = np.zeros_like(scores)
    if n <= 0:
        return p
    s = scores[:, :n]
    e = np.exp(s - s.max(axis=1, keepdims=True))
    p[:, :n] = e / e.sum(axis=1, keepdims=True)
    return p


def qkv_projection(x2d: np.ndarray, w_qkv: np.ndarray, b_qkv: np.ndarray) -> np.ndarray:
    """QKV = X Wqkv + bqkv over all tokens: [M,H] x [H,3H] -> [M,3H].

    [FT] "Faster Transformer 优化原理": the Q, K and V projections are three
    of the eight matrix multiplies of a layer.
    """
    return x2d @ w_qkv + b_qkv


def head_split(qkv2d: np.ndarray, batch: int, seq: int, head_num: int, size_per_head: int) -> np.ndarray:
    """[M,3H] -> [3, B, nh, S, d]:  out[t, b, h, s, :] = qkv[b*S+s, t*H + h*d : t*H + (h+1)*d].

    [FT] "Faster Transformer 优化原理": one of the six custom kernels adds the
    bias and rearranges the projections into per-head blocks (the bias is added
    in qkv_projection here).
    """
    H = head_num * size_per_head
    t = qkv2d.reshape(batch, seq, 3, head_num, size_per_head)
    out = np.empty((3, batch, head_num, seq, size_per_head), dtype=qkv2d.dtype)
    for which in range(3):
        for h in range(head_num):
            out[which, :, h, :, :] = t[:, :, which, h, :]
    assert out.shape[-1] * head_num == H
    return out


def attention(qkv_split: np.ndarray, valid_len: Sequence[int], seqs: Optional[Sequence[int]] = None) -> np.ndarray:
    """Masked scaled-dot-product attention with heads merged back.

    qkv_split: [3, B, nh, S, d].  For sequence b with n = clamp(valid_len[b], 0, S)
    and head h:  Sc = Q K^T / sqrt(d);  P = softmax over keys j < n;  ctx = P V.
    Returns ctx as [len(seqs), S, nh*d] with head h in columns h*d .. h*d+d-1.

    [FT] "Faster Transformer 优化原理": the batched QK^T and PV multiplies, the
    SoftMax kernel between them and the transpose that merges heads.
    """
    _, B, nh, S, d = qkv_split.shape
    if seqs is None:
        seqs = range(B)
    seqs = list(seqs)
    ctx = np.zeros((len(seqs), S, nh * d))
    scale = 1.0 / math.sqrt(d)
    for out_i, b in enumerate(seqs):
        n = int(min(max(int(valid_len[b]), 0), S))
        for h in range(nh):
            q = qkv_split[0, b, h]
            k = qkv_split[1, b, h]
            v = qkv_split[2, b, h]
            p = softmax_masked((q @ k.T) * scale, n)
            ctx[out_i, :, h * d:(h + 1) * d] = p @ v
    return ctx


def bias_residual_layernorm(a: np.ndarray, bias: np.ndarray, resid: np.ndarray,
                            gamma: np.ndarray, beta: np.ndarray) -> np.ndarray:
    """LN(resid + a + bias) row-wise.

    [FT] "Faster Transformer 优化原理": add-bias + residual + Layer Normalization
    is one fused custom kernel (it runs twice per layer).
    """
    return layer_norm(resid + a + bias, gamma, beta)


def ffn1_gelu(h1: np.ndarray, w_ff1: np.ndarray, b_ff1: np.ndarray, gelu: str = "erf") -> np.ndarray:
    """U = GELU(H1 W1 + b1).  [FT] "Faster Transformer 优化原理": GEMM + add-bias/GELU kernel."""
    return GELU[gelu](h1 @ w_ff1 + b_ff1)


def encoder_layer(x: np.ndarray, valid_len: Sequence[int], lw: Dict[str, np.ndarray],
                  head_num: int, size_per_head: int, gelu: str = "erf") -> np.ndarray:
    """One post-LN encoder layer over a batch x [B, S, H] (float64).

    QKV projection -> head split -> masked scaled softmax attention (heads merged)
    -> output projection -> bias + residual + LN -> FFN1 + GELU -> FFN2
    -> bias + residual + LN.  [FT] "什么是 Faster Transformer" (the layer is the
    unit of the encoder stack) and "Faster Transformer 优化原理" (its kernels).
    """
    B, S, H = x.shape
    x2d = x.reshape(B * S, H)
    qkv = qkv_projection(x2d, lw["w_qkv"], lw["b_qkv"])
    ctx = attention(head_split(qkv, B, S, head_num, size_per_head), valid_len).reshape(B * S, H)
    a = ctx @ lw["w_o"]
    h1 = bias_residual_layernorm(a, lw["b_o"], x2d, lw["ln1_g"], lw["ln1_b"])
    u = ffn1_gelu(h1, lw["w_ff1"], lw["b_ff1"], gelu)
    y = u @ lw["w_ff2"]
    out = bias_residual_layernorm(y, lw["b_ff2"], h1, lw["ln2_g"], lw["ln2_b"])
    return out.reshape(B, S, H)


def encoder_forward(x: np.ndarray, valid_len: Sequence[int], layers: List[Dict[str, np.ndarray]],
                    head_num: int, size_per_head: int, seqs: Optional[Sequence[int]] = None,
                    gelu: str = "erf") -> np.ndarray:
    """The encoder stack: X_0 = x, X_{l+1} = layer_l(X_l), output X_L.

    Sequences never interact, so ``seqs`` restricts the work to a subset of the
    batch (the result holds those sequences, in that order).
    [FT] "什么是 Faster Transformer": the multi-layer encoder forward.
    """
    x = np.asarray(x, dtype=np.float64)
    vl = np.asarray(valid_len)
    if seqs is not None:
        idx = np.asarray(list(seqs), dtype=np.int64)
        x = x[idx]
        vl = vl[idx]
    for lw in layers:
        x = encoder_layer(x, vl, lw, head_num, size_per_head, gelu)
    return x
