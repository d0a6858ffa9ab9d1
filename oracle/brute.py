"""Brute-force scalar-loop encoder forward for tiny shapes (pure Python, float64).

TEST INFRASTRUCTURE ONLY: it exists to pin the numpy oracle in
encoder_oracle.py.  Every product, sum and normalisation is an explicit
Python loop over scalars with math.exp / math.erf / math.sqrt; no numpy
arithmetic, no blocking, no reuse of intermediate buffers across steps.

Source page: the Faster Transformer write-up ("有钱任性：英伟达训练80亿参数量
GPT-2，1475块V100 53分钟训练BERT", sections "什么是 Faster Transformer" and
"Faster Transformer 优化原理"); same readings as encoder_oracle.py.
"""
from __future__ import annotations

import math
from typing import Dict, List, Sequence

LN_EPS = 1e-12


def _matvec_row(row: List[float], w, b) -> List[float]:
    """y[j] = sum_k row[k] * w[k][j] + b[j]."""
    n_in = len(row)
    n_out = len(b)
    out = []
    for j in range(n_out):
        s = 0.0
        for k in range(n_in):
            s += row[k] * float(w[k][j])
        out.append(s + float(b[j]))
    return out


def _ln_row(z: List[float], g, be) -> List[float]:
    n = len(z)
    mu = 0.0
    for v in z:
        mu += v
    mu /= n
    var = 0.0
    for v in z:
        var += (v - mu) * (v - mu)
    var /= n
    inv = 1.0 / math.sqrt(var + LN_EPS)
    return [float(g[i]) * (z[i] - mu) * inv + float(be[i]) for i in range(n)]


def _gelu(t: float) -> float:
    return 0.5 * t * (1.0 + math.erf(t / math.sqrt(2.0)))


def layer_one_sequence(xs: List[List[float]], n: int, lw: Dict, nh: int, d: int) -> List[List[float]]:
    """One post-LN encoder layer for one sequence xs [S][H] with n valid keys."""
    S = len(xs)
    H = nh * d
    n = min(max(n, 0), S)
    qkv = [_matvec_row(xs[i], lw["w_qkv"], lw["b_qkv"]) for i in range(S)]
    ctx = [[0.0] * H for _ in range(S)]
    for h in range(nh):
        for i in range(S):
            if n == 0:
                continue
            scores = []
            for j in range(n):
                s = 0.0
                for c in range(d):
                    s += qkv[i][h * d + c] * qkv[j][H + h * d + c]
                scores.append(s / math.sqrt(d))
            m = max(scores)
            es = [math.exp(s - m) for s in scores]
            tot = 0.0
            for e in es:
                tot += e
            for c in range(d):
                acc = 0.0
                for j in range(n):
                    acc += (es[j] / tot) * qkv[j][2 * H + h * d + c]
                ctx[i][h * d + c] = acc
    out = []
    for i in range(S):
        a = _matvec_row(ctx[i], lw["w_o"], lw["b_o"])
        z1 = [xs[i][c] + a[c] for c in range(H)]
        h1 = _ln_row(z1, lw["ln1_g"], lw["ln1_b"])
        u = [_gelu(v) for v in _matvec_row(h1, lw["w_ff1"], lw["b_ff1"])]
        y = _matvec_row(u, lw["w_ff2"], lw["b_ff2"])
        z2 = [h1[c] + y[c] for c in range(H)]
        out.append(_ln_row(z2, lw["ln2_g"], lw["ln2_b"]))
    return out


def encoder_forward(x, valid_len: Sequence[int], layers: List[Dict], nh: int, d: int):
    """x: nested [B][S][H] (or an array); returns nested lists of floats."""
    res = []
    for b in range(len(x)):
        xs = [[float(v) for v in row] for row in x[b]]
        for lw in layers:
            xs = layer_one_sequence(xs, int(valid_len[b]), lw, nh, d)
        res.append(xs)
    return res


# ---------------------------------------------------------------- decoder (same readings as decoder_oracle.py)

def _attend(qrows, krows, vrows, limits, qoff, koff, voff, nh, d):
    """ctx[i] over keys j < limits[i] for every head; rows are [R][...] lists,
    head h of Q at columns qoff + h*d, of K at koff + h*d, of V at voff + h*d."""
    out = [[0.0] * (nh * d) for _ in qrows]
    for h in range(nh):
        for i, q in enumerate(qrows):
            lim = limits[i]
            if lim <= 0:
                continue
            scores = []
            for j in range(lim):
                s = 0.0
                for c in range(d):
                    s += q[qoff + h * d + c] * krows[j][koff + h * d + c]
                scores.append(s / math.sqrt(d))
            m = max(scores)
            es = [math.exp(s - m) for s in scores]
            tot = 0.0
            for e in es:
                tot += e
            for c in range(d):
                acc = 0.0
                for j in range(lim):
                    acc += (es[j] / tot) * vrows[j][voff + h * d + c]
                out[i][h * d + c] = acc
    return out


def decoder_layer_one_sequence(ys, nt: int, mem, nm: int, lw: Dict, nh: int, d: int):
    """One post-LN decoder layer for one target sequence ys [T][H] against its
    memory mem [S][H]: causal self-attention (keys j <= i, j < nt), LN1,
    cross-attention (keys j < nm), LN2, FFN, LN3."""
    T, S, H = len(ys), len(mem), nh * d
    nt, nm = min(max(nt, 0), T), min(max(nm, 0), S)
    qkv = [_matvec_row(ys[i], lw["w_qkv"], lw["b_qkv"]) for i in range(T)]
    ctx = _attend(qkv, qkv, qkv, [min(i + 1, nt) for i in range(T)], 0, H, 2 * H, nh, d)
    h1 = []
    for i in range(T):
        a = _matvec_row(ctx[i], lw["w_o"], lw["b_o"])
        h1.append(_ln_row([ys[i][c] + a[c] for c in range(H)], lw["ln1_g"], lw["ln1_b"]))
    q2 = [_matvec_row(h1[i], lw["w_q2"], lw["b_q2"]) for i in range(T)]
    kv2 = [_matvec_row(mem[j], lw["w_kv2"], lw["b_kv2"]) for j in range(S)]
    ctx2 = _attend(q2, kv2, kv2, [nm] * T, 0, 0, H, nh, d)
    out = []
    for i in range(T):
        a = _matvec_row(ctx2[i], lw["w_o2"], lw["b_o2"])
        h2 = _ln_row([h1[i][c] + a[c] for c in range(H)], lw["ln2_g"], lw["ln2_b"])
        u = [_gelu(v) for v in _matvec_row(h2, lw["w_ff1"], lw["b_ff1"])]
        y = _matvec_row(u, lw["w_ff2"], lw["b_ff2"])
        out.append(_ln_row([h2[c] + y[c] for c in range(H)], lw["ln3_g"], lw["ln3_b"]))
    return out


def decoder_forward(y, tgt_len: Sequence[int], mem, mem_len: Sequence[int], layers: List[Dict], nh: int, d: int):
    res = []
    for b in range(len(y)):
        ys = [[float(v) for v in row] for row in y[b]]
        ms = [[float(v) for v in row] for row in mem[b]]
        for lw in layers:
            ys = decoder_layer_one_sequence(ys, int(tgt_len[b]), ms, int(mem_len[b]), lw, nh, d)
        res.append(ys)
    return res
