"""Pins for the float64 decoder oracle (CPU only).

The decoder oracle (oracle/decoder_oracle.py) is checked against things other
than itself: the library routine torch.nn.TransformerDecoderLayer in float64
(post-LN, erf GELU, causal target mask, key padding masks), a brute-force
scalar-loop restatement, the already-pinned encoder attention, and invariants
the definition fixes (causality, padding, an empty memory).  Planted mistakes
at the end show that each plausible slip fails the library cross-check.
"""
import math

import numpy as np
import pytest
import torch

import encoder_inputs as EI
from oracle import brute
from oracle import decoder_oracle as D
from oracle import encoder_oracle as O


def _workload(nh=2, d=4, F=8, L=1, B=3, T=5, S=6, tlo=1, thi=None, mlo=1, mhi=None, seed=0, std=0.3):
    sh = EI.EncoderShape(nh, d, F, L)
    wl = EI.DecoderWorkload("dec-tiny", sh, B, T, S, "fp32", tlo, T if thi is None else thi, mlo,
                            S if mhi is None else mhi, ln_affine_random=True, seed=seed, weight_std=std)
    return EI.make_decoder_inputs(wl)


def _torch_layer(lw, nh, d, F):
    """torch.nn.TransformerDecoderLayer in float64 with the oracle's parameters
    ([in, out] matrices transposed into torch's [out, in])."""
    H = nh * d
    layer = torch.nn.TransformerDecoderLayer(d_model=H, nhead=nh, dim_feedforward=F, dropout=0.0,
                                             activation="gelu", layer_norm_eps=1e-12, batch_first=True,
                                             norm_first=False, dtype=torch.float64)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    with torch.no_grad():
        layer.self_attn.in_proj_weight.copy_(t(lw["w_qkv"].T))
        layer.self_attn.in_proj_bias.copy_(t(lw["b_qkv"]))
        layer.self_attn.out_proj.weight.copy_(t(lw["w_o"].T))
        layer.self_attn.out_proj.bias.copy_(t(lw["b_o"]))
        layer.multihead_attn.in_proj_weight.copy_(t(np.concatenate([lw["w_q2"].T, lw["w_kv2"].T], axis=0)))
        layer.multihead_attn.in_proj_bias.copy_(t(np.concatenate([lw["b_q2"], lw["b_kv2"]])))
        layer.multihead_attn.out_proj.weight.copy_(t(lw["w_o2"].T))
        layer.multihead_attn.out_proj.bias.copy_(t(lw["b_o2"]))
        layer.linear1.weight.copy_(t(lw["w_ff1"].T))
        layer.linear1.bias.copy_(t(lw["b_ff1"]))
        layer.linear2.weight.copy_(t(lw["w_ff2"].T))
        layer.linear2.bias.copy_(t(lw["b_ff2"]))
        for i, norm in ((1, layer.norm1), (2, layer.norm2), (3, layer.norm3)):
            norm.weight.copy_(t(lw[f"ln{i}_g"]))
            norm.bias.copy_(t(lw[f"ln{i}_b"]))
    layer.train()              # dropout is 0; training mode keeps the reference (non-fused) code path
    return layer


def _torch_forward(y, tl, mem, ml, layers, nh, d, F):
    B, T, _ = y.shape
    S = mem.shape[1]
    tgt_mask = torch.triu(torch.ones(T, T, dtype=torch.bool), diagonal=1)        # key j > query i
    tpad = torch.from_numpy(np.arange(T)[None, :] >= np.asarray(tl)[:, None])
    mpad = torch.from_numpy(np.arange(S)[None, :] >= np.asarray(ml)[:, None])
    out = torch.from_numpy(y)
    m = torch.from_numpy(mem)
    with torch.no_grad():
        for lw in layers:
            out = _torch_layer(lw, nh, d, F)(out, m, tgt_mask=tgt_mask, tgt_key_padding_mask=tpad,
                                            memory_key_padding_mask=mpad)
    return out.numpy()


@pytest.mark.parametrize("nh,d,F,L,B,T,S", [(2, 4, 8, 1, 3, 5, 6), (4, 8, 64, 2, 2, 9, 7), (1, 16, 32, 1, 2, 1, 4)])
def test_decoder_matches_torch_transformer_decoder_layer(nh, d, F, L, B, T, S):
    inp = _workload(nh, d, F, L, B, T, S, seed=nh * 10 + T)
    y, tl, mem, ml, layers = inp.as_float64()
    got = D.decoder_forward(y, tl, mem, ml, layers, nh, d)
    ref = _torch_forward(y, tl, mem, ml, layers, nh, d, F)
    assert np.max(np.abs(got - ref)) < 1e-10


def test_decoder_matches_brute_force_scalar_loops():
    # lengths 0 included: an empty target (every self-attention row empty) and an
    # empty memory (every cross-attention row empty)
    inp = _workload(nh=2, d=2, F=4, L=2, B=3, T=4, S=3, tlo=0, mlo=0, seed=3)
    y, tl, mem, ml, layers = inp.as_float64()
    tl[0], ml[1] = 0, 0
    got = D.decoder_forward(y, tl, mem, ml, layers, 2, 2)
    ref = np.array(brute.decoder_forward(y, tl, mem, ml, layers, 2, 2))
    assert np.max(np.abs(got - ref)) < 1e-13


def test_causality_later_target_tokens_do_not_change_earlier_outputs():
    inp = _workload(nh=2, d=4, F=8, L=2, B=2, T=6, S=5, tlo=6, thi=6, seed=5)
    y, tl, mem, ml, layers = inp.as_float64()
    base = D.decoder_forward(y, tl, mem, ml, layers, 2, 4)
    for i in range(6):
        y2 = y.copy()
        y2[:, i + 1:] = np.random.default_rng(i).normal(0, 3, y2[:, i + 1:].shape)
        got = D.decoder_forward(y2, tl, mem, ml, layers, 2, 4)
        assert np.array_equal(got[:, :i + 1], base[:, :i + 1])
        if i < 5:
            assert not np.array_equal(got[:, i + 1:], base[:, i + 1:])


def test_padding_of_memory_and_target_does_not_change_valid_outputs():
    inp = _workload(nh=2, d=4, F=8, L=2, B=3, T=6, S=7, tlo=2, thi=5, mlo=2, mhi=6, seed=6)
    y, tl, mem, ml, layers = inp.as_float64()
    base = D.decoder_forward(y, tl, mem, ml, layers, 2, 4)
    rng = np.random.default_rng(7)
    y2, mem2 = y.copy(), mem.copy()
    for b in range(3):
        y2[b, tl[b]:] = rng.normal(0, 3, y2[b, tl[b]:].shape)
        mem2[b, ml[b]:] = rng.normal(0, 3, mem2[b, ml[b]:].shape)
    got = D.decoder_forward(y2, tl, mem2, ml, layers, 2, 4)
    for b in range(3):
        assert np.array_equal(got[b, :tl[b]], base[b, :tl[b]])


def test_causal_self_attention_row_is_encoder_attention_over_its_prefix():
    """Row i of the causal self-attention equals the (pinned) encoder attention
    with valid length min(i + 1, nt), taken at row i."""
    rng = np.random.default_rng(8)
    T, d = 7, 4
    q, k, v = (rng.normal(size=(T, d)) for _ in range(3))
    for nt in (1, 4, 7):
        got = D.self_attention_causal(q, k, v, nt)
        qkv = np.stack([q, k, v])[:, None, None]
        for i in range(T):
            want = O.attention(qkv, [min(i + 1, nt)])[0, i]
            assert np.allclose(got[i], want, rtol=0, atol=1e-14)


def test_cross_attention_is_encoder_attention_when_lengths_match():
    rng = np.random.default_rng(9)
    q, k, v = (rng.normal(size=(6, 8)) for _ in range(3))
    for nm in (1, 3, 6):
        got = D.cross_attention(q, k, v, nm)
        want = O.attention(np.stack([q, k, v])[:, None, None], [nm])[0]
        assert np.allclose(got, want, rtol=0, atol=1e-14)


def test_empty_memory_leaves_only_the_cross_attention_bias():
    """nm = 0: the cross-attention context is 0, so the layer equals the same
    layer with Wo2 = 0 and any memory length."""
    inp = _workload(nh=2, d=4, F=8, L=1, B=2, T=4, S=5, seed=10)
    y, tl, mem, ml, layers = inp.as_float64()
    empty = D.decoder_forward(y, tl, mem, np.zeros_like(ml), layers, 2, 4)
    layers0 = [dict(lw, w_o2=np.zeros_like(lw["w_o2"])) for lw in layers]
    got = D.decoder_forward(y, tl, mem, ml, layers0, 2, 4)
    assert np.allclose(empty, got, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- planted mistakes

def _bad_causal(q, k, v, nt):          # off by one: a query does not attend to itself
    T, dd = q.shape
    return D._softmax_rows((q @ k.T) / math.sqrt(dd), [min(i, nt) for i in range(T)]) @ v


def _no_causal(q, k, v, nt):
    T, dd = q.shape
    return D._softmax_rows((q @ k.T) / math.sqrt(dd), [nt] * T) @ v


def _swapped_kv(q, k, v, nm):
    T, dd = q.shape
    return D._softmax_rows((q @ v.T) / math.sqrt(dd), [nm] * T) @ k


def _cross_mask_plus_one(q, k, v, nm):
    T, dd = q.shape
    return D._softmax_rows((q @ k.T) / math.sqrt(dd), [min(nm + 1, k.shape[0])] * T) @ v


@pytest.mark.parametrize("target,fn", [("self_attention_causal", _bad_causal), ("self_attention_causal", _no_causal),
                                       ("cross_attention", _swapped_kv), ("cross_attention", _cross_mask_plus_one)],
                         ids=["causal-off-by-one", "no-causal-mask", "cross-k-v-swapped", "memory-mask-plus-one"])
def test_planted_decoder_mistake_is_caught(monkeypatch, target, fn):
    inp = _workload(nh=2, d=4, F=8, L=1, B=3, T=5, S=6, tlo=5, thi=5, mlo=2, mhi=5, seed=11)
    y, tl, mem, ml, layers = inp.as_float64()
    ref = _torch_forward(y, tl, mem, ml, layers, 2, 4, 8)
    monkeypatch.setattr(D, target, fn)
    got = D.decoder_forward(y, tl, mem, ml, layers, 2, 4)
    assert np.max(np.abs(got - ref)) > 1e-6
