"""Pins for the float64 oracle (CPU only).

The oracle is checked against things other than itself: hand-worked values
(tests/golden), textbook constants, invariants the definition fixes, a
brute-force scalar-loop implementation on tiny shapes, and the library
routine torch.nn.TransformerEncoderLayer in float64.  The planted-mistake
tests at the end show that each plausible slip in the oracle fails a pin.
"""
import math
import os

import numpy as np
import pytest
import torch

import encoder_inputs as EI
from oracle import brute
from oracle import encoder_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _tiny_workload(nh=2, d=4, F=8, L=1, B=3, S=5, lo=1, hi=None, seed=0, affine=True, std=0.3):
    sh = EI.EncoderShape(nh, d, F, L)
    wl = EI.Workload("tiny", sh, B, S, "fp32", lo, S if hi is None else hi,
                     ln_affine_random=affine, seed=seed, weight_std=std)
    return wl, EI.make_inputs(wl)


def _f64(inp):
    return inp.as_float64()


# ---------------------------------------------------------------- golden values

def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def test_gelu_matches_normal_cdf_table():
    for t, phi in _read_golden("gelu_normal_cdf.txt"):
        t, phi = float(t), float(phi)
        assert abs(O.gelu_erf(np.array([t]))[0] - t * phi) < 1e-15


def test_attention_hand_worked_example():
    rows = _read_golden("attention_hand_worked.txt")
    q = np.array([[float(v) for v in r[1:]] for r in rows if r[0] == "q"])
    k = np.array([[float(v) for v in r[1:]] for r in rows if r[0] == "k"])
    v = np.array([[float(v) for v in r[1:]] for r in rows if r[0] == "v"])
    qkv = np.stack([q, k, v])[:, None, None]                 # [3, B=1, nh=1, S=2, d=4]
    for tag, n in (("n2", 2), ("n1", 1)):
        want = np.array([[float(x) for x in r[1:]] for r in rows if r[0] == tag])
        got = O.attention(qkv, [n])[0]
        assert np.max(np.abs(got - want)) < 1e-15


# ---------------------------------------------------------------- step invariants

def test_softmax_rows_sum_to_one_and_mask_is_exact():
    rng = np.random.default_rng(3)
    sc = rng.normal(0, 3, (7, 9))
    for n in range(0, 10):
        p = O.softmax_masked(sc, n)
        assert np.all(p >= 0)
        assert np.all(p[:, n:] == 0.0)
        if n > 0:
            assert np.max(np.abs(p.sum(1) - 1.0)) < 1e-12
        else:
            assert np.all(p == 0.0)


def test_layernorm_moments():
    rng = np.random.default_rng(4)
    z = rng.normal(5, 7, (6, 768))
    y = O.layer_norm(z, np.ones(768), np.zeros(768))
    assert np.max(np.abs(y.mean(1))) < 1e-12
    assert np.max(np.abs(y.var(1) - 1.0)) < 1e-9
    y2 = O.layer_norm(z, 2 * np.ones(768), 3 * np.ones(768))
    assert np.max(np.abs(y2.mean(1) - 3.0)) < 1e-12
    assert np.max(np.abs(y2.std(1) - 2.0)) < 1e-9


def test_layernorm_two_elements_closed_form():
    # For H = 2 the normalised row is (-1, +1) ordered like the inputs (eps negligible).
    z = np.array([[1.0, 4.0], [10.0, -3.0]])
    y = O.layer_norm(z, np.array([1.0, 1.0]), np.array([0.0, 0.0]))
    assert np.allclose(y, [[-1, 1], [1, -1]], atol=1e-12)


def test_gelu_special_values_and_tanh_form():
    assert O.gelu_erf(np.array([0.0]))[0] == 0.0
    t = np.array([8.0, 12.0, 30.0])
    assert np.max(np.abs(O.gelu_erf(t) - t)) < 1e-13
    assert np.max(np.abs(O.gelu_erf(-t))) < 1e-13
    grid = np.linspace(-6, 6, 2001)
    diff = np.abs(O.gelu_tanh(grid) - O.gelu_erf(grid))
    assert 1e-5 < diff.max() < 1e-3      # the two forms differ by a few 1e-4 at most


def test_head_split_index_formula():
    B, S, nh, d = 2, 3, 3, 2
    H = nh * d
    qkv = np.arange(B * S * 3 * H, dtype=np.float64).reshape(B * S, 3 * H)
    out = O.head_split(qkv, B, S, nh, d)
    for t in range(3):
        for b in range(B):
            for h in range(nh):
                for s in range(S):
                    for c in range(d):
                        assert out[t, b, h, s, c] == qkv[b * S + s, t * H + h * d + c]


# ---------------------------------------------------------------- closed forms

def test_single_valid_key_gives_value_row():
    wl, inp = _tiny_workload(B=2, S=5, lo=1, hi=1)
    x, vl, layers = _f64(inp)
    lw = layers[0]
    nh, d = wl.shape.head_num, wl.shape.size_per_head
    H = nh * d
    B, S = wl.batch, wl.seq
    qkv = O.qkv_projection(x.reshape(B * S, H), lw["w_qkv"], lw["b_qkv"])
    ctx = O.attention(O.head_split(qkv, B, S, nh, d), vl)
    for b in range(B):
        v0 = x[b, 0] @ lw["w_qkv"][:, 2 * H:] + lw["b_qkv"][2 * H:]
        assert np.max(np.abs(ctx[b] - v0[None, :])) < 1e-14


def test_zero_query_weights_give_uniform_attention():
    wl, inp = _tiny_workload(B=3, S=6, lo=2, hi=6)
    x, vl, layers = _f64(inp)
    lw = dict(layers[0])
    nh, d = wl.shape.head_num, wl.shape.size_per_head
    H = nh * d
    B, S = wl.batch, wl.seq
    for zero_cols in (slice(0, H), slice(H, 2 * H)):          # Wq = bq = 0, then Wk = bk = 0
        w = lw["w_qkv"].copy(); b = lw["b_qkv"].copy()
        w[:, zero_cols] = 0.0; b[zero_cols] = 0.0
        qkv = O.qkv_projection(x.reshape(B * S, H), w, b)
        ctx = O.attention(O.head_split(qkv, B, S, nh, d), vl)
        for bi in range(B):
            n = int(vl[bi])
            v = x[bi] @ w[:, 2 * H:] + b[2 * H:]
            assert np.max(np.abs(ctx[bi] - v[:n].mean(0)[None, :])) < 1e-13


def test_single_head_matches_textbook_sdpa():
    # nh = 1: plain scaled dot-product attention; torch's SDPA is the library routine.
    rng = np.random.default_rng(7)
    S, d, n = 9, 16, 6
    q, k, v = (rng.normal(0, 1, (S, d)) for _ in range(3))
    got = O.attention(np.stack([q, k, v])[:, None, None], [n])[0]
    mask = torch.zeros(S, S, dtype=torch.bool)
    mask[:, :n] = True
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None], attn_mask=mask[None])
    assert np.max(np.abs(got - ref[0].numpy())) < 1e-13


def test_zero_valid_len_gives_zero_context_and_finite_output():
    wl, inp = _tiny_workload(B=2, S=4, lo=0, hi=0)
    x, vl, layers = _f64(inp)
    assert list(vl) == [0, 0]
    nh, d = wl.shape.head_num, wl.shape.size_per_head
    qkv = O.qkv_projection(x.reshape(8, nh * d), layers[0]["w_qkv"], layers[0]["b_qkv"])
    assert np.all(O.attention(O.head_split(qkv, 2, 4, nh, d), vl) == 0.0)
    out = O.encoder_forward(x, vl, layers, nh, d)
    assert np.all(np.isfinite(out))


# ---------------------------------------------------------------- whole-layer invariants

def test_permutation_equivariance_over_valid_tokens():
    wl, inp = _tiny_workload(nh=2, d=4, F=8, L=2, B=2, S=7, lo=5, hi=7, seed=11)
    x, vl, layers = _f64(inp)
    nh, d = wl.shape.head_num, wl.shape.size_per_head
    out = O.encoder_forward(x, vl, layers, nh, d)
    rng = np.random.default_rng(5)
    xp = x.copy()
    perms = []
    for b in range(wl.batch):
        n = int(vl[b])
        p = np.concatenate([rng.permutation(n), np.arange(n, wl.seq)])
        perms.append(p)
        xp[b] = x[b, p]
    outp = O.encoder_forward(xp, vl, layers, nh, d)
    for b in range(wl.batch):
        n = int(vl[b])
        rel = np.linalg.norm(outp[b, :n] - out[b, perms[b]][:n]) / np.linalg.norm(out[b, :n])
        assert rel < 1e-12


def test_padding_tokens_do_not_change_valid_outputs():
    wl, inp = _tiny_workload(nh=2, d=4, F=8, L=2, B=3, S=6, lo=2, hi=5, seed=12)
    x, vl, layers = _f64(inp)
    nh, d = wl.shape.head_num, wl.shape.size_per_head
    out = O.encoder_forward(x, vl, layers, nh, d)
    x2 = x.copy()
    rng = np.random.default_rng(9)
    for b in range(wl.batch):
        n = int(vl[b])
        x2[b, n:] = rng.normal(0, 10, x2[b, n:].shape)
    out2 = O.encoder_forward(x2, vl, layers, nh, d)
    for b in range(wl.batch):
        n = int(vl[b])
        assert np.max(np.abs(out2[b, :n] - out[b, :n])) <= 1e-15


def test_identical_tokens_give_identical_outputs():
    wl, inp = _tiny_workload(nh=2, d=4, F=8, L=2, B=1, S=5, lo=5, hi=5, seed=13)
    x, vl, layers = _f64(inp)
    x[0, :] = x[0, 0]
    out = O.encoder_forward(x, vl, layers, wl.shape.head_num, wl.shape.size_per_head)
    assert np.max(np.abs(out[0] - out[0, :1])) < 1e-14


def test_sequence_subset_equals_full_batch_rows():
    wl, inp = _tiny_workload(nh=2, d=4, F=8, L=2, B=5, S=4, lo=1, seed=14)
    x, vl, layers = _f64(inp)
    full = O.encoder_forward(x, vl, layers, 2, 4)
    sub = O.encoder_forward(x, vl, layers, 2, 4, seqs=[4, 1])
    assert np.array_equal(sub, full[[4, 1]])


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("nh,d,S,L", [(1, 2, 1, 1), (1, 4, 3, 2), (2, 2, 5, 1), (2, 4, 5, 2), (2, 4, 3, 1)])
def test_matches_brute_force_scalar_loops(nh, d, S, L):
    wl, inp = _tiny_workload(nh=nh, d=d, F=8, L=L, B=3, S=S, lo=1, seed=nh * 100 + d * 10 + S)
    x, vl, layers = _f64(inp)
    got = O.encoder_forward(x, vl, layers, nh, d)
    want = np.array(brute.encoder_forward(x, vl, layers, nh, d))
    assert np.max(np.abs(got - want)) < 1e-13


# ---------------------------------------------------------------- library routine

def _torch_layer(lw, H, nh, F):
    layer = torch.nn.TransformerEncoderLayer(
        d_model=H, nhead=nh, dim_feedforward=F, dropout=0.0, activation="gelu",
        batch_first=True, norm_first=False, layer_norm_eps=1e-12, dtype=torch.float64)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    with torch.no_grad():
        layer.self_attn.in_proj_weight.copy_(t(lw["w_qkv"].T))
        layer.self_attn.in_proj_bias.copy_(t(lw["b_qkv"]))
        layer.self_attn.out_proj.weight.copy_(t(lw["w_o"].T))
        layer.self_attn.out_proj.bias.copy_(t(lw["b_o"]))
        layer.linear1.weight.copy_(t(lw["w_ff1"].T))
        layer.linear1.bias.copy_(t(lw["b_ff1"]))
        layer.linear2.weight.copy_(t(lw["w_ff2"].T))
        layer.linear2.bias.copy_(t(lw["b_ff2"]))
        layer.norm1.weight.copy_(t(lw["ln1_g"]))
        layer.norm1.bias.copy_(t(lw["ln1_b"]))
        layer.norm2.weight.copy_(t(lw["ln2_g"]))
        layer.norm2.bias.copy_(t(lw["ln2_b"]))
    layer.train()          # dropout is 0; training mode keeps torch off its fused fast path
    return layer


def torch_encoder(x, vl, layers, nh):
    B, S, H = x.shape
    F = layers[0]["w_ff1"].shape[1]
    mask = torch.arange(S)[None, :] >= torch.from_numpy(np.asarray(vl, dtype=np.int64))[:, None]
    h = torch.from_numpy(x)
    with torch.no_grad():
        for lw in layers:
            h = _torch_layer(lw, H, nh, F)(h, src_key_padding_mask=mask)
    return h.numpy()


def _valid_rel(a, b, vl):
    num = sum(np.sum((a[i, :n] - b[i, :n]) ** 2) for i, n in enumerate(vl))
    den = sum(np.sum(b[i, :n] ** 2) for i, n in enumerate(vl))
    return math.sqrt(num / den)


@pytest.mark.parametrize("nh,d,F,L,S", [(2, 8, 32, 1, 7), (4, 8, 64, 2, 9), (3, 16, 48, 2, 33)])
def test_matches_torch_transformer_encoder_layer(nh, d, F, L, S):
    wl, inp = _tiny_workload(nh=nh, d=d, F=F, L=L, B=4, S=S, lo=1, seed=S + L, std=0.1)
    x, vl, layers = _f64(inp)
    got = O.encoder_forward(x, vl, layers, nh, d)
    ref = torch_encoder(x, vl, layers, nh)
    for b in range(wl.batch):
        n = int(vl[b])
        assert np.max(np.abs(got[b, :n] - ref[b, :n])) < 1e-10


# ---------------------------------------------------------------- planted mistakes

def _mutant_cases():
    def no_scale(qkv_split, valid_len, seqs=None):
        q = qkv_split.copy()
        q[0] *= math.sqrt(q.shape[-1])
        return _orig["attention"](q, valid_len, seqs)

    def mask_off_by_one(scores, n):
        return _orig["softmax_masked"](scores, min(n + 1, scores.shape[1]))

    def unbiased_var(z, gamma, beta, eps=O.LN_EPS):
        mu = z.mean(-1, keepdims=True)
        var = ((z - mu) ** 2).sum(-1, keepdims=True) / (z.shape[-1] - 1)
        return gamma * (z - mu) / np.sqrt(var + eps) + beta

    def big_eps(z, gamma, beta, eps=O.LN_EPS):
        return _orig["layer_norm"](z, gamma, beta, 1e-3)

    def no_residual(a, bias, resid, gamma, beta):
        return O.layer_norm(a + bias, gamma, beta)

    def tanh_gelu(h1, w, b, gelu="erf"):
        return O.gelu_tanh(h1 @ w + b)

    def transposed_split(qkv2d, batch, seq, nh, d):
        t = _orig["head_split"](qkv2d, batch, seq, nh, d)
        return t[[1, 0, 2]]            # Q and K swapped (scores transposed)

    def dropped_bias(x2d, w, b):
        return x2d @ w

    return {
        "attention": no_scale,
        "softmax_masked": mask_off_by_one,
        "layer_norm": unbiased_var,
        "layer_norm_eps": big_eps,
        "bias_residual_layernorm": no_residual,
        "ffn1_gelu": tanh_gelu,
        "head_split": transposed_split,
        "qkv_projection": dropped_bias,
    }


_orig = {k: getattr(O, k) for k in ("attention", "softmax_masked", "layer_norm", "head_split")}


@pytest.mark.parametrize("name", sorted(_mutant_cases().keys()))
def test_planted_mistake_is_caught(monkeypatch, name):
    fn = _mutant_cases()[name]
    target = "layer_norm" if name == "layer_norm_eps" else name
    monkeypatch.setattr(O, target, fn)
    wl, inp = _tiny_workload(nh=2, d=8, F=32, L=1, B=3, S=7, lo=2, seed=21, std=0.2, affine=True)
    x, vl, layers = _f64(inp)
    if name == "layer_norm_eps":
        x = x * 1e-2              # small rows make eps matter
    got = O.encoder_forward(x, vl, layers, 2, 8)
    ref = torch_encoder(x, vl, layers, 2)
    worst = max(np.max(np.abs(got[b, :int(vl[b])] - ref[b, :int(vl[b])])) for b in range(wl.batch))
    assert worst > 1e-6, f"planted mistake {name} was not detected (diff {worst:g})"


def test_gelu_tanh_form_matches_library_routine():
    # torch.nn.functional.gelu(approximate="tanh") is the library form of the same approximation.
    t = np.linspace(-9, 9, 4001)
    ref = torch.nn.functional.gelu(torch.from_numpy(t), approximate="tanh").numpy()
    assert np.max(np.abs(O.gelu_tanh(t) - ref)) < 1e-15
    # GELU(t) - GELU(-t) = t holds for both forms (the inner function is odd)
    assert np.max(np.abs(O.gelu_tanh(t) - O.gelu_tanh(-t) - t)) < 1e-14
    assert np.max(np.abs(O.gelu_erf(t) - O.gelu_erf(-t) - t)) < 1e-14


def test_tanh_gelu_encoder_matches_torch_tanh_gelu():
    wl, inp = _tiny_workload(nh=2, d=8, F=32, L=1, B=3, S=7, lo=1, seed=31, std=0.1)
    x, vl, layers = _f64(inp)
    got = O.encoder_forward(x, vl, layers, 2, 8, gelu="tanh")
    layer = _torch_layer(layers[0], 16, 2, 32)
    layer.activation = lambda v: torch.nn.functional.gelu(v, approximate="tanh")
    mask = torch.arange(7)[None, :] >= torch.from_numpy(np.asarray(vl, dtype=np.int64))[:, None]
    with torch.no_grad():
        ref = layer(torch.from_numpy(x), src_key_padding_mask=mask).numpy()
    for b in range(3):
        n = int(vl[b])
        assert np.max(np.abs(got[b, :n] - ref[b, :n])) < 1e-10
