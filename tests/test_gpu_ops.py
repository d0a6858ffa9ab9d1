"""Each kernel of the forward path alone against its oracle step (GPU).

Inputs are seeded and in the storage dtype; the oracle step runs in float64
on exactly those values.  Shapes span several GEMM tiles (128 rows) and
ragged tails, every supported head size, and the structures of the
workloads (4x32, 12x64, 16x64, 8x128).
"""
import numpy as np
import pytest

import encoder_inputs as EI
from oracle import encoder_oracle as O
from parity_utils import empty_dev, max_abs, rel_l2, to_dev, to_host, valid_mask

pytestmark = pytest.mark.gpu

SHAPES = [(4, 32, 512), (12, 64, 3072), (16, 64, 4096), (8, 128, 2048)]
BATCH_SEQ = [(1, 1), (3, 37), (2, 128), (5, 131)]

# Single-GEMM outputs are the exact product rounded once to FP16 (half an ulp,
# 2^-11 relative) plus FP32 accumulation error; attention also rounds P to FP16.
GEMM_REL_L2 = 1e-3
ATTN_REL_L2 = 2e-3
LN_MAX_ABS = 4e-3            # |LN output| <= ~5, one FP16 ulp there is 2^-8
FP32_REL_L2 = 1e-5


def _setup(shape, batch, seq, dtype="fp16", seed=0):
    nh, d, F = shape
    sh = EI.EncoderShape(nh, d, F, 1)
    wl = EI.Workload("ops", sh, batch, seq, dtype, 1, seq, seed=seed, ln_affine_random=True)
    inp = EI.make_inputs(wl)
    from parity_utils import encoder_from_inputs
    enc = encoder_from_inputs(inp)
    x64, vl, layers64 = inp.as_float64()
    return wl, inp, enc, x64, vl, layers64[0]


def _ulp_bound(ref):
    return 2.0 ** -10 * max(1.0, float(np.max(np.abs(ref))))


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}_F{s[2]}")
@pytest.mark.parametrize("batch,seq", BATCH_SEQ, ids=lambda v: str(v))
def test_qkv_projection_and_head_split(shape, batch, seq):
    wl, inp, enc, x64, vl, lw = _setup(shape, batch, seq)
    nh, d = shape[0], shape[1]
    H = nh * d
    out = empty_dev((3, batch, nh, seq, d), "fp16")
    enc.op_qkv(0, to_dev(inp.x), out, batch, seq)
    got = to_host(out)
    ref = O.head_split(O.qkv_projection(x64.reshape(-1, H), lw["w_qkv"], lw["b_qkv"]), batch, seq, nh, d)
    assert rel_l2(got, ref) < GEMM_REL_L2
    assert max_abs(got, ref) < _ulp_bound(ref)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}_F{s[2]}")
@pytest.mark.parametrize("batch,seq", BATCH_SEQ + [(2, 512), (3, 200), (4, 96), (3, 65)], ids=lambda v: str(v))
def test_attention(shape, batch, seq):
    nh, d, _ = shape
    wl, inp, enc, x64, vl, lw = _setup(shape, batch, seq)
    qkv = EI.random_array((3, batch, nh, seq, d), "fp16", seed=7)
    vlen = np.random.default_rng(3).integers(1, seq + 1, batch).astype(np.int32)
    vlen[0] = seq
    ctx = empty_dev((batch * seq, nh * d), "fp16")
    enc.op_attention(to_dev(qkv), to_dev(vlen), ctx, batch, seq)
    got = to_host(ctx).reshape(batch, seq, nh * d)
    ref = O.attention(qkv.astype(np.float64), vlen)
    assert rel_l2(got, ref) < ATTN_REL_L2
    assert max_abs(got, ref) < 4 * _ulp_bound(ref)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}_F{s[2]}")
@pytest.mark.parametrize("batch,seq", BATCH_SEQ, ids=lambda v: str(v))
def test_out_proj_ffn1_ffn2(shape, batch, seq):
    nh, d, F = shape
    H = nh * d
    M = batch * seq
    wl, inp, enc, x64, vl, lw = _setup(shape, batch, seq)
    ctx = EI.random_array((M, H), "fp16", seed=11)
    resid = EI.random_array((M, H), "fp16", seed=14)
    a = empty_dev((M, H), "fp16")
    enc.op_out_proj_ln(0, to_dev(ctx), to_dev(resid), a, M)
    ref = O.bias_residual_layernorm(ctx.astype(np.float64) @ lw["w_o"], lw["b_o"], resid.astype(np.float64),
                                    lw["ln1_g"], lw["ln1_b"])
    got = to_host(a)
    assert rel_l2(got, ref) < GEMM_REL_L2 and max_abs(got, ref) < LN_MAX_ABS

    h1 = EI.random_array((M, H), "fp16", seed=12)
    u = empty_dev((M, F), "fp16")
    enc.op_ffn1(0, to_dev(h1), u, M)
    ref = O.ffn1_gelu(h1.astype(np.float64), lw["w_ff1"], lw["b_ff1"])
    got = to_host(u)
    assert rel_l2(got, ref) < GEMM_REL_L2 and max_abs(got, ref) < _ulp_bound(ref)

    uu = EI.random_array((M, F), "fp16", seed=13, std=0.5)
    y = empty_dev((M, H), "fp16")
    enc.op_ffn2_ln(0, to_dev(uu), to_dev(h1), y, M)
    ref = O.bias_residual_layernorm(uu.astype(np.float64) @ lw["w_ff2"], lw["b_ff2"], h1.astype(np.float64),
                                    lw["ln2_g"], lw["ln2_b"])
    got = to_host(y)
    assert rel_l2(got, ref) < GEMM_REL_L2 and max_abs(got, ref) < LN_MAX_ABS


@pytest.mark.parametrize("shape,M", [((4, 64, 1024), 9300), ((12, 64, 3072), 4000), ((16, 64, 4096), 2600),
                                     ((12, 64, 3072), 16384)], ids=lambda v: str(v))
def test_fused_layernorm_gemms(shape, M):
    """Enough tokens for the 2-CTA tiles: the GEMMs write the LayerNorm of their rows
    (row statistics exchanged across the cluster that covers the row; clusters of
    2, 6 and 8 CTAs for H = 256, 768, 1024).  Both GEMMs fuse by default for
    H <= 768; the options' value 2 fuses wherever supported.  Against the oracle
    step, and against the unfused path (GEMM writing bias + residual, then the
    LayerNorm kernel; both fusion options 0)."""
    nh, d, F = shape
    H = nh * d
    wl, inp, enc, x64, vl, lw = _setup(shape, 1, M)
    enc.set_option("ln_fuse_out_proj", 2)         # wherever supported (H = 1024 too)
    enc.set_option("ln_fuse_ffn2", 2)
    ctx = EI.random_array((M, H), "fp16", seed=41)
    resid = EI.random_array((M, H), "fp16", seed=42, mean=0.2)
    uu = EI.random_array((M, F), "fp16", seed=43, std=0.5)

    def run(e):
        a = empty_dev((M, H), "fp16")
        e.op_out_proj_ln(0, to_dev(ctx), to_dev(resid), a, M)
        y = empty_dev((M, H), "fp16")
        e.op_ffn2_ln(0, to_dev(uu), a, y, M)
        return to_host(a), to_host(y)

    got_a, got_y = run(enc)
    ref_a = O.bias_residual_layernorm(ctx.astype(np.float64) @ lw["w_o"], lw["b_o"], resid.astype(np.float64),
                                      lw["ln1_g"], lw["ln1_b"])
    ref_y = O.bias_residual_layernorm(uu.astype(np.float64) @ lw["w_ff2"], lw["b_ff2"], got_a.astype(np.float64),
                                      lw["ln2_g"], lw["ln2_b"])
    for g, r in ((got_a, ref_a), (got_y, ref_y)):
        assert rel_l2(g, r) < GEMM_REL_L2 and max_abs(g, r) < LN_MAX_ABS
    assert enc.device_status() == 0
    wl, inp, enc1, x64, vl, lw = _setup(shape, 1, M)
    enc1.set_option("ln_fuse_out_proj", False)
    enc1.set_option("ln_fuse_ffn2", False)
    un_a, un_y = run(enc1)
    assert rel_l2(got_a, un_a) < GEMM_REL_L2 and rel_l2(got_y, un_y) < GEMM_REL_L2


@pytest.mark.parametrize("shape,M", [((4, 32, 512), 4100), ((8, 32, 1024), 2053), ((12, 64, 3072), 5000),
                                     ((10, 64, 2560), 3001), ((16, 64, 4096), 2049), ((12, 64, 3072), 32768)],
                         ids=lambda v: str(v))
def test_layernorm_kernel_many_rows(shape, M):
    """The LayerNorm kernel after a GEMM that wrote z = acc + bias + residual,
    at thousands of rows (both fusions off so that it runs), hidden sizes 128
    to 1024 and ragged row counts, against the oracle step."""
    nh, d, F = shape
    H = nh * d
    wl, inp, enc, x64, vl, lw = _setup(shape, 1, M)
    enc.set_option("ln_fuse_ffn2", False)
    enc.set_option("ln_fuse_out_proj", False)
    ctx = EI.random_array((M, H), "fp16", seed=51)
    resid = EI.random_array((M, H), "fp16", seed=52, mean=0.3)
    a = empty_dev((M, H), "fp16")
    enc.op_out_proj_ln(0, to_dev(ctx), to_dev(resid), a, M)
    ref = O.bias_residual_layernorm(ctx.astype(np.float64) @ lw["w_o"], lw["b_o"], resid.astype(np.float64),
                                    lw["ln1_g"], lw["ln1_b"])
    got = to_host(a)
    assert rel_l2(got, ref) < GEMM_REL_L2 and max_abs(got, ref) < LN_MAX_ABS
    assert enc.device_status() == 0


@pytest.mark.parametrize("shape", [(4, 32, 512), (12, 64, 3072)], ids=lambda s: f"{s[0]}x{s[1]}")
def test_fp32_steps(shape):
    nh, d, F = shape
    H = nh * d
    batch, seq = 3, 37
    M = batch * seq
    wl, inp, enc, x64, vl, lw = _setup(shape, batch, seq, dtype="fp32")
    qkv = empty_dev((3, batch, nh, seq, d), "fp32")
    enc.op_qkv(0, to_dev(inp.x), qkv, batch, seq)
    ref_qkv = O.head_split(O.qkv_projection(x64.reshape(-1, H), lw["w_qkv"], lw["b_qkv"]), batch, seq, nh, d)
    assert rel_l2(to_host(qkv), ref_qkv) < FP32_REL_L2
    ctx = empty_dev((M, H), "fp32")
    vlen = np.array([37, 1, 20], np.int32)
    enc.op_attention(qkv, to_dev(vlen), ctx, batch, seq)
    ref_ctx = O.attention(to_host(qkv).astype(np.float64), vlen).reshape(M, H)
    assert rel_l2(to_host(ctx), ref_ctx) < FP32_REL_L2
    h1 = EI.random_array((M, H), "fp32", seed=5)
    u = empty_dev((M, F), "fp32")
    enc.op_ffn1(0, to_dev(h1), u, M)
    assert rel_l2(to_host(u), O.ffn1_gelu(h1.astype(np.float64), lw["w_ff1"], lw["b_ff1"])) < FP32_REL_L2
    out = empty_dev((M, H), "fp32")
    enc.op_out_proj_ln(0, ctx, to_dev(h1), out, M)
    ref = O.bias_residual_layernorm(to_host(ctx).astype(np.float64) @ lw["w_o"], lw["b_o"], h1.astype(np.float64),
                                    lw["ln1_g"], lw["ln1_b"])
    assert rel_l2(to_host(out), ref) < FP32_REL_L2
    uu = EI.random_array((M, F), "fp32", seed=7, std=0.5)
    y = empty_dev((M, H), "fp32")
    enc.op_ffn2_ln(0, to_dev(uu), out, y, M)
    ref_y = O.bias_residual_layernorm(uu.astype(np.float64) @ lw["w_ff2"], lw["b_ff2"],
                                      to_host(out).astype(np.float64), lw["ln2_g"], lw["ln2_b"])
    assert rel_l2(to_host(y), ref_y) < FP32_REL_L2


@pytest.mark.parametrize("seq", [40, 100, 300], ids=str)
def test_attention_valid_len_clamping_and_empty(seq):
    """Lengths outside [0, seq] are clamped; n == 0 gives ctx = 0 (seq 40 runs the
    mma.sync kernel, seq 100 the one-block tensor-core kernel, seq 300 the
    multi-block one)."""
    shape = (12, 64, 3072)
    nh, d, _ = shape
    batch = 4
    wl, inp, enc, x64, vl, lw = _setup(shape, batch, seq)
    qkv = EI.random_array((3, batch, nh, seq, d), "fp16", seed=8)
    vlen = np.array([seq + 7, 0, -3, 1], np.int32)      # clamp to [0, seq]
    ctx = empty_dev((batch * seq, nh * d), "fp16")
    enc.op_attention(to_dev(qkv), to_dev(vlen), ctx, batch, seq)
    got = to_host(ctx).reshape(batch, seq, nh * d)
    ref = O.attention(qkv.astype(np.float64), np.clip(vlen, 0, seq))
    assert np.all(got[1] == 0) and np.all(got[2] == 0)   # n == 0: ctx = 0, no NaN
    assert np.all(np.isfinite(got))
    assert rel_l2(got, ref) < ATTN_REL_L2


def test_gemm_bounded_waits_never_fired():
    shape = (12, 64, 3072)
    wl, inp, enc, x64, vl, lw = _setup(shape, 5, 131)
    M = 5 * 131
    y = empty_dev((M, 768), "fp16")
    resid = to_dev(EI.random_array((M, 768), "fp16", seed=2))
    enc.op_ffn2_ln(0, to_dev(EI.random_array((M, 3072), "fp16", seed=1)), resid, y, M)
    assert enc.device_status() == 0


@pytest.mark.parametrize("form", ["erf", "tanh"])
@pytest.mark.parametrize("hidden,batch,seq", [(128, 3, 37), (256, 4, 96)], ids=["one-cta", "cta-pair"])
def test_gelu_epilogue_against_exact_erf(hidden, batch, seq, form):
    """W1 = I, b1 = 0 turns FFN1 into GELU of its FP16 input; inputs span [-8, 8].
    The result must be the exact GELU (erf form, or the tanh form) rounded once to FP16."""
    from transformer_encoder_bert_b200 import Encoder
    nh, d = hidden // 32, 32
    M = batch * seq
    lw = {k: v for k, v in _setup((nh, d, hidden), 1, 8)[1].layers[0].items()}
    lw["w_ff1"] = np.eye(hidden, dtype=np.float16)
    lw["b_ff1"] = np.zeros(hidden, np.float16)
    enc = Encoder(nh, d, hidden, [lw], "fp16")
    enc.set_gelu(form)
    h1 = np.linspace(-8, 8, M * hidden).astype(np.float16).reshape(M, hidden)
    u = empty_dev((M, hidden), "fp16")
    enc.op_ffn1(0, to_dev(h1), u, M)
    got = to_host(u).astype(np.float64)
    ref = O.GELU[form](h1.astype(np.float64))
    # one FP16 rounding of the exact value: |got - ref| <= half an ulp of |ref| (+ tiny slack)
    ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(got - ref) <= 0.5 * ulp + 1e-6)


@pytest.mark.parametrize("option", ["pair_tiles", "tma_store"])
@pytest.mark.parametrize("batch,seq", [(2, 128), (5, 131)], ids=str)
def test_alternative_gemm_paths(option, batch, seq):
    """The one-CTA tile path (used for small M) and the direct-store epilogue (used when
    the output map cannot be built) on shapes that normally take the pair / TMA-store path."""
    shape = (12, 64, 3072)
    nh, d, F = shape
    H = nh * d
    M = batch * seq
    wl, inp, enc, x64, vl, lw = _setup(shape, batch, seq)
    assert enc.get_option(option)
    enc.set_option(option, False)
    h1 = EI.random_array((M, H), "fp16", seed=12)
    u = empty_dev((M, F), "fp16")
    enc.op_ffn1(0, to_dev(h1), u, M)
    ref = O.ffn1_gelu(h1.astype(np.float64), lw["w_ff1"], lw["b_ff1"])
    got = to_host(u)
    assert rel_l2(got, ref) < GEMM_REL_L2 and max_abs(got, ref) < _ulp_bound(ref)
    out = empty_dev((3, batch, nh, seq, d), "fp16")
    enc.op_qkv(0, to_dev(inp.x), out, batch, seq)
    ref = O.head_split(O.qkv_projection(x64.reshape(-1, H), lw["w_qkv"], lw["b_qkv"]), batch, seq, nh, d)
    assert rel_l2(to_host(out), ref) < GEMM_REL_L2
    # bias + residual epilogue: residual through TMA, or per-lane loads without TMA stores
    ctx = EI.random_array((M, H), "fp16", seed=15)
    resid = EI.random_array((M, H), "fp16", seed=16)
    z = empty_dev((M, H), "fp16")
    enc.op_out_proj_ln(0, to_dev(ctx), to_dev(resid), z, M)
    ref = O.bias_residual_layernorm(ctx.astype(np.float64) @ lw["w_o"], lw["b_o"], resid.astype(np.float64),
                                    lw["ln1_g"], lw["ln1_b"])
    got = to_host(z)
    assert rel_l2(got, ref) < GEMM_REL_L2 and max_abs(got, ref) < LN_MAX_ABS


@pytest.mark.parametrize("batch,seq", [(3, 128), (4, 96), (3, 65), (2, 200)], ids=str)
def test_attention_mma_sync_path_for_long_sequences(batch, seq):
    """Size-64 heads on sequences longer than 64 run on the tensor-core (tcgen05)
    kernels; the mma.sync kernel for the same shapes stays checked through the
    tc_attention option."""
    shape = (12, 64, 3072)
    nh, d, _ = shape
    wl, inp, enc, x64, vl, lw = _setup(shape, batch, seq)
    enc.set_option("tc_attention", False)
    qkv = EI.random_array((3, batch, nh, seq, d), "fp16", seed=17)
    vlen = np.array([seq] + [max(1, seq // (i + 2)) for i in range(batch - 1)], np.int32)
    ctx = empty_dev((batch * seq, nh * d), "fp16")
    enc.op_attention(to_dev(qkv), to_dev(vlen), ctx, batch, seq)
    got = to_host(ctx).reshape(batch, seq, nh * d)
    ref = O.attention(qkv.astype(np.float64), vlen)
    assert rel_l2(got, ref) < ATTN_REL_L2


@pytest.mark.parametrize("seq", [128, 96, 80], ids=str)
def test_attention_tc_items_beyond_the_resident_grid(seq):
    """64 < seq <= 128: the persistent tcgen05 kernel runs about four CTAs per
    SM, each taking (sequence, head) items in turn and loading the next item's
    Q, K and V while it computes the current one.  64 sequences x 12 heads =
    768 items, more than the resident CTAs; lengths 0 (zero rows), 1, multiples of 16
    and their neighbours, and seq itself.  Every row of every item against the
    oracle; a second call gives the same bits."""
    shape = (12, 64, 3072)
    nh, d, _ = shape
    batch = 64
    wl, inp, enc, x64, vl, lw = _setup(shape, batch, seq)
    qkv = EI.random_array((3, batch, nh, seq, d), "fp16", seed=seq)
    base = [0, 1, 15, 16, 17, 31, 32, 33, 47, 63, 64, 65, seq - 1, seq]
    vlen = np.array([base[i % len(base)] if i % 3 else (i * 37) % (seq + 1) for i in range(batch)], np.int32)
    ctx = empty_dev((batch * seq, nh * d), "fp16")
    enc.op_attention(to_dev(qkv), to_dev(vlen), ctx, batch, seq)
    got = to_host(ctx).reshape(batch, seq, nh * d)
    ref = O.attention(qkv.astype(np.float64), vlen)
    assert np.all(np.isfinite(got))
    for b in np.nonzero(vlen == 0)[0]:
        assert np.all(got[b] == 0)
    assert rel_l2(got, ref) < ATTN_REL_L2
    assert max_abs(got, ref) < 4 * _ulp_bound(ref)
    ctx2 = empty_dev((batch * seq, nh * d), "fp16")
    enc.op_attention(to_dev(qkv), to_dev(vlen), ctx2, batch, seq)
    assert np.array_equal(to_host(ctx2).reshape(batch, seq, nh * d), got)
    assert enc.device_status() == 0


@pytest.mark.parametrize("batch,seq,lens", [
    (3, 300, [300, 129, 1]),          # 3 query blocks: the second CTA's upper block lies past seq
    (2, 256, [256, 128]),             # key blocks exactly full; one block only
    (4, 512, [512, 385, 257, 130]),   # 1 or 2 valid keys in the last block
    (2, 129, [129, 65]),
], ids=str)
@pytest.mark.parametrize("key_boost", [1.0, 6.0], ids=["plain", "rescaled"])
def test_attention_long_sequences_tensor_core(batch, seq, lens, key_boost):
    """Sequences longer than one 128-key block: the tensor-core kernel walks the
    key blocks with a running maximum.  key_boost multiplies the keys of block j
    by key_boost**j, so later blocks raise the row maximum far above the first
    block's and the accumulated output and row sum must be rescaled."""
    shape = (16, 64, 4096)
    nh, d, _ = shape
    wl, inp, enc, x64, vl, lw = _setup(shape, batch, seq)
    qkv = EI.random_array((3, batch, nh, seq, d), "fp16", seed=29).astype(np.float32)
    for j in range(1, (seq + 127) // 128):
        qkv[1, :, :, 128 * j:128 * (j + 1)] *= key_boost ** j
    qkv = qkv.astype(np.float16)
    vlen = np.array(lens, np.int32)
    ctx = empty_dev((batch * seq, nh * d), "fp16")
    enc.op_attention(to_dev(qkv), to_dev(vlen), ctx, batch, seq)
    got = to_host(ctx).reshape(batch, seq, nh * d)
    ref = O.attention(qkv.astype(np.float64), vlen)
    assert np.all(np.isfinite(got))
    assert rel_l2(got, ref) < ATTN_REL_L2
    assert max_abs(got, ref) < 4 * _ulp_bound(ref)
    assert enc.device_status() == 0


@pytest.mark.parametrize("batch,seq", [(1, 32), (8, 32), (1, 7), (3, 37)], ids=str)
def test_split_k_gemms(batch, seq):
    """At small M the GEMMs run split-K: a cluster of CTAs shares each 128x128 tile,
    each CTA one range of the k-blocks, and the partial tiles are summed in rank
    order through distributed shared memory.  Every epilogue (head split, plain,
    erf-GELU, tanh-GELU, bias + residual + LayerNorm) against its oracle step; a repeated call is bit-identical
    (the sum's order does not depend on timing); the unsplit kernel
    (split_k option off) agrees within the GEMM bound."""
    shape = (12, 64, 3072)
    nh, d, F = shape
    H = nh * d
    M = batch * seq
    ctx = EI.random_array((M, H), "fp16", seed=31)
    h1 = EI.random_array((M, H), "fp16", seed=32)
    uu = EI.random_array((M, F), "fp16", seed=33, std=0.5)

    def run(enc):
        qkv = empty_dev((3, batch, nh, seq, d), "fp16")
        enc.op_qkv(0, to_dev(inp.x), qkv, batch, seq)
        a = empty_dev((M, H), "fp16")
        enc.op_out_proj_ln(0, to_dev(ctx), to_dev(h1), a, M)
        u = empty_dev((M, F), "fp16")
        enc.op_ffn1(0, to_dev(h1), u, M)
        enc.set_gelu("tanh")
        ut = empty_dev((M, F), "fp16")
        enc.op_ffn1(0, to_dev(h1), ut, M)
        enc.set_gelu("erf")
        y = empty_dev((M, H), "fp16")
        enc.op_ffn2_ln(0, to_dev(uu), to_dev(ctx), y, M)
        return [to_host(t) for t in (qkv, a, u, ut, y)]

    wl, inp, enc, x64, vl, lw = _setup(shape, batch, seq)
    got = run(enc)
    refs = [
        O.head_split(O.qkv_projection(x64.reshape(-1, H), lw["w_qkv"], lw["b_qkv"]), batch, seq, nh, d),
        O.bias_residual_layernorm(ctx.astype(np.float64) @ lw["w_o"], lw["b_o"], h1.astype(np.float64),
                                  lw["ln1_g"], lw["ln1_b"]),
        O.ffn1_gelu(h1.astype(np.float64), lw["w_ff1"], lw["b_ff1"]),
        O.ffn1_gelu(h1.astype(np.float64), lw["w_ff1"], lw["b_ff1"], gelu="tanh"),
        O.bias_residual_layernorm(uu.astype(np.float64) @ lw["w_ff2"], lw["b_ff2"], ctx.astype(np.float64),
                                  lw["ln2_g"], lw["ln2_b"]),
    ]
    for g, r in zip(got, refs):
        assert rel_l2(g, r) < GEMM_REL_L2 and max_abs(g, r) < max(_ulp_bound(r), LN_MAX_ABS)
    again = run(enc)
    for g, a in zip(got, again):
        assert np.array_equal(g, a)
    assert enc.device_status() == 0
    wl, inp, enc1, x64, vl, lw = _setup(shape, batch, seq)
    enc1.set_option("split_k", False)
    for g, r in zip(got, run(enc1)):
        assert rel_l2(g, r) < GEMM_REL_L2
