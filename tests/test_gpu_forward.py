"""The whole encoder stack through the C ABI against the float64 oracle (GPU).

Tolerances on valid tokens (query rows i < valid_len):
  FP32 mode:                 relative L2 <= 1e-5 per layer
  FP16 storage, FP32 accum.: relative L2 <= 5e-3 and max abs <= 3e-2 after one
                             layer; relative L2 <= 2e-2 after 12 layers.
The full-size workloads run in the same launch configuration the bench times;
the oracle checks a seeded sample of their sequences (sequences never
interact), always including the first, the last and a shortest one.
"""
import numpy as np
import pytest

import encoder_inputs as EI
from oracle import encoder_oracle as O
from parity_utils import (FP16_LAYER_MAX_ABS, FP16_LAYER_REL_L2, FP16_STACK_REL_L2, FP32_LAYER_REL_L2,
                          encoder_from_inputs, max_abs, rel_l2, to_dev, to_host, valid_mask)

pytestmark = pytest.mark.gpu


def _run(inp, enc=None):
    enc = enc or encoder_from_inputs(inp)
    out = enc.forward(to_dev(inp.x), to_dev(inp.valid_len))
    return enc, to_host(out)


def _oracle(inp, seqs=None):
    x64, vl, layers = inp.as_float64()
    sh = inp.workload.shape
    return O.encoder_forward(x64, vl, layers, sh.head_num, sh.size_per_head, seqs=seqs)


def _check(got, ref, vl, seq, rel_tol, abs_tol=None):
    m = valid_mask(vl, seq)
    r = rel_l2(got, ref, m)
    assert r < rel_tol, f"relative L2 {r:.3e} >= {rel_tol:g}"
    if abs_tol is not None:
        a = max_abs(got, ref, m)
        assert a < abs_tol, f"max abs {a:.3e} >= {abs_tol:g}"
    return r


def test_tiny_fp32_one_layer():
    inp = EI.make_inputs(EI.named_workload("tiny-fp32", 1))
    _, got = _run(inp)
    _check(got, _oracle(inp), inp.valid_len, 32, FP32_LAYER_REL_L2)


def test_fp32_two_layers_ragged():
    sh = EI.EncoderShape(12, 64, 3072, 2)
    inp = EI.make_inputs(EI.Workload("fp32-2L", sh, 3, 45, "fp32", 1, 45, ln_affine_random=True))
    _, got = _run(inp)
    _check(got, _oracle(inp), inp.valid_len, 45, 2 * FP32_LAYER_REL_L2)


def test_bert_base_one_layer_fp16():
    wl = EI.named_workload("bert-base-s32", 8)
    inp = EI.make_inputs(wl.with_(shape=EI.EncoderShape(12, 64, 3072, 1)))
    _, got = _run(inp)
    _check(got, _oracle(inp), inp.valid_len, 32, FP16_LAYER_REL_L2, FP16_LAYER_MAX_ABS)


def test_bert_base_twelve_layers_fp16():
    inp = EI.make_inputs(EI.named_workload("bert-base-s32", 8))
    _, got = _run(inp)
    _check(got, _oracle(inp), inp.valid_len, 32, FP16_STACK_REL_L2)


@pytest.mark.parametrize("seq", [1, 7, 31, 32, 33, 96, 127, 128, 129, 512])
@pytest.mark.parametrize("vl_kind", ["one", "full"])
def test_edge_sequence_lengths_one_layer(seq, vl_kind):
    sh = EI.EncoderShape(12, 64, 3072, 1)
    batch = 3
    lo = hi = 1 if vl_kind == "one" else seq
    inp = EI.make_inputs(EI.Workload("edge", sh, batch, seq, "fp16", lo, hi, seed=seq))
    _, got = _run(inp)
    _check(got, _oracle(inp), inp.valid_len, seq, FP16_LAYER_REL_L2, FP16_LAYER_MAX_ABS)


@pytest.mark.parametrize("nh,d,F", [(4, 32, 512), (12, 64, 3072), (16, 64, 4096), (8, 128, 2048), (2, 128, 256)])
def test_head_structures_two_layers(nh, d, F):
    sh = EI.EncoderShape(nh, d, F, 2)
    inp = EI.make_inputs(EI.Workload("heads", sh, 5, 53, "fp16", 1, 53, seed=nh + d, ln_affine_random=True))
    _, got = _run(inp)
    _check(got, _oracle(inp), inp.valid_len, 53, 2 * FP16_LAYER_REL_L2)


FULL_SIZE = [
    ("bert-base-s32", 512, None, 4),
    ("pruned-s32", 1024, None, 6),
    ("bert-base", 256, 128, 3),
    ("bert-base", 256, 96, 3),
    ("bert-large", 256, 128, 3),
    ("bert-large", 32, 512, 3),
]


@pytest.mark.parametrize("kind,batch,seq,nsample", FULL_SIZE, ids=lambda v: str(v))
def test_full_size_workloads_sampled(kind, batch, seq, nsample):
    wl = EI.named_workload(kind, batch, seq)
    inp = EI.make_inputs(wl)
    _, got = _run(inp)
    assert np.all(np.isfinite(got[valid_mask(inp.valid_len, wl.seq)]))
    seqs = EI.sample_sequences(wl.batch, nsample, inp.valid_len)
    ref = _oracle(inp, seqs)
    _check(got[seqs], ref, inp.valid_len[seqs], wl.seq, FP16_STACK_REL_L2)


@pytest.mark.parametrize("dtype", ["fp16", "fp32"])
def test_tanh_gelu_variant(dtype):
    sh = EI.EncoderShape(12, 64, 3072, 2)
    inp = EI.make_inputs(EI.Workload("tanh", sh, 4, 40, dtype, 1, 40, seed=6, ln_affine_random=True))
    enc = encoder_from_inputs(inp)
    enc.set_gelu("tanh")
    got = to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len)))
    x64, vl, layers = inp.as_float64()
    ref = O.encoder_forward(x64, vl, layers, 12, 64, gelu="tanh")
    tol = 2 * (FP16_LAYER_REL_L2 if dtype == "fp16" else FP32_LAYER_REL_L2)
    _check(got, ref, vl, 40, tol)
    # and it differs measurably from the erf form (the switch takes effect)
    ref_erf = O.encoder_forward(x64, vl, layers, 12, 64, gelu="erf")
    assert rel_l2(ref, ref_erf, valid_mask(vl, 40)) > 1e-6


def test_padding_tokens_do_not_change_valid_outputs():
    sh = EI.EncoderShape(12, 64, 3072, 2)
    inp = EI.make_inputs(EI.Workload("pad", sh, 6, 70, "fp16", 5, 60, seed=4))
    enc, got = _run(inp)
    x2 = inp.x.copy()
    rng = np.random.default_rng(0)
    for b, n in enumerate(inp.valid_len):
        x2[b, n:] = rng.normal(0, 3, x2[b, n:].shape).astype(np.float16)
    got2 = to_host(enc.forward(to_dev(x2), to_dev(inp.valid_len)))
    m = valid_mask(inp.valid_len, 70)
    assert np.array_equal(got[m], got2[m])


def test_permutation_equivariance_over_valid_tokens():
    sh = EI.EncoderShape(12, 64, 3072, 2)
    inp = EI.make_inputs(EI.Workload("perm", sh, 4, 48, "fp16", 20, 48, seed=9))
    enc, got = _run(inp)
    rng = np.random.default_rng(1)
    x2 = inp.x.copy()
    perms = []
    for b, n in enumerate(inp.valid_len):
        p = np.concatenate([rng.permutation(n), np.arange(n, 48)])
        perms.append(p)
        x2[b] = inp.x[b, p]
    got2 = to_host(enc.forward(to_dev(x2), to_dev(inp.valid_len)))
    for b, n in enumerate(inp.valid_len):
        assert rel_l2(got2[b, :n], got[b, perms[b]][:n]) < 2 * FP16_LAYER_REL_L2


def test_identical_tokens_give_identical_outputs():
    sh = EI.EncoderShape(12, 64, 3072, 2)
    inp = EI.make_inputs(EI.Workload("same", sh, 2, 33, "fp16", 33, 33, seed=2))
    inp.x[:] = inp.x[:, :1]
    _, got = _run(inp)
    assert np.max(np.abs(got - got[:, :1])) < 1e-2


def test_deterministic_and_host_entry_point_matches():
    inp = EI.make_inputs(EI.named_workload("bert-base-s32", 16))
    enc, got = _run(inp)
    again = to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len)))
    assert np.array_equal(got, again)
    host = enc.forward_host(inp.x, inp.valid_len)
    assert np.array_equal(got, host)
    assert enc.device_status() == 0


def test_plain_stream_order_is_bit_identical():
    """The pdl option off launches every kernel in plain stream order; the kernels
    are the same, so the output is the same bit for bit, and switching it back
    on restores the default."""
    inp = EI.make_inputs(EI.named_workload("bert-base-s32", 16))
    enc, got = _run(inp)
    assert enc.get_option("pdl")
    enc.set_option("pdl", False)
    assert not enc.get_option("pdl")
    plain = to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len)))
    assert np.array_equal(got, plain)
    enc.set_option("pdl", True)
    assert np.array_equal(got, to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len))))
    assert enc.device_status() == 0


def test_option_argument_checks():
    inp = EI.make_inputs(EI.Workload("args", EI.EncoderShape(4, 32, 512, 1), 2, 8, "fp16", 1, 8))
    enc = encoder_from_inputs(inp)
    assert enc.lib.enc_set_option(enc.handle, 2, 2) == 1       # value not 0 or 1: ENC_ERR_INVALID_ARG
    assert enc.lib.enc_set_option(enc.handle, 99, 1) == 1      # unknown option
    assert enc.lib.enc_set_option(None, 2, 1) == 1             # null handle
    assert enc.get_option("tc_attention") and enc.get_option("ln_fuse_out_proj") == 1
    assert enc.lib.enc_set_option(enc.handle, 5, 3) == 1       # the fusion switches take 0..2
    assert enc.lib.enc_set_option(enc.handle, 5, 2) == 0


def test_host_argument_checks():
    import torch
    from transformer_encoder_bert_b200 import EncError
    inp = EI.make_inputs(EI.Workload("args", EI.EncoderShape(4, 32, 512, 1), 2, 8, "fp16", 1, 8))
    enc = encoder_from_inputs(inp)
    x = to_dev(inp.x)
    vl = to_dev(inp.valid_len)
    with pytest.raises(EncError) as e:
        enc.forward(x, vl, out=x)                       # out overlaps x
    assert e.value.status == 1
    buf = torch.empty(x.numel() + 8, dtype=torch.float16, device="cuda")
    with pytest.raises(EncError) as e:
        enc.forward(x, vl, out=buf[1:1 + x.numel()].view_as(x))     # not 16-byte aligned
    assert e.value.status == 1
    with pytest.raises(EncError):
        enc.op_ffn1(3, x, x, 16)                        # layer out of range


def test_recorded_forward_replays_bit_exact():
    import torch
    from transformer_encoder_bert_b200 import EncError
    inp = EI.make_inputs(EI.named_workload("bert-base-s32", 8))
    enc = encoder_from_inputs(inp)
    x, vl = to_dev(inp.x), to_dev(inp.valid_len)
    ref = to_host(enc.forward(x, vl))
    out = torch.zeros_like(x)
    g = enc.record(x, vl, out)
    assert np.all(to_host(out) == 0)                  # recording runs nothing
    n0 = enc.launch_count()
    s = torch.cuda.Stream()
    for _ in range(3):
        g.launch(stream=s)
    s.synchronize()
    assert enc.launch_count() - n0 == 3 * enc.kernels_per_forward(8, 32)
    assert np.array_equal(to_host(out), ref)
    # new input values in the same buffers are picked up at replay time
    x2 = EI.make_inputs(EI.named_workload("bert-base-s32", 8).with_(seed=5)).x
    x.copy_(to_dev(x2))
    g.launch()
    torch.cuda.synchronize()
    assert np.array_equal(to_host(out), to_host(enc.forward(x, vl)))
    # the workspace is pinned while the graph exists
    big = torch.empty((64, 32, 768), dtype=torch.float16, device="cuda")
    with pytest.raises(EncError):
        enc.forward(big, to_dev(np.full(64, 32, np.int32)))
    g.close()
    enc.forward(big, to_dev(np.full(64, 32, np.int32)))
    assert enc.device_status() == 0


@pytest.mark.parametrize("chunks,layers", [(2, 12), (4, 12), (4, 2), (3, 3)])
def test_host_entry_point_chunked_pipeline_matches_device_forward(chunks, layers):
    # 256 x 32 tokens: the first and last layers run chunk by chunk while the
    # copies of the other chunks are in flight.  Bit-identical to the whole-batch
    # forward when the chunks run the same kernels; when the chunks are too small
    # for the GEMMs that fuse the LayerNorm (which keep z in FP32 instead of
    # rounding it to FP16 first), within the FP16 per-layer bound.
    import torch
    wl = EI.named_workload("bert-base-s32", 256)
    inp = EI.make_inputs(wl.with_(shape=EI.EncoderShape(12, 64, 3072, layers)))
    enc = encoder_from_inputs(inp)
    dev = to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len)))
    same_kernels = enc.kernels_per_forward(256 // chunks, 32) == enc.kernels_per_forward(256, 32)
    enc.set_host_chunks(chunks)
    hx = torch.from_numpy(inp.x).pin_memory()
    hvl = torch.from_numpy(inp.valid_len).pin_memory()
    hout = torch.empty_like(hx).pin_memory()
    enc.forward_host_ptr(hx.data_ptr(), hvl.data_ptr(), hout.data_ptr(), 256, 32)
    m = valid_mask(inp.valid_len, 32)
    if same_kernels:
        assert np.array_equal(hout.numpy(), dev)
    else:
        assert rel_l2(hout.numpy(), dev, m) < FP16_LAYER_REL_L2
    pageable = enc.forward_host(inp.x, inp.valid_len)
    assert np.array_equal(pageable, hout.numpy())


def test_pipelined_host_entry_point_matches_device_forward():
    """enc_forward_host_async: four different batches in flight through the two
    staging slots (each call's input copy and the previous call's output copy
    overlap the encoder); every output equals the device forward bit for bit,
    and a synchronous host call after them sees the slots free."""
    import torch
    wl = EI.named_workload("bert-base-s32", 64)
    sh = EI.EncoderShape(12, 64, 3072, 2)
    batches = [EI.make_inputs(wl.with_(shape=sh, seed=100 + i)) for i in range(4)]
    enc = encoder_from_inputs(batches[0])        # one set of weights; x and valid_len differ per batch
    refs = [to_host(enc.forward(to_dev(b.x), to_dev(b.valid_len))) for b in batches]
    hx = [torch.from_numpy(b.x).pin_memory() for b in batches]
    hvl = [torch.from_numpy(b.valid_len).pin_memory() for b in batches]
    hout = [torch.zeros_like(t).pin_memory() for t in hx]
    stream = torch.cuda.current_stream()
    for i in range(4):
        enc.forward_host_async_ptr(hx[i].data_ptr(), hvl[i].data_ptr(), hout[i].data_ptr(), 64, 32)
    enc.host_join()
    stream.synchronize()
    for i in range(4):
        assert np.array_equal(hout[i].numpy(), refs[i]), i
    again = enc.forward_host(batches[1].x, batches[1].valid_len)
    assert np.array_equal(again, refs[1])
    assert enc.device_status() == 0


def test_pipelined_host_entry_point_alternating_shapes():
    """enc_forward_host_async with calls of different sizes in flight together
    (64, 16, 64, 16, 48 sequences): the smaller call's staging slot must lie
    outside the larger call's, whose encoder run and copies may still be in
    flight.  Every output equals the device forward bit for bit."""
    import torch
    sh = EI.EncoderShape(12, 64, 3072, 2)
    wl = EI.named_workload("bert-base-s32", 64).with_(shape=sh)
    sizes = [64, 16, 64, 16, 48]
    batches = [EI.make_inputs(wl.with_(batch=b, seed=200 + i)) for i, b in enumerate(sizes)]
    enc = encoder_from_inputs(batches[0])
    refs = [to_host(enc.forward(to_dev(b.x), to_dev(b.valid_len))) for b in batches]
    hx = [torch.from_numpy(b.x).pin_memory() for b in batches]
    hvl = [torch.from_numpy(b.valid_len).pin_memory() for b in batches]
    hout = [torch.zeros_like(t).pin_memory() for t in hx]
    for i, b in enumerate(sizes):
        enc.forward_host_async_ptr(hx[i].data_ptr(), hvl[i].data_ptr(), hout[i].data_ptr(), b, 32)
    enc.host_join()
    torch.cuda.current_stream().synchronize()
    for i in range(len(sizes)):
        assert np.array_equal(hout[i].numpy(), refs[i]), i
    assert enc.device_status() == 0


# ---------------------------------------------------------------- padding removal

@pytest.mark.parametrize("seq,lo,hi,L", [(32, 1, 32, 12), (37, 0, 37, 2), (96, 64, 96, 2), (128, 64, 128, 2),
                                         (512, 256, 512, 1)])
def test_packed_forward_matches_oracle_and_zeroes_padding(seq, lo, hi, L):
    sh = EI.EncoderShape(12, 64, 3072, L)
    inp = EI.make_inputs(EI.Workload("packed", sh, 6, seq, "fp16", lo, hi, seed=seq + L))
    if lo == 0:
        inp.valid_len[1] = 0                      # an empty sequence in the middle of the batch
    enc = encoder_from_inputs(inp)
    dense = to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len)))
    enc.set_packing(True)
    assert enc.kernels_per_forward(6, seq) == 7 * L + 3
    got = to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len)))
    m = valid_mask(inp.valid_len, seq)
    assert np.all(got[~m] == 0)
    tol = FP16_STACK_REL_L2 if L > 2 else L * FP16_LAYER_REL_L2
    _check(got, _oracle(inp), inp.valid_len, seq, tol)
    assert rel_l2(got, dense, m) < tol
    assert enc.device_status() == 0


@pytest.mark.parametrize("seq", [128, 100], ids=str)
def test_packed_forward_many_attention_items(seq):
    """Padding removal with more (sequence, head) items than the persistent
    tcgen05 attention keeps resident (64 x 12 = 768): empty sequences (no rows
    in the packed layout) among ragged ones; one layer against the oracle, and
    the padded rows zero."""
    sh = EI.EncoderShape(12, 64, 3072, 1)
    inp = EI.make_inputs(EI.Workload("packed-items", sh, 64, seq, "fp16", 0, seq, seed=seq))
    inp.valid_len[::9] = 0
    enc = encoder_from_inputs(inp)
    enc.set_packing(True)
    got = to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len)))
    m = valid_mask(inp.valid_len, seq)
    assert np.all(got[~m] == 0)
    _check(got, _oracle(inp), inp.valid_len, seq, FP16_LAYER_REL_L2)
    assert enc.device_status() == 0


@pytest.mark.parametrize("batch,seq,per_layer", [
    (64, 96, 7),      # 24 row blocks on 22 fused-cluster slots: neither LayerNorm fused
    (64, 128, 6),     # 32 row blocks: FFN2 only
    (128, 96, 6),     # 48: FFN2 only
    (128, 128, 5),    # 64: both
    (256, 96, 6),     # 96: FFN2 only
    (512, 32, 5),     # 64: both
    (256, 128, 5),    # 128: both
], ids=str)
def test_layernorm_fusion_follows_wave_fill(batch, seq, per_layer):
    """The default LayerNorm fusion compares how full the last wave of the
    fused kernel (one 6-CTA cluster per 256 rows) and of the unfused GEMM (a CTA
    pair per 256x256 tile) would be: the kernels per layer at BERT-Base token
    counts from 6144 to 32768, and one layer at the first of them against the
    same encoder with both fusions forced on."""
    sh = EI.EncoderShape(12, 64, 3072, 1)
    inp = EI.make_inputs(EI.Workload("wave-fill", sh, batch, seq, "fp16", 1, seq, seed=batch + seq))
    enc = encoder_from_inputs(inp)
    assert enc.kernels_per_forward(batch, seq) == per_layer
    if (batch, seq) == (64, 96):
        got = to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len)))
        enc.set_option("ln_fuse_out_proj", 2)
        enc.set_option("ln_fuse_ffn2", 2)
        assert enc.kernels_per_forward(batch, seq) == 5
        fused = to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len)))
        m = valid_mask(inp.valid_len, seq)
        assert rel_l2(got, fused, m) < FP16_LAYER_REL_L2
        assert enc.device_status() == 0


PACKED_FULL_SIZE = [
    ("bert-base-s32", 512, None, 4),
    ("bert-base", 256, 128, 3),
    ("bert-large", 256, 128, 3),
]


@pytest.mark.parametrize("kind,batch,seq,nsample", PACKED_FULL_SIZE, ids=lambda v: str(v))
def test_packed_full_size_against_oracle(kind, batch, seq, nsample):
    """Padding removal at the sizes the bench runs it: every GEMM takes the 2-CTA
    tiles chosen from the padded token count and reads the real count T from the
    device, and for hidden sizes up to 768 the output-projection and FFN2 GEMMs
    write LayerNorms 1 and 2 themselves (5 launches per layer; 7 for BERT-Large),
    plus the offsets, pack and unpack kernels.  A seeded sample of sequences (the first, the last and a shortest one
    among them) against the oracle; every padded row is zero."""
    wl = EI.named_workload(kind, batch, seq)
    inp = EI.make_inputs(wl)
    enc = encoder_from_inputs(inp)
    enc.set_packing(True)
    L = wl.shape.num_layers
    per_layer = 5 if wl.shape.hidden <= 768 else 7
    assert enc.kernels_per_forward(wl.batch, wl.seq) == per_layer * L + 3
    got = to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len)))
    m = valid_mask(inp.valid_len, wl.seq)
    assert np.all(got[~m] == 0)
    assert np.all(np.isfinite(got[m]))
    seqs = EI.sample_sequences(wl.batch, nsample, inp.valid_len)
    ref = _oracle(inp, seqs)
    _check(got[seqs], ref, inp.valid_len[seqs], wl.seq, FP16_STACK_REL_L2)
    assert enc.device_status() == 0


def test_packed_mode_replays_and_host_entry_point():
    import torch
    inp = EI.make_inputs(EI.named_workload("bert-base-s32", 128))
    enc = encoder_from_inputs(inp)
    enc.set_packing(True)
    x, vl = to_dev(inp.x), to_dev(inp.valid_len)
    ref = to_host(enc.forward(x, vl))
    out = torch.empty_like(x)
    g = enc.record(x, vl, out)
    g.launch()
    torch.cuda.synchronize()
    assert np.array_equal(to_host(out), ref)
    g.close()
    assert np.array_equal(enc.forward_host(inp.x, inp.valid_len), ref)


def test_packed_mode_needs_fp16():
    from transformer_encoder_bert_b200 import EncError
    inp = EI.make_inputs(EI.named_workload("tiny-fp32", 1))
    enc = encoder_from_inputs(inp)
    with pytest.raises(EncError) as e:
        enc.set_packing(True)
    assert e.value.status == 2


# ---------------------------------------------------------------- single-launch small-batch forward

@pytest.mark.parametrize("batch", [1, 8])
def test_single_launch_forward_bert_base_against_oracle(batch):
    """BERT-Base, 12 layers, seq 32, batch 1 and 8: one persistent kernel runs the
    whole stack (grid-wide barriers between the steps, LayerNorms applied as the
    next GEMM loads its operand).  Against the oracle on every sequence, and
    against the per-step kernels within the 12-layer bound."""
    inp = EI.make_inputs(EI.named_workload("bert-base-s32", batch))
    enc = encoder_from_inputs(inp)
    assert not enc.get_option("persistent")       # off by default: the per-step graph measured faster
    enc.set_option("persistent", True)
    assert enc.kernels_per_forward(batch, 32) == 1
    n0 = enc.launch_count()
    got = to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len)))
    assert enc.launch_count() - n0 == 1
    _check(got, _oracle(inp), inp.valid_len, 32, FP16_STACK_REL_L2)
    enc.set_option("persistent", False)
    assert enc.kernels_per_forward(batch, 32) > 1
    per_step = to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len)))
    assert rel_l2(got, per_step, valid_mask(inp.valid_len, 32)) < FP16_STACK_REL_L2
    assert enc.device_status() == 0


@pytest.mark.parametrize("nh,d,F,L,batch,seq", [
    (4, 32, 512, 2, 5, 37),        # pruned structure, ragged token count (185 rows)
    (16, 64, 4096, 2, 2, 128),     # BERT-Large structure, 256 tokens (FFN2 in units of 8 features)
    (8, 128, 2048, 2, 3, 21),      # size-128 heads
    (12, 64, 3072, 1, 1, 1),       # one token
    (12, 64, 3072, 2, 4, 64),      # 256 tokens, longer sequences
], ids=str)
def test_single_launch_forward_structures(nh, d, F, L, batch, seq):
    sh = EI.EncoderShape(nh, d, F, L)
    inp = EI.make_inputs(EI.Workload("single", sh, batch, seq, "fp16", 1, seq, seed=nh + seq,
                                     ln_affine_random=True))
    inp.valid_len[0] = seq
    enc = encoder_from_inputs(inp)
    enc.set_option("persistent", True)
    assert enc.kernels_per_forward(batch, seq) == 1
    got = to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len)))
    _check(got, _oracle(inp), inp.valid_len, seq, L * FP16_LAYER_REL_L2)
    assert enc.device_status() == 0


def test_single_launch_forward_empty_sequence_and_tanh_gelu():
    sh = EI.EncoderShape(12, 64, 3072, 2)
    inp = EI.make_inputs(EI.Workload("single-empty", sh, 4, 33, "fp16", 1, 33, seed=8))
    inp.valid_len[2] = 0                       # no valid key: ctx = 0 for that sequence
    enc = encoder_from_inputs(inp)
    enc.set_option("persistent", True)
    enc.set_gelu("tanh")
    assert enc.kernels_per_forward(4, 33) == 1
    got = to_host(enc.forward(to_dev(inp.x), to_dev(inp.valid_len)))
    x64, vl, layers = inp.as_float64()
    ref = O.encoder_forward(x64, vl, layers, 12, 64, gelu="tanh")
    _check(got, ref, vl, 33, 2 * FP16_LAYER_REL_L2)
    assert np.all(np.isfinite(got))
    assert enc.device_status() == 0


def test_single_launch_forward_replays_and_is_deterministic():
    import torch
    inp = EI.make_inputs(EI.named_workload("bert-base-s32", 2))
    enc = encoder_from_inputs(inp)
    enc.set_option("persistent", True)
    x, vl = to_dev(inp.x), to_dev(inp.valid_len)
    ref = to_host(enc.forward(x, vl))
    assert np.array_equal(ref, to_host(enc.forward(x, vl)))      # fixed summation order
    out = torch.zeros_like(x)
    g = enc.record(x, vl, out)
    n0 = enc.launch_count()
    for _ in range(3):
        g.launch()
    torch.cuda.synchronize()
    assert enc.launch_count() - n0 == 3
    assert np.array_equal(to_host(out), ref)
    g.close()
    assert enc.device_status() == 0


def test_single_launch_forward_wait_timeout_sets_status():
    """Failure detection without a GPU fault: with the test_stall option one CTA
    waits on a flag that nothing sets instead of joining the first grid-wide
    barrier; every wait of that launch gives up after 20 ms, the kernel returns
    and reports status 1.  The context stays usable: the next forward is correct."""
    inp = EI.make_inputs(EI.named_workload("bert-base-s32", 1).with_(shape=EI.EncoderShape(12, 64, 3072, 2)))
    enc = encoder_from_inputs(inp)
    enc.set_option("persistent", True)
    x, vl = to_dev(inp.x), to_dev(inp.valid_len)
    enc.set_option("test_stall", True)
    enc.forward(x, vl)
    assert enc.device_status() == 1
    enc.set_option("test_stall", False)
    got = to_host(enc.forward(x, vl))
    _check(got, _oracle(inp), inp.valid_len, 32, 2 * FP16_LAYER_REL_L2)
    assert enc.device_status() == 0
