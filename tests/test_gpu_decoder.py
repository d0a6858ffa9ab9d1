"""The decoder forward through the C ABI against the float64 decoder oracle (GPU).

FP16 storage, FP32 accumulation; tolerances on valid target rows (i < tgt_len)
as for the encoder: relative L2 <= 5e-3 per layer (and max abs <= 3e-2 after
one layer).  Shapes span several 64-row query blocks and 64-key blocks with
ragged tails, every head size, target and memory lengths of different sizes,
and empty target and memory sequences.
"""
import numpy as np
import pytest

import encoder_inputs as EI
from oracle import decoder_oracle as DO
from parity_utils import FP16_LAYER_MAX_ABS, FP16_LAYER_REL_L2, max_abs, rel_l2, to_dev, to_host, valid_mask

pytestmark = pytest.mark.gpu


def _decoder(inp):
    from transformer_encoder_bert_b200 import Decoder
    sh = inp.workload.shape
    return Decoder(sh.head_num, sh.size_per_head, sh.ffn_dim, inp.layers)


def _run(dec, inp):
    return to_host(dec.forward(to_dev(inp.y), to_dev(inp.tgt_len), to_dev(inp.mem), to_dev(inp.mem_len)))


def _oracle(inp, gelu="erf"):
    y, tl, mem, ml, layers = inp.as_float64()
    sh = inp.workload.shape
    return DO.decoder_forward(y, tl, mem, ml, layers, sh.head_num, sh.size_per_head, gelu=gelu)


@pytest.mark.parametrize("nh,d,F,L,B,T,S", [
    (12, 64, 3072, 1, 3, 37, 45),      # BERT-Base structure, ragged target and memory
    (4, 32, 512, 2, 5, 70, 33),        # several query blocks; the memory shorter than the target
    (8, 128, 2048, 1, 2, 129, 200),    # size-128 heads, key blocks with ragged tails
    (16, 64, 4096, 1, 2, 64, 64),      # BERT-Large structure
], ids=str)
def test_decoder_matches_oracle(nh, d, F, L, B, T, S):
    sh = EI.EncoderShape(nh, d, F, L)
    wl = EI.DecoderWorkload("dec", sh, B, T, S, "fp16", 1, T, 1, S, ln_affine_random=True, seed=nh + T)
    inp = EI.make_decoder_inputs(wl)
    dec = _decoder(inp)
    got = _run(dec, inp)
    ref = _oracle(inp)
    m = valid_mask(inp.tgt_len, T)
    assert rel_l2(got, ref, m) < L * FP16_LAYER_REL_L2
    if L == 1:
        assert max_abs(got, ref, m) < FP16_LAYER_MAX_ABS
    assert dec.device_status() == 0


def test_decoder_fused_layernorm_gemms_at_size():
    """Enough target tokens (32 x 128) for the 2-CTA tiles: with both fusions
    asked for wherever supported, the three bias + residual + LayerNorm steps
    run in their GEMMs' epilogues (row statistics exchanged across the
    cluster), 9 launches per layer; sampled sequences against the oracle, and
    against the same decoder with both fusions off."""
    sh = EI.EncoderShape(12, 64, 3072, 1)
    B, T, S = 32, 128, 96
    wl = EI.DecoderWorkload("dec-fused", sh, B, T, S, "fp16", T // 2, T, S // 2, S, ln_affine_random=True, seed=7)
    inp = EI.make_decoder_inputs(wl)
    dec = _decoder(inp)
    dec.set_option("ln_fuse_out_proj", 2)
    dec.set_option("ln_fuse_ffn2", 2)
    n0 = dec.launch_count()
    got = _run(dec, inp)
    assert dec.launch_count() - n0 == 9
    pick = [0, 1, B - 1]
    sub = EI.make_decoder_inputs(wl)
    sub.y, sub.mem = inp.y[pick], inp.mem[pick]
    sub.tgt_len, sub.mem_len = inp.tgt_len[pick], inp.mem_len[pick]
    ref = _oracle(sub)
    m = valid_mask(sub.tgt_len, T)
    assert rel_l2(got[pick], ref, m) < FP16_LAYER_REL_L2
    assert max_abs(got[pick], ref, m) < FP16_LAYER_MAX_ABS
    dec.set_option("ln_fuse_out_proj", 0)
    dec.set_option("ln_fuse_ffn2", 0)
    n0 = dec.launch_count()
    unfused = _run(dec, inp)
    assert dec.launch_count() - n0 == 12
    mall = valid_mask(inp.tgt_len, T)
    assert rel_l2(got, unfused, mall) < FP16_LAYER_REL_L2
    assert dec.device_status() == 0


def test_decoder_empty_target_and_memory_and_tanh_gelu():
    sh = EI.EncoderShape(12, 64, 3072, 2)
    wl = EI.DecoderWorkload("dec-empty", sh, 4, 40, 50, "fp16", 1, 40, 1, 50, seed=3)
    inp = EI.make_decoder_inputs(wl)
    inp.tgt_len[1] = 0                    # no valid target key: self-attention context 0
    inp.mem_len[2] = 0                    # empty memory: cross-attention context 0
    dec = _decoder(inp)
    dec.set_gelu("tanh")
    got = _run(dec, inp)
    assert np.all(np.isfinite(got))
    ref = _oracle(inp, gelu="tanh")
    for b in (0, 2, 3):                   # sequence 1 has no valid rows
        m = np.arange(40) < inp.tgt_len[b]
        assert rel_l2(got[b][m], ref[b][m]) < 2 * FP16_LAYER_REL_L2
    # the empty target's rows are still defined: every row attends to no key
    ref1 = ref[1]
    assert rel_l2(got[1], ref1) < 2 * FP16_LAYER_REL_L2


def test_decoder_causality_on_the_gpu():
    """Changing target tokens after position i leaves rows <= i bit-identical
    (every step is row-wise except the causal attention, which never reads
    later keys)."""
    sh = EI.EncoderShape(12, 64, 3072, 2)
    wl = EI.DecoderWorkload("dec-causal", sh, 2, 96, 48, "fp16", 96, 96, 48, 48, seed=4)
    inp = EI.make_decoder_inputs(wl)
    dec = _decoder(inp)
    base = _run(dec, inp)
    for i in (0, 31, 64, 95):
        y2 = inp.y.copy()
        y2[:, i + 1:] = np.random.default_rng(i).normal(0, 2, y2[:, i + 1:].shape).astype(np.float16)
        import dataclasses
        got = _run(dec, dataclasses.replace(inp, y=y2))
        assert np.array_equal(got[:, :i + 1], base[:, :i + 1])


def test_decoder_and_encoder_handles_are_not_interchangeable():
    from transformer_encoder_bert_b200 import EncError
    sh = EI.EncoderShape(4, 32, 512, 1)
    inp = EI.make_decoder_inputs(EI.DecoderWorkload("dec-args", sh, 2, 8, 8, "fp16", 1, 8, 1, 8))
    dec = _decoder(inp)
    y = to_dev(inp.y)
    assert dec.lib.enc_forward(dec.handle, y.data_ptr(), to_dev(inp.tgt_len).data_ptr(), y.data_ptr(), 2, 8,
                               None) == 1
    with pytest.raises(EncError):
        dec.forward(y, to_dev(inp.tgt_len), to_dev(inp.mem), to_dev(inp.mem_len), out=y)   # out overlaps y
