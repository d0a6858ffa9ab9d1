"""enc_forward_noalloc against enc_forward (GPU).

Some callers cannot allocate device memory when they run the encoder: a
server whose device memory is all handed out by its own pool allocator, or a
latency-bound loop that cannot afford cudaMalloc / cudaFree, which may
synchronise the whole device.  enc_forward_noalloc serves them: it keeps its
intermediates in a fixed device array compiled into the library instead of
memory it allocates.  It must give what enc_forward gives.

This file is collected last, so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest

import encoder_inputs as EI
from parity_utils import FP16_STACK_REL_L2, encoder_from_inputs, rel_l2, to_dev, to_host, valid_mask

pytestmark = pytest.mark.gpu

STATIC_WORKSPACE_BYTES = 32 << 20      # ENC_STATIC_WORKSPACE_BYTES in include/enc.h


def test_noalloc_forward_matches_enc_forward_on_two_calls_in_a_row():
    """Two calls in a row with different inputs on a fresh handle (one that never
    grew a workspace of its own), each against enc_forward of another handle
    with the same weights, within the 12-layer FP16 bound.  The second call
    leaves the device's free memory unchanged."""
    import torch
    wl = EI.named_workload("bert-base-s32", 32)          # 1024 tokens, 18.9 MB of scratch
    first = EI.make_inputs(wl)
    second = EI.make_inputs(wl.with_(seed=1))
    ref_enc = encoder_from_inputs(first)
    enc = encoder_from_inputs(first)
    assert enc.workspace_bytes(wl.batch, wl.seq) <= STATIC_WORKSPACE_BYTES
    runs = [(to_dev(i.x), to_dev(i.valid_len), i.valid_len) for i in (first, second)]
    refs = [to_host(ref_enc.forward(x, vl)) for x, vl, _ in runs]
    outs = [torch.full_like(runs[0][0], float("nan")) for _ in runs]
    torch.cuda.synchronize()

    enc.forward_noalloc(runs[0][0], runs[0][1], outs[0])
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    enc.forward_noalloc(runs[1][0], runs[1][1], outs[1])
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before

    for (_, _, vl), ref, out in zip(runs, refs, outs):
        got = to_host(out)
        m = valid_mask(vl, wl.seq)
        assert np.all(np.isfinite(got[m]))
        assert rel_l2(got, ref, m) < FP16_STACK_REL_L2
    assert enc.device_status() == 0


def test_noalloc_forward_rejects_batches_beyond_the_static_workspace():
    """A batch whose scratch exceeds the fixed array is refused before anything
    is enqueued (ENC_ERR_UNSUPPORTED, with the sizes in the message); a batch
    that fits still runs afterwards."""
    import torch
    from transformer_encoder_bert_b200 import EncError
    wl = EI.named_workload("bert-base-s32", 64).with_(shape=EI.EncoderShape(12, 64, 3072, 2))
    inp = EI.make_inputs(wl)
    enc = encoder_from_inputs(inp)
    assert enc.workspace_bytes(64, 32) > STATIC_WORKSPACE_BYTES
    x, vl = to_dev(inp.x), to_dev(inp.valid_len)
    out = torch.zeros_like(x)
    with pytest.raises(EncError) as e:
        enc.forward_noalloc(x, vl, out)
    assert e.value.status == 2
    assert "static workspace" in str(e.value)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0        # nothing ran
    small = EI.make_inputs(wl.with_(batch=8, seed=3))
    got = enc.forward_noalloc(to_dev(small.x), to_dev(small.valid_len), torch.empty_like(to_dev(small.x)))
    ref = enc.forward(to_dev(small.x), to_dev(small.valid_len))
    m = valid_mask(small.valid_len, wl.seq)
    assert rel_l2(to_host(got), to_host(ref), m) < FP16_STACK_REL_L2
    assert enc.device_status() == 0
