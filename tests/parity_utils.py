"""Helpers shared by the GPU parity tests (comparison metrics and device transfer)."""
from __future__ import annotations

import math

import numpy as np

# Tolerances of the FP16 path against the float64 oracle, on valid tokens.
FP16_LAYER_REL_L2 = 5e-3
FP16_LAYER_MAX_ABS = 3e-2
FP16_STACK_REL_L2 = 2e-2
FP32_LAYER_REL_L2 = 1e-5


def to_dev(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_host(t) -> np.ndarray:
    return t.detach().cpu().numpy()


def empty_dev(shape, dtype: str):
    import torch
    return torch.empty(shape, dtype=torch.float16 if dtype == "fp16" else torch.float32, device="cuda")


def valid_mask(valid_len, seq):
    vl = np.clip(np.asarray(valid_len), 0, seq)
    return np.arange(seq)[None, :] < vl[:, None]


def rel_l2(got, ref, mask=None) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if mask is not None:
        got, ref = got[mask], ref[mask]
    den = math.sqrt(float(np.sum(ref * ref)))
    return math.sqrt(float(np.sum((got - ref) ** 2))) / max(den, 1e-300)


def max_abs(got, ref, mask=None) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if mask is not None:
        got, ref = got[mask], ref[mask]
    return float(np.max(np.abs(got - ref))) if got.size else 0.0


def encoder_from_inputs(inp, layers=None):
    from transformer_encoder_bert_b200 import Encoder
    wl = inp.workload
    sh = wl.shape
    return Encoder(sh.head_num, sh.size_per_head, sh.ffn_dim, inp.layers if layers is None else layers, wl.dtype)
