"""ctypes binding of the encoder's C ABI (include/enc.h).

Argument marshalling only: every step of the forward pass runs in the CUDA
library.  PyTorch supplies device memory and the current stream.  Loading
fails loudly when the library has not been built; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence

import numpy as np

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libbertenc.so")

ENC_OK = 0
STATUS_NAMES = {0: "ENC_OK", 1: "ENC_ERR_INVALID_ARG", 2: "ENC_ERR_UNSUPPORTED", 3: "ENC_ERR_OOM",
                4: "ENC_ERR_CUDA", 5: "ENC_ERR_DEVICE"}
DTYPE_CODES = {"fp32": 0, "fp16": 1}
NP_DTYPES = {"fp32": np.float32, "fp16": np.float16}

# enc_option codes (kernel-path switches; every choice computes the same result to rounding).
OPTION_CODES = {"pair_tiles": 0, "tma_store": 1, "tc_attention": 2, "split_k": 3, "ln_fuse_ffn2": 4,
                "ln_fuse_out_proj": 5, "pdl": 6, "persistent": 7, "test_stall": 8}

# Field order of enc_layer_weights.
WEIGHT_FIELDS = ("w_qkv", "b_qkv", "w_o", "b_o", "ln1_g", "ln1_b",
                 "w_ff1", "b_ff1", "w_ff2", "b_ff2", "ln2_g", "ln2_b")

# Every symbol include/enc.h declares, with (restype, argtypes).
_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "enc_create": (_i, [_i, _i, _i, _i, _i, _vp, ctypes.POINTER(_vp)]),
    "enc_forward": (_i, [_vp, _vp, _vp, _vp, _i, _i, _vp]),
    "enc_forward_noalloc": (_i, [_vp, _vp, _vp, _vp, _i, _i, _vp]),
    "enc_forward_host": (_i, [_vp, _vp, _vp, _vp, _i, _i, _vp]),
    "enc_forward_host_async": (_i, [_vp, _vp, _vp, _vp, _i, _i, _vp]),
    "enc_host_join": (_i, [_vp, _vp]),
    "enc_reserve": (_i, [_vp, _i, _i]),
    "enc_workspace_bytes": (_sz, [_vp, _i, _i]),
    "enc_destroy": (_i, [_vp]),
    "enc_last_error": (ctypes.c_char_p, []),
    "enc_device_status": (_i, [_vp, ctypes.POINTER(ctypes.c_int32)]),
    "enc_set_gelu": (_i, [_vp, _i]),
    "enc_set_packing": (_i, [_vp, _i]),
    "enc_set_host_chunks": (_i, [_vp, _i]),
    "enc_set_option": (_i, [_vp, _i, _i]),
    "enc_get_option": (_i, [_vp, _i, ctypes.POINTER(_i)]),
    "enc_graph_create": (_i, [_vp, _vp, _vp, _vp, _i, _i, ctypes.POINTER(_vp)]),
    "enc_graph_launch": (_i, [_vp, _vp]),
    "enc_graph_destroy": (_i, [_vp]),
    "enc_kernels_per_forward": (_i, [_vp, _i, _i]),
    "enc_launch_count": (ctypes.c_uint64, [_vp]),
    "enc_set_trace_events": (_i, [_vp, _vp, _i]),
    "enc_decoder_create": (_i, [_i, _i, _i, _i, _i, _vp, ctypes.POINTER(_vp)]),
    "enc_decoder_forward": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp]),
    "enc_op_qkv": (_i, [_vp, _i, _vp, _vp, _i, _i, _vp]),
    "enc_op_attention": (_i, [_vp, _vp, _vp, _vp, _i, _i, _vp]),
    "enc_op_out_proj_ln": (_i, [_vp, _i, _vp, _vp, _vp, _i, _vp]),
    "enc_op_ffn1": (_i, [_vp, _i, _vp, _vp, _i, _vp]),
    "enc_op_ffn2_ln": (_i, [_vp, _i, _vp, _vp, _vp, _i, _vp]),
}


class EncLayerWeights(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in WEIGHT_FIELDS]


# Field order of enc_decoder_layer_weights.
DECODER_WEIGHT_FIELDS = ("w_qkv", "b_qkv", "w_o", "b_o", "ln1_g", "ln1_b", "w_q2", "b_q2", "w_kv2", "b_kv2",
                         "w_o2", "b_o2", "ln2_g", "ln2_b", "w_ff1", "b_ff1", "w_ff2", "b_ff2", "ln3_g", "ln3_b")


class EncDecoderLayerWeights(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in DECODER_WEIGHT_FIELDS]


class EncError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libbertenc.so (built in-tree by transformer_encoder_bert_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is missing; build it with "
                           "`python -m transformer_encoder_bert_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int):
    if status != ENC_OK:
        raise EncError(status, load_library().enc_last_error().decode())


def _current_stream(stream=None) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return getattr(stream, "cuda_stream", stream)


def _dptr(t, dtype_np=None) -> int:
    """Device pointer of a CUDA torch tensor (checked: on GPU, contiguous)."""
    if not (hasattr(t, "is_cuda") and t.is_cuda):
        raise TypeError("expected a CUDA torch tensor")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


class Encoder:
    """A BERT-style post-LN encoder stack behind the C ABI.

    layers: per-layer dicts with the keys of WEIGHT_FIELDS holding numpy arrays
    (host) or CUDA torch tensors, in the storage dtype, [in, out] row-major.
    """

    def __init__(self, head_num: int, size_per_head: int, ffn_dim: int,
                 layers: Sequence[Dict], dtype: str = "fp16"):
        self.lib = load_library()
        self.head_num, self.size_per_head, self.ffn_dim = head_num, size_per_head, ffn_dim
        self.hidden = head_num * size_per_head
        self.num_layers = len(layers)
        self.dtype = dtype
        self.np_dtype = NP_DTYPES[dtype]
        arr = (EncLayerWeights * max(1, len(layers)))()
        keep = []
        for i, lw in enumerate(layers):
            for name in WEIGHT_FIELDS:
                v = lw[name]
                if isinstance(v, np.ndarray):
                    v = np.ascontiguousarray(v, dtype=self.np_dtype)
                    keep.append(v)
                    setattr(arr[i], name, v.ctypes.data)
                else:
                    keep.append(v)
                    setattr(arr[i], name, _dptr(v))
        h = ctypes.c_void_p()
        _check(self.lib.enc_create(head_num, size_per_head, ffn_dim, len(layers), DTYPE_CODES[dtype],
                                   ctypes.cast(arr, ctypes.c_void_p), ctypes.byref(h)))
        self.handle = h

    # -------------------------------------------------------------- lifetime
    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            _check(self.lib.enc_destroy(self.handle))
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # -------------------------------------------------------------- whole stack
    def set_gelu(self, form: str):
        """"erf" (default) or "tanh"."""
        _check(self.lib.enc_set_gelu(self.handle, {"erf": 0, "tanh": 1}[form]))

    def set_packing(self, enable: bool):
        """Padding removal: compute valid tokens only; padded output rows become zeros."""
        _check(self.lib.enc_set_packing(self.handle, 1 if enable else 0))

    def set_option(self, name: str, value):
        """One kernel-path switch (see OPTION_CODES and enc_option in include/enc.h):
        a bool, or 0/1/2 for the two LayerNorm fusions."""
        _check(self.lib.enc_set_option(self.handle, OPTION_CODES[name], int(value)))

    def get_option(self, name: str) -> int:
        v = ctypes.c_int(0)
        _check(self.lib.enc_get_option(self.handle, OPTION_CODES[name], ctypes.byref(v)))
        return int(v.value)

    def set_host_chunks(self, chunks: int):
        _check(self.lib.enc_set_host_chunks(self.handle, chunks))

    def reserve(self, batch: int, seq: int):
        _check(self.lib.enc_reserve(self.handle, batch, seq))

    def workspace_bytes(self, batch: int, seq: int) -> int:
        return int(self.lib.enc_workspace_bytes(self.handle, batch, seq))

    def forward(self, x, valid_len, out=None, stream=None):
        """x: CUDA [B, S, H] tensor in the storage dtype; valid_len: CUDA int32 [B]."""
        import torch
        B, S, H = x.shape
        if out is None:
            out = torch.empty_like(x)
        _check(self.lib.enc_forward(self.handle, _dptr(x), _dptr(valid_len), _dptr(out), B, S,
                                    _current_stream(stream)))
        return out

    def forward_noalloc(self, x, valid_len, out, stream=None):
        """enc_forward_noalloc: the forward with its scratch in the library's fixed
        device array (no device allocation); out must be given."""
        B, S, H = x.shape
        _check(self.lib.enc_forward_noalloc(self.handle, _dptr(x), _dptr(valid_len), _dptr(out), B, S,
                                            _current_stream(stream)))
        return out

    def forward_host(self, x: np.ndarray, valid_len: np.ndarray, out: Optional[np.ndarray] = None,
                     stream=None) -> np.ndarray:
        """Host arrays in, host array out (copies and the stack run on the stream; synchronous)."""
        x = np.ascontiguousarray(x, dtype=self.np_dtype)
        vl = np.ascontiguousarray(valid_len, dtype=np.int32)
        if out is None:
            out = np.empty_like(x)
        B, S, _ = x.shape
        _check(self.lib.enc_forward_host(self.handle, x.ctypes.data, vl.ctypes.data, out.ctypes.data,
                                         B, S, _current_stream(stream)))
        return out

    def forward_host_ptr(self, x_ptr: int, vl_ptr: int, out_ptr: int, batch: int, seq: int, stream=None):
        """enc_forward_host on raw host pointers (e.g. pinned torch tensors)."""
        _check(self.lib.enc_forward_host(self.handle, x_ptr, vl_ptr, out_ptr, batch, seq,
                                         _current_stream(stream)))

    def forward_host_async_ptr(self, x_ptr: int, vl_ptr: int, out_ptr: int, batch: int, seq: int, stream=None):
        """enc_forward_host_async on raw (pinned) host pointers; see host_join."""
        _check(self.lib.enc_forward_host_async(self.handle, x_ptr, vl_ptr, out_ptr, batch, seq,
                                               _current_stream(stream)))

    def host_join(self, stream=None):
        """Make the stream wait for every copy of earlier forward_host_async calls."""
        _check(self.lib.enc_host_join(self.handle, _current_stream(stream)))

    def record(self, x, valid_len, out) -> "RecordedForward":
        """Record one forward on these CUDA tensors as a CUDA graph (see enc_graph_create)."""
        B, S, _ = x.shape
        g = ctypes.c_void_p()
        _check(self.lib.enc_graph_create(self.handle, _dptr(x), _dptr(valid_len), _dptr(out), B, S,
                                         ctypes.byref(g)))
        return RecordedForward(self, g, (x, valid_len, out))

    def kernels_per_forward(self, batch: int, seq: int) -> int:
        return int(self.lib.enc_kernels_per_forward(self.handle, batch, seq))

    def launch_count(self) -> int:
        return int(self.lib.enc_launch_count(self.handle))

    def set_trace_events(self, events, prepare: bool = True):
        """events: list of torch.cuda.Event(enable_timing=True), or None to switch tracing off.

        torch creates an event's CUDA object on its first record(); with prepare=True
        every event is recorded once (and the device synchronised) first.  Pass
        prepare=False for events that have been recorded before, to arm tracing
        without any host synchronisation."""
        if not events:
            _check(self.lib.enc_set_trace_events(self.handle, None, 0))
            self._trace_keep = None
            return
        if prepare:
            import torch
            for e in events:
                e.record()
            torch.cuda.synchronize()
        arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        self._trace_keep = (arr, list(events))
        _check(self.lib.enc_set_trace_events(self.handle, ctypes.cast(arr, ctypes.c_void_p), len(events)))

    def device_status(self) -> int:
        code = ctypes.c_int32(0)
        st = self.lib.enc_device_status(self.handle, ctypes.byref(code))
        if st not in (ENC_OK, 5):
            _check(st)
        return int(code.value)

    # -------------------------------------------------------------- single steps
    def op_qkv(self, layer: int, x, qkv, batch: int, seq: int, stream=None):
        _check(self.lib.enc_op_qkv(self.handle, layer, _dptr(x), _dptr(qkv), batch, seq, _current_stream(stream)))

    def op_attention(self, qkv, valid_len, ctx, batch: int, seq: int, stream=None):
        _check(self.lib.enc_op_attention(self.handle, _dptr(qkv), _dptr(valid_len), _dptr(ctx), batch, seq,
                                         _current_stream(stream)))

    def op_out_proj_ln(self, layer: int, ctx, resid, out, tokens: int, stream=None):
        """out = LN1(ctx Wo + bo + resid)."""
        _check(self.lib.enc_op_out_proj_ln(self.handle, layer, _dptr(ctx), _dptr(resid), _dptr(out), tokens,
                                           _current_stream(stream)))

    def op_ffn1(self, layer: int, h1, u, tokens: int, stream=None):
        _check(self.lib.enc_op_ffn1(self.handle, layer, _dptr(h1), _dptr(u), tokens, _current_stream(stream)))

    def op_ffn2_ln(self, layer: int, u, resid, out, tokens: int, stream=None):
        """out = LN2(u W2 + b2 + resid)."""
        _check(self.lib.enc_op_ffn2_ln(self.handle, layer, _dptr(u), _dptr(resid), _dptr(out), tokens,
                                       _current_stream(stream)))


class Decoder:
    """The decoder stack behind the C ABI (enc_decoder_create / enc_decoder_forward).

    layers: per-layer dicts with the keys of DECODER_WEIGHT_FIELDS (numpy FP16
    arrays, [in, out] row-major)."""

    def __init__(self, head_num: int, size_per_head: int, ffn_dim: int, layers: Sequence[Dict]):
        self.lib = load_library()
        self.hidden = head_num * size_per_head
        arr = (EncDecoderLayerWeights * max(1, len(layers)))()
        keep = []
        for i, lw in enumerate(layers):
            for name in DECODER_WEIGHT_FIELDS:
                v = np.ascontiguousarray(lw[name], dtype=np.float16)
                keep.append(v)
                setattr(arr[i], name, v.ctypes.data)
        h = ctypes.c_void_p()
        _check(self.lib.enc_decoder_create(head_num, size_per_head, ffn_dim, len(layers), DTYPE_CODES["fp16"],
                                           ctypes.cast(arr, ctypes.c_void_p), ctypes.byref(h)))
        self.handle = h

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            _check(self.lib.enc_destroy(self.handle))
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_gelu(self, form: str):
        _check(self.lib.enc_set_gelu(self.handle, {"erf": 0, "tanh": 1}[form]))

    def set_option(self, name: str, value):
        """One kernel-path switch (OPTION_CODES, enc_option in include/enc.h)."""
        _check(self.lib.enc_set_option(self.handle, OPTION_CODES[name], int(value)))

    def launch_count(self) -> int:
        return int(self.lib.enc_launch_count(self.handle))

    def forward(self, y, tgt_len, mem, mem_len, out=None, stream=None):
        """y: CUDA [B, T, H] FP16; mem: CUDA [B, S, H] FP16; lengths: CUDA int32 [B]."""
        import torch
        B, T, _ = y.shape
        S = mem.shape[1]
        if out is None:
            out = torch.empty_like(y)
        _check(self.lib.enc_decoder_forward(self.handle, _dptr(y), _dptr(tgt_len), _dptr(mem), _dptr(mem_len),
                                            _dptr(out), B, T, S, _current_stream(stream)))
        return out

    def device_status(self) -> int:
        code = ctypes.c_int32(0)
        st = self.lib.enc_device_status(self.handle, ctypes.byref(code))
        if st not in (ENC_OK, 5):
            _check(st)
        return int(code.value)


class RecordedForward:
    """A forward recorded by Encoder.record; launch() replays it on a stream."""

    def __init__(self, enc: Encoder, g: ctypes.c_void_p, keep):
        self.enc, self.g, self._keep = enc, g, keep

    def launch(self, stream=None):
        _check(self.enc.lib.enc_graph_launch(self.g, _current_stream(stream)))

    def close(self):
        if self.g is not None and self.g.value:
            _check(self.enc.lib.enc_graph_destroy(self.g))
        self.g = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def declared_symbols(header: Optional[str] = None) -> List[str]:
    """Names of the functions include/enc.h declares (parsed from the header text)."""
    import re
    if header is None:
        header = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "enc.h")
    with open(header) as f:
        text = f.read()
    return sorted(set(re.findall(r"ENC_API\s+[\w\s\*]+?\b(enc_\w+)\s*\(", text)))
