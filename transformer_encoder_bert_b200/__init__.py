"""B200 (sm_100a) forward pass of a BERT-style post-LayerNorm Transformer encoder.

The product is the C-ABI library lib/libbertenc.so (include/enc.h); this
package builds it (``build``) and binds it (``Encoder``).
"""
from .binding import Decoder, Encoder, EncError, load_library, LIB_PATH  # noqa: F401

__all__ = ["Decoder", "Encoder", "EncError", "load_library", "LIB_PATH"]
