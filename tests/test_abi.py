"""The C-ABI library loads on a machine without a GPU and exports every symbol
include/enc.h declares; host-side argument checks fail before any CUDA work."""
import ctypes

import pytest

from transformer_encoder_bert_b200 import binding as B


def test_header_declares_the_boundary():
    names = B.declared_symbols()
    for required in ("enc_create", "enc_forward", "enc_destroy", "enc_last_error"):
        assert required in names
    assert len(names) >= 14


def test_library_exports_every_declared_symbol():
    lib = B.load_library()
    for name in B.declared_symbols():
        assert hasattr(lib, name), f"{name} is declared in include/enc.h but not exported"


def test_binding_covers_every_declared_symbol():
    assert sorted(B.SIGNATURES) == B.declared_symbols()


def test_layer_weight_struct_matches_header_order():
    import os, re
    text = open(os.path.join(os.path.dirname(B.__file__), "..", "include", "enc.h")).read()
    body = text[text.index("typedef struct {"):text.index("} enc_layer_weights;")]
    fields = re.findall(r"const void\*\s*(\w+);", body)
    assert tuple(fields) == B.WEIGHT_FIELDS
    assert ctypes.sizeof(B.EncLayerWeights) == 12 * ctypes.sizeof(ctypes.c_void_p)


def _create(nh, d, F, L, dtype=1, weights=None):
    lib = B.load_library()
    h = ctypes.c_void_p(123)
    st = lib.enc_create(nh, d, F, L, dtype, weights, ctypes.byref(h))
    return st, h, lib.enc_last_error().decode()


@pytest.mark.parametrize("args,status", [
    ((0, 64, 3072, 12), 1),          # head_num must be > 0
    ((12, 48, 3072, 12), 2),         # size_per_head not in {32, 64, 128}
    ((12, 64, 3071, 12), 1),         # ffn_dim not a multiple of 8
    ((12, 64, 3072, 0), 1),          # num_layers must be > 0
    ((12, 64, 3072, 12), 1),         # weights is NULL
])
def test_create_rejects_bad_arguments_without_a_gpu(args, status):
    st, h, msg = _create(*args)
    assert st == status
    assert h.value is None           # *out is cleared on error
    assert msg


def test_null_handle_paths():
    lib = B.load_library()
    assert lib.enc_destroy(None) == 0
    assert lib.enc_workspace_bytes(None, 1, 1) == 0
    assert lib.enc_forward(None, None, None, None, 1, 1, None) == 1
    assert b"null handle" in lib.enc_last_error()
