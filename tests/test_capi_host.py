"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
entry point that include/treeverify.h declares, and rejects bad arguments before
touching the device."""
import ctypes
import os
import re

import pytest

import __graft_entry__
import tree_speculative_decoding_04_b200 as tv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    __graft_entry__.build()
    return tv.load()


def _declared():
    txt = open(os.path.join(ROOT, "include", "treeverify.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", txt, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_header_declares_the_four_calls():
    d = _declared()
    for name in ("tree_build_mask", "tree_attention", "tree_accept", "kv_commit_realign"):
        assert name in d
    assert set(d) == set(tv.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert lib.tv_status_string(0) == b"TV_OK"
    assert lib.tv_status_string(1) == b"TV_ERR_INVALID_ARG"
    assert lib.tv_status_string(2) == b"TV_ERR_UNSUPPORTED"
    assert lib.tv_status_string(3) == b"TV_ERR_CUDA"
    assert lib.tv_version() >= 100


def test_argument_errors_are_synchronous(lib):
    P = ctypes.c_void_p
    z = P(0)
    dummy = P(256)  # never dereferenced: these calls must fail on the host first
    # negative sizes
    assert lib.tree_build_mask(dummy, -1, 4, 3, dummy, dummy, dummy, z) == 1
    # tree too large
    assert lib.tree_build_mask(dummy, 1, 256, 3, dummy, dummy, dummy, z) == 2
    # null outputs
    assert lib.tree_build_mask(dummy, 1, 4, 3, z, dummy, dummy, z) == 1
    # empty batch is a no-op
    assert lib.tree_build_mask(z, 0, 4, 3, z, z, z, z) == 0
    # attention: Hq not a multiple of Hkv, unsupported head dim, bad scale, misaligned q
    assert lib.tree_attention(dummy, dummy, dummy, 64, dummy, dummy, dummy, dummy, 1, 3, 6, 4, 128,
                              ctypes.c_float(0.1), dummy, z, 0, 0, z, ctypes.c_float(0), z, 0, z) == 1
    assert lib.tree_attention(dummy, dummy, dummy, 64, dummy, dummy, dummy, dummy, 1, 3, 8, 4, 96,
                              ctypes.c_float(0.1), dummy, z, 0, 0, z, ctypes.c_float(0), z, 0, z) == 2
    assert lib.tree_attention(dummy, dummy, dummy, 64, dummy, dummy, dummy, dummy, 1, 3, 8, 4, 128,
                              ctypes.c_float(0.0), dummy, z, 0, 0, z, ctypes.c_float(0), z, 0, z) == 1
    assert lib.tree_attention(P(258), dummy, dummy, 64, dummy, dummy, dummy, dummy, 1, 3, 8, 4, 128,
                              ctypes.c_float(0.1), dummy, z, 0, 0, z, ctypes.c_float(0), z, 0, z) == 1
    # an unknown launch flag; rotation without depths, without a base, or at head dim 64; a slot map of no slots
    assert lib.tree_attention(dummy, dummy, dummy, 64, dummy, dummy, dummy, dummy, 1, 3, 8, 4, 128,
                              ctypes.c_float(0.1), dummy, z, 0, 4, z, ctypes.c_float(0), z, 0, z) == 1
    assert lib.tree_attention(dummy, dummy, dummy, 64, dummy, dummy, dummy, dummy, 1, 3, 8, 4, 128,
                              ctypes.c_float(0.1), dummy, z, 0, 2, z, ctypes.c_float(1e4), z, 0, z) == 1
    assert lib.tree_attention(dummy, dummy, dummy, 64, dummy, dummy, dummy, dummy, 1, 3, 8, 4, 128,
                              ctypes.c_float(0.1), dummy, z, 0, 2, dummy, ctypes.c_float(0.5), z, 0, z) == 1
    assert lib.tree_attention(dummy, dummy, dummy, 64, dummy, dummy, dummy, dummy, 1, 3, 8, 4, 64,
                              ctypes.c_float(0.1), dummy, z, 0, 2, dummy, ctypes.c_float(1e4), z, 0, z) == 2
    assert lib.tree_attention(dummy, dummy, dummy, 64, dummy, dummy, dummy, dummy, 1, 3, 8, 4, 128,
                              ctypes.c_float(0.1), dummy, z, 0, 0, z, ctypes.c_float(0), dummy, 0, z) == 1
    # the workspace size is a pure function of the shape; D = 64 needs none
    assert lib.tree_attention_workspace_size(1, 64, 32, 32, 64, 2120) == 0
    assert lib.tree_attention_workspace_size(-1, 64, 32, 32, 128, 2120) == 0
    # accept: V < 1
    assert lib.tree_accept(dummy, dummy, dummy, dummy, dummy, dummy, 1, 3, 0, 3, dummy, dummy, dummy, dummy, z) == 1
    # commit: bad realign flag, unsupported D
    assert lib.kv_commit_realign(dummy, dummy, 1, 1, 1, 128, 64, 3, dummy, dummy, dummy, 3, dummy, dummy, dummy, 2,
                                 z, z, z, 0, z) == 1
    assert lib.kv_commit_realign(dummy, dummy, 1, 1, 1, 80, 64, 3, dummy, dummy, dummy, 3, dummy, dummy, dummy, 0,
                                 z, z, z, 0, z) == 2
    # commit: a slot map of no slots
    assert lib.kv_commit_realign(dummy, dummy, 1, 1, 1, 128, 64, 3, dummy, dummy, dummy, 3, dummy, dummy, dummy, 0,
                                 z, z, dummy, 0, z) == 1
    # tree-row append: negative size, unsupported D, tree too large, null rows, misaligned rows, empty
    assert lib.tree_kv_write(dummy, dummy, dummy, dummy, -1, 1, 1, 128, 64, 3, dummy, dummy, z,
                             ctypes.c_float(0), z, 0, z) == 1
    assert lib.tree_kv_write(dummy, dummy, dummy, dummy, 1, 1, 1, 96, 64, 3, dummy, dummy, z,
                             ctypes.c_float(0), z, 0, z) == 2
    assert lib.tree_kv_write(dummy, dummy, dummy, dummy, 1, 1, 1, 128, 512, 256, dummy, dummy, z,
                             ctypes.c_float(0), z, 0, z) == 2
    assert lib.tree_kv_write(dummy, dummy, z, dummy, 1, 1, 1, 128, 64, 3, dummy, dummy, z,
                             ctypes.c_float(0), z, 0, z) == 1
    assert lib.tree_kv_write(dummy, dummy, P(264), dummy, 1, 1, 1, 128, 64, 3, dummy, dummy, z,
                             ctypes.c_float(0), z, 0, z) == 1
    assert lib.tree_kv_write(z, z, z, z, 0, 1, 1, 128, 64, 3, z, z, z, ctypes.c_float(0), z, 0, z) == 0
    # tree-row append: rotation without a base
    assert lib.tree_kv_write(dummy, dummy, dummy, dummy, 1, 1, 1, 128, 64, 3, dummy, dummy, dummy, ctypes.c_float(0),
                             z, 0, z) == 1


def test_binding_refuses_host_tensors():
    import torch

    parent = torch.zeros((1, 4), dtype=torch.int32)
    with pytest.raises(tv.TVError):
        tv.tree_build_mask(parent, 3, torch.zeros((1, 4, 1), dtype=torch.int32),
                           torch.zeros((1, 4), dtype=torch.int32), torch.zeros((1,), dtype=torch.int32))


def test_status_bits_agree_between_header_binding_and_oracle():
    """The per-sequence status bits carry the same meaning in the header, the
    binding and the oracle (defined separately in each: no shared source)."""
    import oracle

    txt = open(os.path.join(ROOT, "include", "treeverify.h")).read()
    hdr = {m.group(1): int(m.group(2)) for m in re.finditer(r"#define TV_(SEQ_\w+|MAX_TREE_ROWS)\s+(\d+)", txt)}
    assert hdr == {"SEQ_BAD_PARENT": 1, "SEQ_TOO_DEEP": 2, "SEQ_TIMEOUT": 4, "SEQ_BAD_GEOMETRY": 8,
                   "MAX_TREE_ROWS": 256}
    for name, val in hdr.items():
        assert getattr(tv, name) == val
    assert (oracle.BAD_PARENT, oracle.TOO_DEEP, oracle.BAD_GEOMETRY) == (
        hdr["SEQ_BAD_PARENT"], hdr["SEQ_TOO_DEEP"], hdr["SEQ_BAD_GEOMETRY"])
