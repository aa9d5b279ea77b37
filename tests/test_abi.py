"""The C ABI loads, exports every declared symbol and rejects bad arguments
before touching the GPU (runs without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dspark.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dspark_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from speculative_decoding_semi_b200 import binding
    return binding.lib


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"dspark_markov_draft", "dspark_schedule", "dspark_verify"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for s in range(6):
        assert lib.dspark_status_string(s)


def test_workspace_bytes_limits(lib):
    assert lib.dspark_workspace_bytes(64, 8, 151936, 256) > 0
    assert lib.dspark_workspace_bytes(0, 8, 151936, 256) == 0
    assert lib.dspark_workspace_bytes(64, 0, 151936, 256) == 0
    assert lib.dspark_workspace_bytes(64, 33, 151936, 256) == 0
    assert lib.dspark_workspace_bytes(64, 8, 151937, 256) == 0      # V % 8 != 0
    assert lib.dspark_workspace_bytes(64, 8, 151936, 513) == 0


def test_invalid_arguments_rejected_before_launch(lib):
    P = ctypes.c_void_p
    nul = None
    fake = P(4096)  # never dereferenced: validation fails first
    # NULL pointers
    st = lib.dspark_markov_draft(nul, fake, fake, 1, 256, fake, fake, 4, 4, 1024, fake, fake, fake, fake,
                                 fake, 1 << 30, None)
    assert st == 1
    # misaligned pointer
    st = lib.dspark_verify(P(4097), fake, fake, fake, fake, fake, fake, fake, fake, 4, 4, 1024,
                           fake, fake, fake, fake, 1 << 30, None)
    assert st == 1
    # bad dtype
    st = lib.dspark_markov_draft(fake, fake, fake, 7, 32, fake, fake, 4, 4, 1024, fake, fake, fake, fake,
                                 fake, 1 << 30, None)
    assert st == 1
    # workspace too small
    st = lib.dspark_markov_draft(fake, fake, fake, 0, 32, fake, fake, 4, 4, 1024, fake, fake, fake, fake,
                                 fake, 16, None)
    assert st == 1
    # profile shorter than the batch; too many schedule items
    st = lib.dspark_schedule(fake, fake, fake, 3, 4, 4, fake, fake, fake, fake, fake, 1 << 30, None)
    assert st == 1
    st = lib.dspark_schedule(fake, fake, fake, 1 << 20, 2048, 16, fake, fake, fake, fake, fake, 1 << 30, None)
    assert st == 1
    st = lib.dspark_workspace_init(nul, 1 << 20, None)
    assert st == 1


def test_variant_b_shapes_rejected_before_launch(lib):
    """Variant B runs on the tensor-core kernels only: other shapes return
    DSPARK_ERR_UNSUPPORTED (2) before anything touches the GPU."""
    P = ctypes.c_void_p
    fake = P(4096)
    ws = 1 << 40
    # fp32 factors; r = 32; V % 32 != 0; B > 512
    for dt, r, B, V in ((0, 64, 4, 1024), (1, 32, 4, 1024), (1, 64, 4, 1000), (1, 64, 513, 1024)):
        st = lib.dspark_markov_draft_b(fake, fake, fake, dt, r, fake, fake, B, 4, V, fake, fake, fake, fake,
                                       fake, ws, None)
        assert st == 2, (dt, r, B, V)
        st = lib.dspark_rnn_draft_b(fake, fake, fake, fake, dt, r, fake, fake, B, 4, V, fake, fake, fake, fake,
                                    fake, ws, None)
        assert st == 2, (dt, r, B, V)
    for r, B, V in ((32, 4, 1024), (64, 4, 1000), (64, 513, 1024)):
        st = lib.dspark_verify_b(fake, fake, fake, fake, fake, r, fake, fake, fake, fake, fake, fake, B, 4, V,
                                 fake, fake, fake, fake, ws, None)
        assert st == 2, (r, B, V)
    # NULL operand rows / base are invalid arguments
    st = lib.dspark_markov_draft_b(fake, fake, fake, 1, 64, fake, fake, 4, 4, 1024, fake, fake, fake, None,
                                   fake, ws, None)
    assert st == 1
    st = lib.dspark_verify_b(fake, fake, None, fake, fake, 64, fake, fake, fake, fake, fake, fake, 4, 4, 1024,
                             fake, fake, fake, fake, ws, None)
    assert st == 1
    # variant A entry points still need z
    st = lib.dspark_markov_draft(fake, fake, fake, 1, 64, fake, fake, 4, 4, 1024, fake, fake, fake, None,
                                 fake, ws, None)
    assert st == 1


def test_probe_library_rejects_bad_arguments():
    """The benchmark's L2 read probe (its own shared object, outside the
    library's path) loads without a GPU and rejects bad arguments before any
    launch."""
    path = os.path.join(ROOT, "speculative_decoding_semi_b200", "libdspark_probe.so")
    probe = ctypes.CDLL(path)
    probe.dspark_probe_l2_read.restype = ctypes.c_int
    probe.dspark_probe_l2_read.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p,
                                           ctypes.c_size_t, ctypes.c_void_p]
    probe.dspark_probe_sink_words.restype = ctypes.c_size_t
    assert probe.dspark_probe_l2_read(None, 1 << 20, 4, None, 1 << 20, None) == 1
    assert probe.dspark_probe_l2_read(ctypes.c_void_p(16), 1 << 20, 4, None, 1 << 20, None) == 1
    assert probe.dspark_probe_l2_read(ctypes.c_void_p(17), 1 << 20, 4, ctypes.c_void_p(64), 1 << 20, None) == 1
    assert probe.dspark_probe_l2_read(ctypes.c_void_p(16), 24, 4, ctypes.c_void_p(64), 1 << 20, None) == 1
    assert probe.dspark_probe_l2_read(ctypes.c_void_p(16), 1 << 20, 0, ctypes.c_void_p(64), 1 << 20, None) == 1
