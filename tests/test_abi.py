"""CPU checks of the C ABI: the library builds, loads and exports every symbol the
header declares; host-side logic (keep count, workspace size, argument validation)
behaves as documented.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

from video_dit_dynamic_b200 import build as sbuild
from video_dit_dynamic_b200 import sbsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sbsa.h")


@pytest.fixture(scope="module")
def lib():
    sbuild.build()
    return sbsa.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sbsa_[a-z0-9_]+)\s*\(", text)))


def test_header_declarations_match_binding_list():
    assert declared_functions() == sorted(sbsa.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in sbsa.STATUS_NAMES.items():
        assert sbsa.sbsa_status_string(code) == name
    assert sbsa.sbsa_status_string(99) == "SBSA_ERR_UNKNOWN"
    assert sbsa.sbsa_version() >= 100


def test_keep_blocks_rounding(lib):
    assert [sbsa.sbsa_keep_blocks(256, f) for f in (1.0, 0.5, 0.3, 0.2, 0.1)] == [256, 128, 77, 51, 26]
    assert sbsa.sbsa_keep_blocks(960, 0.10) == 96
    assert sbsa.sbsa_keep_blocks(591, 0.15) == 89
    assert sbsa.sbsa_keep_blocks(16, 0.25) == 4
    assert sbsa.sbsa_keep_blocks(10, 0.0) == 1
    assert sbsa.sbsa_keep_blocks(10, 5.0) == 10
    assert sbsa.sbsa_keep_blocks(0, 0.5) == 0
    assert sbsa.sbsa_keep_blocks(10, float("nan")) == 0


def test_workspace_bytes(lib):
    s = sbsa.make_shape(1, 40, 122880, 128, 128)
    k = 96
    rows = 40 * 960
    means = rows * 128 * 4
    want = means + means + ((rows + 1) * 4 + 255) // 256 * 256 + rows * k * 4
    assert sbsa.sbsa_workspace_bytes(s, k) == want
    assert sbsa.sbsa_workspace_bytes(s, 0) == 0
    assert sbsa.sbsa_workspace_bytes(s, 961) == 0
    bad = sbsa.make_shape(1, 1, 100, 96, 64)
    assert sbsa.sbsa_workspace_bytes(bad, 1) == 0


def _status(lib, fn, *args):
    return getattr(lib, fn)(*args)


def test_argument_errors_return_before_launch(lib):
    P = ctypes.c_void_p
    good = sbsa.make_shape(1, 2, 1000, 64, 64)
    fake = P(0x10000)  # never dereferenced: validation fails first or the call is not made
    # null pointers
    assert lib.sbsa_pool_qk(ctypes.byref(good), None, fake, fake, fake, None) == 1
    # misaligned pointer
    assert lib.sbsa_pool_qk(ctypes.byref(good), P(0x10008), fake, fake, fake, None) == 1
    assert b"aligned" in lib.sbsa_last_error_message()
    # unsupported head_dim / block size
    assert lib.sbsa_pool_qk(ctypes.byref(sbsa.make_shape(1, 2, 1000, 96, 64)), fake, fake, fake, fake, None) == 2
    assert lib.sbsa_pool_qk(ctypes.byref(sbsa.make_shape(1, 2, 1000, 64, 32)), fake, fake, fake, fake, None) == 2
    # Lp not the rounded-up L
    s = sbsa.Shape(1, 2, 1000, 1088, 64, 64)
    assert lib.sbsa_pool_qk(ctypes.byref(s), fake, fake, fake, fake, None) == 1
    # too many blocks
    s = sbsa.make_shape(1, 1, 64 * 2049, 64, 64)
    assert lib.sbsa_pool_qk(ctypes.byref(s), fake, fake, fake, fake, None) == 2
    # k out of range
    assert lib.sbsa_select_blocks(ctypes.byref(good), fake, fake, 0, fake, fake, None) == 1
    assert lib.sbsa_select_blocks(ctypes.byref(good), fake, fake, 17, fake, fake, None) == 1
    # non-finite scale
    assert lib.sbsa_attention_fwd(ctypes.byref(good), fake, fake, fake, fake, fake, ctypes.c_float(float("inf")),
                                  fake, None) == 1
    # workspace missing, misaligned or too small
    assert lib.sbsa_forward(ctypes.byref(good), fake, fake, fake, 4, ctypes.c_float(0), fake, None, None, 0,
                            None) == 3
    assert lib.sbsa_forward(ctypes.byref(good), fake, fake, fake, 4, ctypes.c_float(0), fake, None, P(0x10010),
                            1 << 30, None) == 3
    assert lib.sbsa_forward(ctypes.byref(good), fake, fake, fake, 4, ctypes.c_float(0), fake, None, P(0x10000),
                            16, None) == 3
    assert b"smaller" in lib.sbsa_last_error_message()
    # null shape
    assert lib.sbsa_pool_qk(None, fake, fake, fake, fake, None) == 1
    # the host entry point: null host or device pointers, a negative chunk, a short workspace
    f0 = ctypes.c_float(0)
    assert lib.sbsa_forward_host(ctypes.byref(good), None, fake, fake, 4, f0, fake, fake, fake, fake, fake, fake,
                                 1 << 30, 0, None, None, None) == 1
    assert lib.sbsa_forward_host(ctypes.byref(good), fake, fake, fake, 4, f0, fake, fake, None, fake, fake, fake,
                                 1 << 30, 0, None, None, None) == 1
    assert lib.sbsa_forward_host(ctypes.byref(good), fake, fake, fake, 4, f0, fake, fake, fake, fake, fake, fake,
                                 1 << 30, -1, None, None, None) == 1
    assert lib.sbsa_forward_host(ctypes.byref(good), fake, fake, fake, 4, f0, fake, fake, fake, fake, fake, fake,
                                 16, 0, None, None, None) == 3


def test_binding_rejects_cpu_tensors(lib):
    import torch
    s = sbsa.make_shape(1, 1, 128, 64, 64)
    x = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    m = torch.zeros(1, 1, 2, 64)
    with pytest.raises(TypeError):
        sbsa.sbsa_pool_qk(s, x, x, m, m, stream=0)


def test_rope_table_size_and_argument_errors():
    from video_dit_dynamic_b200 import sbsa
    # d = 128: 22 frame, 21 row, 21 column pairs; (cos, sin) per grid position and pair
    assert sbsa.sbsa_rope_table_floats(128, (24, 64, 80)) == 2 * (24 * 22 + 64 * 21 + 80 * 21)
    assert sbsa.sbsa_rope_table_floats(64, (2, 3, 4)) == 2 * (2 * 12 + 3 * 10 + 4 * 10)
    assert sbsa.sbsa_rope_table_floats(96, (2, 3, 4)) == 0
    assert sbsa.sbsa_rope_table_floats(128, (0, 3, 4)) == 0
    lib = sbsa.load()
    s = sbsa.make_shape(1, 2, 120, 128, 64)
    # grid does not cover seq_len: rejected before any pointer is looked at
    st = lib.sbsa_rope_pool_qk(ctypes.byref(s), 2, 3, 4, None, None, None, None, None, None, None, None)
    assert st == 1 and b"grid" in lib.sbsa_last_error_message()
    st = lib.sbsa_rope_pool_qk(ctypes.byref(s), 2, 6, 10, None, None, None, None, None, None, None, None)
    assert st == 1 and b"null" in lib.sbsa_last_error_message()
    assert lib.sbsa_rope_table_init(128, 2, 6, 10, 1.0, None, None) == 1   # theta must exceed 1


def test_nvfp4_sizes_and_argument_errors():
    from video_dit_dynamic_b200 import sbsa
    # scale bytes: rows padded to 128, one byte per 16 columns
    assert sbsa.sbsa_nvfp4_scale_bytes(1, 64) == 128 * 4
    assert sbsa.sbsa_nvfp4_scale_bytes(300, 512) == 384 * 32
    assert sbsa.sbsa_nvfp4_scale_bytes(122880, 5120) == 122880 * 320
    assert sbsa.sbsa_nvfp4_scale_bytes(10, 100) == 0 and sbsa.sbsa_nvfp4_scale_bytes(0, 64) == 0
    lib = sbsa.load()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: every call below fails its argument checks
    assert lib.sbsa_nvfp4_gemm(128, 256, 256, None, fake, fake, fake, fake, fake, None, fake, None) == 1
    assert b"null" in lib.sbsa_last_error_message()
    for m, n, k in ((0, 256, 256), (128, 250, 256), (128, 256, 320), (128, 256, 128)):
        st = lib.sbsa_nvfp4_gemm(m, n, k, fake, fake, fake, fake, fake, fake, None, fake, None)
        assert st == 1, (m, n, k)
    # misaligned codes
    st = lib.sbsa_nvfp4_gemm(128, 256, 256, ctypes.c_void_p((1 << 20) + 8), fake, fake, fake, fake, fake, None,
                             fake, None)
    assert st == 1 and b"aligned" in lib.sbsa_last_error_message()
    assert lib.sbsa_nvfp4_quantize(fake, 10, 100, fake, fake, fake, None) == 1
    assert lib.sbsa_nvfp4_amax(fake, 10, 12, fake, None) == 1


def test_peer_exchange_argument_errors():
    from video_dit_dynamic_b200 import sbsa
    lib = sbsa.load()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: every call below fails its argument checks
    shape = sbsa.make_ulysses_shape(2, 256, 256, 4, 128)
    put = lib.sbsa_ulysses_put_qkv
    assert put(ctypes.byref(shape), 0, 2, None, fake, 0, 0, None) == 1
    assert put(ctypes.byref(shape), 0, 2, fake, fake, 0, 2, None) == 1 and b"rank" in lib.sbsa_last_error_message()
    assert put(ctypes.byref(shape), 0, 2, fake, fake, 8, 0, None) == 1  # recv_offset not a multiple of 16
    assert put(ctypes.byref(shape), 0, 3, fake, fake, 0, 0, None) == 1  # chunk beyond heads / world
    assert lib.sbsa_ulysses_put_o(ctypes.byref(shape), 0, 2, fake, ctypes.c_void_p((1 << 20) + 4), 0, 0, None) == 1
    sig = lib.sbsa_peer_signal
    assert sig(None, 0, 0, 2, 1, None) == 1
    assert sig(fake, 0, 2, 2, 1, None) == 1 and sig(fake, 0, 0, 0, 1, None) == 1 and sig(fake, 2, 0, 2, 1, None) == 1
    wait = lib.sbsa_peer_wait
    assert wait(None, 2, 1, 1.0, None) == 1
    assert wait(fake, 0, 1, 1.0, None) == 1 and wait(fake, 2, 1, 0.0, None) == 1 and wait(fake, 2, 1, 61.0, None) == 1
    assert wait(ctypes.c_void_p((1 << 20) + 2), 2, 1, 1.0, None) == 1
