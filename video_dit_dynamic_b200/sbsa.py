"""ctypes binding of libsbsa.so: one Python function per C entry point, same names.

Argument marshalling only (torch tensors -> device pointers, current CUDA stream);
every step of the computation runs in the library's kernels.  There is no fallback:
if the library cannot be loaded, or a tensor is not a CUDA tensor of the right dtype
and layout, the call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch


_HERE = os.path.dirname(os.path.abspath(__file__))

SBSA_OK = 0
STATUS_NAMES = {0: "SBSA_OK", 1: "SBSA_ERR_INVALID_ARG", 2: "SBSA_ERR_UNSUPPORTED", 3: "SBSA_ERR_WORKSPACE",
                4: "SBSA_ERR_CUDA", 5: "SBSA_ERR_TIMEOUT", 6: "SBSA_ERR_BAD_INDEX"}

# Every symbol include/sbsa.h declares.
EXPORTS = ("sbsa_version", "sbsa_status_string", "sbsa_last_error_message", "sbsa_keep_blocks",
           "sbsa_workspace_bytes", "sbsa_pool_qk", "sbsa_select_blocks", "sbsa_attention_fwd", "sbsa_forward",
           "sbsa_check", "sbsa_validate_csr", "sbsa_forward_noalloc", "sbsa_rope_table_floats",
           "sbsa_rope_table_init", "sbsa_rope_pool_qk", "sbsa_key_mean", "sbsa_quantize_qk_fp8",
           "sbsa_attention_fwd_fp8", "sbsa_nvfp4_scale_bytes", "sbsa_nvfp4_amax", "sbsa_nvfp4_quantize",
           "sbsa_nvfp4_gemm", "sbsa_ulysses_qkv_bytes", "sbsa_ulysses_o_bytes", "sbsa_ulysses_pack_qkv",
           "sbsa_ulysses_unpack_qkv", "sbsa_ulysses_pack_o", "sbsa_ulysses_unpack_o", "sbsa_ulysses_put_qkv",
           "sbsa_ulysses_put_o", "sbsa_peer_signal", "sbsa_peer_wait", "sbsa_forward_host",
           "sbsa_set_pipeline_wait_ns")


class SbsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class UlyssesShape(ctypes.Structure):
    _fields_ = [("world", ctypes.c_int32), ("tokens", ctypes.c_int32), ("tokens_padded", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("seq_len", ctypes.c_int32),
                ("seq_len_padded", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32)]

    @property
    def num_blocks(self) -> int:
        return self.seq_len_padded // self.block_size

    def __repr__(self):
        return (f"Shape(B={self.batch}, H={self.heads}, L={self.seq_len}, Lp={self.seq_len_padded}, "
                f"d={self.head_dim}, block={self.block_size})")


def make_shape(batch, heads, seq_len, head_dim, block_size, seq_len_padded=None) -> Shape:
    if seq_len_padded is None:
        seq_len_padded = -(-seq_len // block_size) * block_size
    return Shape(batch, heads, seq_len, seq_len_padded, head_dim, block_size)


_lib = None


def library_path() -> str:
    return os.path.join(_HERE, "libsbsa.so")


def load(path: str | None = None):
    """Load libsbsa.so (raises OSError if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or library_path()
    if not os.path.exists(path):
        raise OSError(f"{path} not found: build it with `python -m video_dit_dynamic_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    SP = ctypes.POINTER(Shape)
    lib.sbsa_version.restype = I32
    lib.sbsa_status_string.argtypes = [ctypes.c_int]
    lib.sbsa_status_string.restype = ctypes.c_char_p
    lib.sbsa_last_error_message.restype = ctypes.c_char_p
    lib.sbsa_keep_blocks.argtypes = [I32, ctypes.c_double]
    lib.sbsa_keep_blocks.restype = I32
    lib.sbsa_workspace_bytes.argtypes = [SP, I32]
    lib.sbsa_workspace_bytes.restype = SZ
    lib.sbsa_pool_qk.argtypes = [SP, P, P, P, P, P]
    lib.sbsa_select_blocks.argtypes = [SP, P, P, I32, P, P, P]
    lib.sbsa_attention_fwd.argtypes = [SP, P, P, P, P, P, ctypes.c_float, P, P]
    lib.sbsa_forward.argtypes = [SP, P, P, P, I32, ctypes.c_float, P, P, P, SZ, P]
    lib.sbsa_forward_noalloc.argtypes = [SP, P, P, P, I32, ctypes.c_float, P, P, P]
    lib.sbsa_forward_host.argtypes = [SP, P, P, P, I32, ctypes.c_float, P, P, P, P, P, P, SZ, I32, P, P, P]
    lib.sbsa_set_pipeline_wait_ns.argtypes = [ctypes.c_uint64]
    lib.sbsa_check.argtypes = [P]
    lib.sbsa_validate_csr.argtypes = [SP, P, P, ctypes.c_int64, I32, P]
    lib.sbsa_rope_table_floats.argtypes = [I32, I32, I32, I32]
    lib.sbsa_rope_table_floats.restype = SZ
    lib.sbsa_rope_table_init.argtypes = [I32, I32, I32, I32, ctypes.c_double, P, P]
    lib.sbsa_rope_pool_qk.argtypes = [SP, I32, I32, I32, P, P, P, P, P, P, P, P]
    lib.sbsa_key_mean.argtypes = [SP, P, P, P]
    lib.sbsa_quantize_qk_fp8.argtypes = [SP, P, P, P, P, P, P, P, P]
    lib.sbsa_attention_fwd_fp8.argtypes = [SP, P, P, P, P, P, P, P, ctypes.c_float, P, P]
    lib.sbsa_nvfp4_scale_bytes.argtypes = [ctypes.c_int64, I32]
    lib.sbsa_nvfp4_scale_bytes.restype = SZ
    lib.sbsa_nvfp4_amax.argtypes = [P, ctypes.c_int64, I32, P, P]
    lib.sbsa_nvfp4_quantize.argtypes = [P, ctypes.c_int64, I32, P, P, P, P]
    lib.sbsa_nvfp4_gemm.argtypes = [I32, I32, I32, P, P, P, P, P, P, P, P, P]
    UP = ctypes.POINTER(UlyssesShape)
    lib.sbsa_ulysses_qkv_bytes.argtypes = [UP, I32]
    lib.sbsa_ulysses_qkv_bytes.restype = SZ
    lib.sbsa_ulysses_o_bytes.argtypes = [UP, I32]
    lib.sbsa_ulysses_o_bytes.restype = SZ
    lib.sbsa_ulysses_pack_qkv.argtypes = [UP, I32, I32, P, P, P]
    lib.sbsa_ulysses_unpack_qkv.argtypes = [UP, I32, I32, P, P, P, P, P]
    lib.sbsa_ulysses_pack_o.argtypes = [UP, I32, I32, P, P, P]
    lib.sbsa_ulysses_unpack_o.argtypes = [UP, I32, I32, P, P, P]
    U64 = ctypes.c_uint64
    lib.sbsa_ulysses_put_qkv.argtypes = [UP, I32, I32, P, P, U64, I32, P]
    lib.sbsa_ulysses_put_o.argtypes = [UP, I32, I32, P, P, U64, I32, P]
    lib.sbsa_peer_signal.argtypes = [P, U64, I32, I32, ctypes.c_uint32, P]
    lib.sbsa_peer_wait.argtypes = [P, I32, ctypes.c_uint32, ctypes.c_double, P]
    for name in ("sbsa_ulysses_pack_qkv", "sbsa_ulysses_unpack_qkv", "sbsa_ulysses_pack_o", "sbsa_ulysses_unpack_o",
                 "sbsa_ulysses_put_qkv", "sbsa_ulysses_put_o", "sbsa_peer_signal", "sbsa_peer_wait"):
        getattr(lib, name).restype = ctypes.c_int
    for name in ("sbsa_pool_qk", "sbsa_select_blocks", "sbsa_attention_fwd", "sbsa_forward", "sbsa_check",
                 "sbsa_validate_csr", "sbsa_forward_noalloc", "sbsa_forward_host", "sbsa_set_pipeline_wait_ns",
                 "sbsa_rope_table_init", "sbsa_rope_pool_qk",
                 "sbsa_key_mean", "sbsa_quantize_qk_fp8", "sbsa_attention_fwd_fp8", "sbsa_nvfp4_amax",
                 "sbsa_nvfp4_quantize", "sbsa_nvfp4_gemm"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _raise_on(status: int):
    if status != SBSA_OK:
        msg = load().sbsa_last_error_message().decode(errors="replace")
        raise SbsaError(status, msg)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dev(t: torch.Tensor, dtype, name: str) -> ctypes.c_void_p:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _check_numel(t: torch.Tensor, n: int, name: str):
    if t.numel() < n:
        raise ValueError(f"{name} has {t.numel()} elements, needs {n}")


# ---------------------------------------------------------------- entry points

def sbsa_version() -> int:
    return int(load().sbsa_version())


def sbsa_status_string(status: int) -> str:
    return load().sbsa_status_string(int(status)).decode()


def sbsa_keep_blocks(num_blocks: int, keep_fraction: float) -> int:
    return int(load().sbsa_keep_blocks(int(num_blocks), float(keep_fraction)))


def sbsa_workspace_bytes(shape: Shape, k_keep: int) -> int:
    return int(load().sbsa_workspace_bytes(ctypes.byref(shape), int(k_keep)))


def sbsa_pool_qk(shape: Shape, q, k, q_mean, k_mean, stream=None):
    n_in = shape.batch * shape.heads * shape.seq_len_padded * shape.head_dim
    n_out = shape.batch * shape.heads * shape.num_blocks * shape.head_dim
    for t, nm, n in ((q, "q", n_in), (k, "k", n_in), (q_mean, "q_mean", n_out), (k_mean, "k_mean", n_out)):
        _check_numel(t, n, nm)
    _raise_on(load().sbsa_pool_qk(ctypes.byref(shape), _dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"),
                                  _dev(q_mean, torch.float32, "q_mean"), _dev(k_mean, torch.float32, "k_mean"),
                                  _stream(stream)))


def sbsa_rope_table_floats(head_dim: int, grid) -> int:
    return int(load().sbsa_rope_table_floats(int(head_dim), int(grid[0]), int(grid[1]), int(grid[2])))


def sbsa_rope_table_init(head_dim: int, grid, theta: float, table, stream=None):
    _check_numel(table, sbsa_rope_table_floats(head_dim, grid), "table")
    _raise_on(load().sbsa_rope_table_init(int(head_dim), int(grid[0]), int(grid[1]), int(grid[2]), float(theta),
                                          _dev(table, torch.float32, "table"), _stream(stream)))


def sbsa_rope_pool_qk(shape: Shape, grid, table, q, k, q_out, k_out, q_mean, k_mean, stream=None):
    n_in = shape.batch * shape.heads * shape.seq_len_padded * shape.head_dim
    n_out = shape.batch * shape.heads * shape.num_blocks * shape.head_dim
    for t, nm, n in ((q, "q", n_in), (k, "k", n_in), (q_out, "q_out", n_in), (k_out, "k_out", n_in),
                     (q_mean, "q_mean", n_out), (k_mean, "k_mean", n_out)):
        _check_numel(t, n, nm)
    _check_numel(table, sbsa_rope_table_floats(shape.head_dim, grid), "table")
    _raise_on(load().sbsa_rope_pool_qk(ctypes.byref(shape), int(grid[0]), int(grid[1]), int(grid[2]),
                                       _dev(table, torch.float32, "table"), _dev(q, torch.bfloat16, "q"),
                                       _dev(k, torch.bfloat16, "k"), _dev(q_out, torch.bfloat16, "q_out"),
                                       _dev(k_out, torch.bfloat16, "k_out"), _dev(q_mean, torch.float32, "q_mean"),
                                       _dev(k_mean, torch.float32, "k_mean"), _stream(stream)))


def sbsa_key_mean(shape: Shape, k_mean, out, stream=None):
    rows = shape.batch * shape.heads
    _check_numel(k_mean, rows * shape.num_blocks * shape.head_dim, "k_mean")
    _check_numel(out, rows * shape.head_dim, "out")
    _raise_on(load().sbsa_key_mean(ctypes.byref(shape), _dev(k_mean, torch.float32, "k_mean"),
                                   _dev(out, torch.float32, "out"), _stream(stream)))


def sbsa_quantize_qk_fp8(shape: Shape, q, k, k_smooth, q8, k8, q_scale, k_scale, stream=None):
    n_in = shape.batch * shape.heads * shape.seq_len_padded * shape.head_dim
    rows = shape.batch * shape.heads * shape.num_blocks
    for t, nm in ((q, "q"), (k, "k"), (q8, "q8"), (k8, "k8")):
        _check_numel(t, n_in, nm)
    _check_numel(q_scale, rows, "q_scale")
    _check_numel(k_scale, rows, "k_scale")
    sm = None
    if k_smooth is not None:
        _check_numel(k_smooth, shape.batch * shape.heads * shape.head_dim, "k_smooth")
        sm = _dev(k_smooth, torch.float32, "k_smooth")
    _raise_on(load().sbsa_quantize_qk_fp8(ctypes.byref(shape), _dev(q, torch.bfloat16, "q"),
                                          _dev(k, torch.bfloat16, "k"), sm, _dev(q8, torch.uint8, "q8"),
                                          _dev(k8, torch.uint8, "k8"), _dev(q_scale, torch.float32, "q_scale"),
                                          _dev(k_scale, torch.float32, "k_scale"), _stream(stream)))


def sbsa_attention_fwd_fp8(shape: Shape, q8, k8, v, q_scale, k_scale, row_ptr, col_idx, scale: float, o,
                           stream=None):
    n_in = shape.batch * shape.heads * shape.seq_len_padded * shape.head_dim
    rows = shape.batch * shape.heads * shape.num_blocks
    for t, nm in ((q8, "q8"), (k8, "k8"), (v, "v"), (o, "o")):
        _check_numel(t, n_in, nm)
    _check_numel(q_scale, rows, "q_scale")
    _check_numel(k_scale, rows, "k_scale")
    _check_numel(row_ptr, rows + 1, "row_ptr")
    _raise_on(load().sbsa_attention_fwd_fp8(ctypes.byref(shape), _dev(q8, torch.uint8, "q8"),
                                            _dev(k8, torch.uint8, "k8"), _dev(v, torch.bfloat16, "v"),
                                            _dev(q_scale, torch.float32, "q_scale"),
                                            _dev(k_scale, torch.float32, "k_scale"),
                                            _dev(row_ptr, torch.int32, "row_ptr"), _dev(col_idx, torch.int32, "col_idx"),
                                            float(scale), _dev(o, torch.bfloat16, "o"), _stream(stream)))


def make_ulysses_shape(world: int, tokens: int, tokens_padded: int, heads: int, head_dim: int = 128) -> UlyssesShape:
    return UlyssesShape(world, tokens, tokens_padded, heads, head_dim)


def sbsa_ulysses_qkv_bytes(shape: UlyssesShape, head_chunk: int) -> int:
    return int(load().sbsa_ulysses_qkv_bytes(ctypes.byref(shape), head_chunk))


def sbsa_ulysses_o_bytes(shape: UlyssesShape, head_chunk: int) -> int:
    return int(load().sbsa_ulysses_o_bytes(ctypes.byref(shape), head_chunk))


def _uly_sizes(shape: UlyssesShape):
    lr, hg = shape.tokens // max(shape.world, 1), shape.heads // max(shape.world, 1)
    return lr, hg


def sbsa_ulysses_pack_qkv(shape: UlyssesShape, head0: int, head_chunk: int, x, send, stream=None):
    lr, _ = _uly_sizes(shape)
    _check_numel(x, lr * 3 * shape.heads * shape.head_dim, "x")
    _check_numel(send, sbsa_ulysses_qkv_bytes(shape, head_chunk), "send")
    _raise_on(load().sbsa_ulysses_pack_qkv(ctypes.byref(shape), head0, head_chunk, _dev(x, torch.bfloat16, "x"),
                                           _dev(send, torch.uint8, "send"), _stream(stream)))


def sbsa_ulysses_unpack_qkv(shape: UlyssesShape, head0: int, head_chunk: int, recv, q, k, v, stream=None):
    _, hg = _uly_sizes(shape)
    _check_numel(recv, sbsa_ulysses_qkv_bytes(shape, head_chunk), "recv")
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _check_numel(t, hg * shape.tokens_padded * shape.head_dim, nm)
    _raise_on(load().sbsa_ulysses_unpack_qkv(ctypes.byref(shape), head0, head_chunk, _dev(recv, torch.uint8, "recv"),
                                             _dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"),
                                             _dev(v, torch.bfloat16, "v"), _stream(stream)))


def sbsa_ulysses_pack_o(shape: UlyssesShape, head0: int, head_chunk: int, o, send, stream=None):
    _, hg = _uly_sizes(shape)
    _check_numel(o, hg * shape.tokens_padded * shape.head_dim, "o")
    _check_numel(send, sbsa_ulysses_o_bytes(shape, head_chunk), "send")
    _raise_on(load().sbsa_ulysses_pack_o(ctypes.byref(shape), head0, head_chunk, _dev(o, torch.bfloat16, "o"),
                                         _dev(send, torch.uint8, "send"), _stream(stream)))


def sbsa_ulysses_unpack_o(shape: UlyssesShape, head0: int, head_chunk: int, recv, y, stream=None):
    lr, _ = _uly_sizes(shape)
    _check_numel(recv, sbsa_ulysses_o_bytes(shape, head_chunk), "recv")
    _check_numel(y, lr * shape.heads * shape.head_dim, "y")
    _raise_on(load().sbsa_ulysses_unpack_o(ctypes.byref(shape), head0, head_chunk, _dev(recv, torch.uint8, "recv"),
                                           _dev(y, torch.bfloat16, "y"), _stream(stream)))


def sbsa_ulysses_put_qkv(shape: UlyssesShape, head0: int, head_chunk: int, x, peer_bases, recv_offset: int,
                         rank: int, stream=None):
    """Pack x and write slice j into rank j's receive buffer at peer_bases[j] + recv_offset
    (peer_bases: int64 CUDA tensor of the world's allocation base addresses)."""
    lr, _ = _uly_sizes(shape)
    _check_numel(x, lr * 3 * shape.heads * shape.head_dim, "x")
    _check_numel(peer_bases, shape.world, "peer_bases")
    _raise_on(load().sbsa_ulysses_put_qkv(ctypes.byref(shape), head0, head_chunk, _dev(x, torch.bfloat16, "x"),
                                          _dev(peer_bases, torch.int64, "peer_bases"), recv_offset, rank,
                                          _stream(stream)))


def sbsa_ulysses_put_o(shape: UlyssesShape, head0: int, head_chunk: int, o, peer_bases, recv_offset: int, rank: int,
                       stream=None):
    _, hg = _uly_sizes(shape)
    _check_numel(o, hg * shape.tokens_padded * shape.head_dim, "o")
    _check_numel(peer_bases, shape.world, "peer_bases")
    _raise_on(load().sbsa_ulysses_put_o(ctypes.byref(shape), head0, head_chunk, _dev(o, torch.bfloat16, "o"),
                                        _dev(peer_bases, torch.int64, "peer_bases"), recv_offset, rank,
                                        _stream(stream)))


def sbsa_peer_signal(peer_bases, flag_offset: int, rank: int, world: int, value: int, stream=None):
    _check_numel(peer_bases, world, "peer_bases")
    _raise_on(load().sbsa_peer_signal(_dev(peer_bases, torch.int64, "peer_bases"), flag_offset, rank, world,
                                      value & 0xFFFFFFFF, _stream(stream)))


def sbsa_peer_wait(flags, world: int, value: int, timeout_s: float = 10.0, stream=None):
    """Device-side wait until the `world` uint32 words at `flags` (an int32 CUDA tensor or a
    view of one) all equal `value`; a wait that runs out latches SBSA_ERR_TIMEOUT."""
    _check_numel(flags, world, "flags")
    _raise_on(load().sbsa_peer_wait(_dev(flags, torch.int32, "flags"), world, value & 0xFFFFFFFF, timeout_s,
                                    _stream(stream)))


def sbsa_nvfp4_scale_bytes(rows: int, cols: int) -> int:
    return int(load().sbsa_nvfp4_scale_bytes(rows, cols))


def sbsa_nvfp4_amax(x, amax, stream=None):
    """amax (1-element fp32 CUDA tensor) = max |x| over a bf16 [rows, cols] CUDA tensor."""
    rows, cols = x.shape
    _check_numel(amax, 1, "amax")
    _raise_on(load().sbsa_nvfp4_amax(_dev(x, torch.bfloat16, "x"), rows, cols, _dev(amax, torch.float32, "amax"),
                                     _stream(stream)))


def sbsa_nvfp4_quantize(x, amax, codes, scales, stream=None):
    """bf16 [rows, cols] -> codes (uint8, rows*cols/2) and scales (uint8, sbsa_nvfp4_scale_bytes)."""
    rows, cols = x.shape
    _check_numel(amax, 1, "amax")
    _check_numel(codes, rows * cols // 2, "codes")
    _check_numel(scales, sbsa_nvfp4_scale_bytes(rows, cols), "scales")
    _raise_on(load().sbsa_nvfp4_quantize(_dev(x, torch.bfloat16, "x"), rows, cols, _dev(amax, torch.float32, "amax"),
                                         _dev(codes, torch.uint8, "codes"), _dev(scales, torch.uint8, "scales"),
                                         _stream(stream)))


def sbsa_nvfp4_gemm(m: int, n: int, k: int, a, a_scales, a_amax, b, b_scales, b_amax, bias, c, stream=None):
    """c [m, n] bf16 = A B^T / (s_A s_B) + bias, A [m, k] and B [n, k] as NVFP4 codes + scales."""
    _check_numel(a, m * k // 2, "a")
    _check_numel(b, n * k // 2, "b")
    _check_numel(a_scales, sbsa_nvfp4_scale_bytes(m, k), "a_scales")
    _check_numel(b_scales, sbsa_nvfp4_scale_bytes(n, k), "b_scales")
    _check_numel(c, m * n, "c")
    bp = None
    if bias is not None:
        _check_numel(bias, n, "bias")
        bp = _dev(bias, torch.float32, "bias")
    _raise_on(load().sbsa_nvfp4_gemm(m, n, k, _dev(a, torch.uint8, "a"), _dev(a_scales, torch.uint8, "a_scales"),
                                     _dev(a_amax, torch.float32, "a_amax"), _dev(b, torch.uint8, "b"),
                                     _dev(b_scales, torch.uint8, "b_scales"), _dev(b_amax, torch.float32, "b_amax"),
                                     bp, _dev(c, torch.bfloat16, "c"), _stream(stream)))


def sbsa_select_blocks(shape: Shape, q_mean, k_mean, k_keep: int, row_ptr, col_idx, stream=None):
    rows = shape.batch * shape.heads * shape.num_blocks
    _check_numel(q_mean, rows * shape.head_dim, "q_mean")
    _check_numel(k_mean, rows * shape.head_dim, "k_mean")
    _check_numel(row_ptr, rows + 1, "row_ptr")
    _check_numel(col_idx, rows * int(k_keep), "col_idx")
    _raise_on(load().sbsa_select_blocks(ctypes.byref(shape), _dev(q_mean, torch.float32, "q_mean"),
                                        _dev(k_mean, torch.float32, "k_mean"), int(k_keep),
                                        _dev(row_ptr, torch.int32, "row_ptr"), _dev(col_idx, torch.int32, "col_idx"),
                                        _stream(stream)))


def sbsa_attention_fwd(shape: Shape, q, k, v, row_ptr, col_idx, scale: float, o, stream=None):
    n_in = shape.batch * shape.heads * shape.seq_len_padded * shape.head_dim
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _check_numel(t, n_in, nm)
    _check_numel(row_ptr, shape.batch * shape.heads * shape.num_blocks + 1, "row_ptr")
    _raise_on(load().sbsa_attention_fwd(ctypes.byref(shape), _dev(q, torch.bfloat16, "q"),
                                        _dev(k, torch.bfloat16, "k"), _dev(v, torch.bfloat16, "v"),
                                        _dev(row_ptr, torch.int32, "row_ptr"), _dev(col_idx, torch.int32, "col_idx"),
                                        float(scale), _dev(o, torch.bfloat16, "o"), _stream(stream)))


def sbsa_forward(shape: Shape, q, k, v, k_keep: int, scale: float, o, col_idx_out, workspace, stream=None):
    n_in = shape.batch * shape.heads * shape.seq_len_padded * shape.head_dim
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _check_numel(t, n_in, nm)
    ci = ctypes.c_void_p(0)
    if col_idx_out is not None:
        _check_numel(col_idx_out, shape.batch * shape.heads * shape.num_blocks * int(k_keep), "col_idx_out")
        ci = _dev(col_idx_out, torch.int32, "col_idx_out")
    if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda:
        raise TypeError("workspace must be a CUDA tensor")
    _raise_on(load().sbsa_forward(ctypes.byref(shape), _dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"),
                                  _dev(v, torch.bfloat16, "v"), int(k_keep), float(scale),
                                  _dev(o, torch.bfloat16, "o"), ci, ctypes.c_void_p(workspace.data_ptr()),
                                  workspace.numel() * workspace.element_size(), _stream(stream)))


def sbsa_forward_noalloc(shape: Shape, q, k, v, k_keep: int, scale: float, o, col_idx_out=None, stream=None):
    """sbsa_forward for callers that cannot allocate device memory (no workspace: the
    library's built-in 16 MiB scratch array holds the block means and block lists).
    Calls that overlap on the GPU share that array and must be serialized."""
    n_in = shape.batch * shape.heads * shape.seq_len_padded * shape.head_dim
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _check_numel(t, n_in, nm)
    ci = ctypes.c_void_p(0)
    if col_idx_out is not None:
        _check_numel(col_idx_out, shape.batch * shape.heads * shape.num_blocks * int(k_keep), "col_idx_out")
        ci = _dev(col_idx_out, torch.int32, "col_idx_out")
    _raise_on(load().sbsa_forward_noalloc(ctypes.byref(shape), _dev(q, torch.bfloat16, "q"),
                                          _dev(k, torch.bfloat16, "k"), _dev(v, torch.bfloat16, "v"), int(k_keep),
                                          float(scale), _dev(o, torch.bfloat16, "o"), ci, _stream(stream)))


def sbsa_check(stream=None):
    _raise_on(load().sbsa_check(_stream(stream)))


def sbsa_validate_csr(shape: Shape, row_ptr, col_idx, nnz: int, require_diagonal: bool = True, stream=None) -> bool:
    """True if the CSR list is well formed; False on SBSA_ERR_BAD_INDEX; raises otherwise."""
    st = load().sbsa_validate_csr(ctypes.byref(shape), _dev(row_ptr, torch.int32, "row_ptr"),
                                  ctypes.c_void_p(col_idx.data_ptr() if col_idx is not None and col_idx.numel() else 0),
                                  int(nnz), 1 if require_diagonal else 0, _stream(stream))
    if st == 6:
        return False
    _raise_on(st)
    return True


# ---------------------------------------------------------------- conveniences

def alloc_workspace(shape: Shape, k_keep: int, device="cuda") -> torch.Tensor:
    """A device byte buffer of sbsa_workspace_bytes() (torch allocations are 256-byte aligned)."""
    n = sbsa_workspace_bytes(shape, k_keep)
    if n == 0:
        raise SbsaError(1, "invalid shape or k_keep for workspace")
    return torch.empty(n, dtype=torch.uint8, device=device)


_copy_streams = {}


def _side_streams(device):
    """Two streams per device, one for host-to-device and one for device-to-host copies."""
    key = torch.device(device).index if torch.device(device).index is not None else torch.cuda.current_device()
    if key not in _copy_streams:
        _copy_streams[key] = (torch.cuda.Stream(device=key), torch.cuda.Stream(device=key))
    return _copy_streams[key]


def _host(t: torch.Tensor, name: str) -> ctypes.c_void_p:
    if t.device.type != "cpu" or t.dtype != torch.bfloat16 or not t.is_contiguous():
        raise SbsaError(1, f"{name} must be a contiguous bf16 host tensor")
    return ctypes.c_void_p(t.data_ptr())


def sbsa_forward_host(shape: Shape, q_host, k_host, v_host, k_keep: int, scale: float, o_host, q, k, v, o, workspace,
                      pairs_per_chunk: int = 0, stream=None, h2d_stream=None, d2h_stream=None):
    """pool -> select -> attend from host tensors through the device buffers q, k, v, o
    (copies and kernels chunked over (batch, head) pairs on three streams)."""
    n = shape.batch * shape.heads * shape.seq_len_padded * shape.head_dim
    for t, nm in ((q_host, "q_host"), (k_host, "k_host"), (v_host, "v_host"), (o_host, "o_host")):
        _check_numel(t, n, nm)
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _check_numel(t, n, nm)
    st = load().sbsa_forward_host(ctypes.byref(shape), _host(q_host, "q_host"), _host(k_host, "k_host"),
                                  _host(v_host, "v_host"), int(k_keep), float(scale), _host(o_host, "o_host"),
                                  _dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"),
                                  _dev(v, torch.bfloat16, "v"), _dev(o, torch.bfloat16, "o"),
                                  _dev(workspace, torch.uint8, "workspace"), workspace.numel(), int(pairs_per_chunk),
                                  _stream(stream),
                                  # NULL copy streams: the copies run on `stream`
                                  _stream(h2d_stream) if h2d_stream is not None else ctypes.c_void_p(0),
                                  _stream(d2h_stream) if d2h_stream is not None else ctypes.c_void_p(0))
    _raise_on(st)


def sbsa_set_pipeline_wait_ns(limit_ns: int):
    """Limit of the kernels' pipeline waits on the current device (1e9 by default; 0 drives
    the give-up path in tests)."""
    _raise_on(load().sbsa_set_pipeline_wait_ns(int(limit_ns)))


def forward_from_host(shape: Shape, q_host, k_host, v_host, k_keep: int, scale: float = 0.0, *, o_host=None,
                      device_buffers=None, stream=None, head_chunk: int | None = None):
    """End-to-end call from host tensors through sbsa_forward_host: Q/K/V copied in (from
    pinned host memory), pool -> select -> attend, O copied out, chunked over (batch,
    head) pairs so that copies and kernels overlap.  ``device_buffers`` (q, k, v, o,
    workspace) may be passed to reuse device memory across calls.  Returns the host output
    tensor.  Asynchronous with respect to the host; the work is complete once ``stream``
    (default: the current stream) is."""
    s = stream or torch.cuda.current_stream()
    if device_buffers is None:
        dq = torch.empty(q_host.shape, dtype=torch.bfloat16, device="cuda")
        dk, dv, do = torch.empty_like(dq), torch.empty_like(dq), torch.empty_like(dq)
        ws = alloc_workspace(shape, k_keep)
    else:
        dq, dk, dv, do, ws = device_buffers
    if o_host is None:
        o_host = torch.empty(do.shape, dtype=do.dtype, pin_memory=True)
    h2d, d2h = _side_streams(dq.device)
    sbsa_forward_host(shape, q_host, k_host, v_host, k_keep, scale, o_host, dq, dk, dv, do, ws,
                      pairs_per_chunk=head_chunk or 0, stream=s, h2d_stream=h2d, d2h_stream=d2h)
    return o_host
