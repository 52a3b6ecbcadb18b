"""CPU oracle for dynamic block-sparse attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline /
reference arm import this package.  The product library (``video_dit_dynamic_b200``)
never imports it and shares no code with it.

This module only marshals numpy arrays into ``liboracle.so``, compiled with gcc from
``sbsa_oracle.c``, which holds all of the oracle's arithmetic (fp64, two-pass softmax).
The method it follows is described in that file's header: block means of Q and K
(page "知识卡片：600倍加速，720p视频实时生成！单卡也能带的动14B模型", 方法/产品要点,
bullet 动态稀疏量化注意力), keep-top blocks with the diagonal forced, and dense
softmax attention inside the kept blocks (page "单卡 RTX 5090 跑 Wan2.2-A14B：720p
视频生成只要 3.8 秒", 四步拆解 item 3).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sbsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16, F64 = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (-O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                               "-fno-fast-math", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_pool.argtypes = [I, I, I, I, I, I, P, I, P]
        lib.oracle_pool.restype = None
        lib.oracle_score_row.argtypes = [I, I, P, P, I, P, P]
        lib.oracle_score_row.restype = None
        lib.oracle_select.argtypes = [I, I, I, I, I, P, P, P, P]
        lib.oracle_select.restype = I
        lib.oracle_attention.argtypes = [I, I, I, I, I, I, P, P, P, I, P, P,
                                         ctypes.c_double, ctypes.c_long, P, P]
        lib.oracle_attention.restype = I
        lib.oracle_rope.argtypes = [I, I, I, I, I, I, I, ctypes.c_double, P, I, P]
        lib.oracle_rope.restype = None
        lib.oracle_e4m3_decode.argtypes = [I]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = I
        lib.oracle_quantize_fp8.argtypes = [I, I, I, I, I, I, P, I, P, P, P]
        lib.oracle_quantize_fp8.restype = None
        lib.oracle_e2m1_decode.argtypes = [I]
        lib.oracle_e2m1_decode.restype = ctypes.c_double
        lib.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        lib.oracle_e2m1_encode.restype = I
        lib.oracle_nvfp4_sf_offset.argtypes = [I, I, I]
        lib.oracle_nvfp4_sf_offset.restype = ctypes.c_size_t
        lib.oracle_nvfp4_quantize.argtypes = [I, I, P, I, ctypes.c_float, P, P]
        lib.oracle_nvfp4_quantize.restype = ctypes.c_float
        lib.oracle_nvfp4_dequantize.argtypes = [I, I, P, P, ctypes.c_float, P]
        lib.oracle_nvfp4_dequantize.restype = None
        lib.oracle_set_threads.argtypes = [I]
        lib.oracle_threads_used.restype = I
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _as_input(x) -> tuple[np.ndarray, int]:
    """Return a C-contiguous numpy view and its dtype code.

    bf16 data is passed as its raw uint16 bit patterns (numpy has no bf16)."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    if x.dtype == np.float64:
        return x, F64
    raise TypeError(f"oracle input dtype {x.dtype} not supported (float32, float64, bf16-as-uint16)")


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def threads_used() -> int:
    return int(_load().oracle_threads_used())


def num_blocks(Lp: int, blk: int) -> int:
    return Lp // blk


def pool(x, L: int, blk: int) -> np.ndarray:
    """Block means over valid tokens.  x: [B,H,Lp,d] -> [B,H,nb,d] float64."""
    xa, dt = _as_input(x)
    B, H, Lp, d = xa.shape
    nb = Lp // blk
    out = np.empty((B, H, nb, d), dtype=np.float64)
    _load().oracle_pool(B, H, L, Lp, d, blk, _ptr(xa), dt, _ptr(out))
    return out


def rope_pairs(d: int) -> tuple[int, int, int]:
    """Rotation pairs per axis (frame, row, column) for head dim d (see sbsa_oracle.c)."""
    ph = d // 6
    return d // 2 - 2 * ph, ph, ph


def rope(x, grid: tuple[int, int, int], theta: float = 10000.0) -> np.ndarray:
    """3D RoPE of x [B][H][Lp][d] (fp64 result, same shape; bf16 given as uint16 bits)."""
    a, dt = _as_input(x)
    B, H, Lp, d = a.shape
    out = np.empty((B, H, Lp, d), dtype=np.float64)
    _load().oracle_rope(B, H, Lp, d, grid[0], grid[1], grid[2], float(theta), _ptr(a), dt, _ptr(out))
    return out


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp64 -> nearest bf16, ties to even, rounded once from the fp64 value; returned
    as uint16 bit patterns."""
    f32 = np.asarray(x, dtype=np.float64)
    # exact: split the fp64 value at bf16 precision with round-half-to-even
    m, e = np.frexp(f32)                       # f = m * 2^e, 0.5 <= |m| < 1
    q = np.rint(m * 256.0) / 256.0             # 8 significant bits, ties to even
    r = np.ldexp(q, e).astype(np.float32)      # exactly representable in bf16
    return (r.view(np.uint32) >> 16).astype(np.uint16)


def rope_pool(x, grid: tuple[int, int, int], L: int, blk: int, theta: float = 10000.0):
    """Step 0 + step 1: rotated tensor as bf16 bits, and the block means of those bf16
    values (what the attention then sees)."""
    rot = rope(x, grid, theta)
    bits = bf16_round(rot)
    return bits, pool(bits, L, blk)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """e4m3 codes (uint8) -> values (fp64)."""
    lib = _load()
    table = np.array([lib.oracle_e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x: float) -> int:
    """One fp32 value -> e4m3 code (nearest, ties to even, saturating at +-448)."""
    return int(_load().oracle_e4m3_encode(float(np.float32(x))))


def quantize_fp8(x, L: int, blk: int, smooth=None):
    """Per-block FP8 codes [B,H,Lp,d] (uint8) and scales [B,H,nb] (fp32) of x, after
    subtracting smooth [B,H,d] (fp32, optional) from every valid token."""
    a, dt = _as_input(x)
    B, H, Lp, d = a.shape
    nb = Lp // blk
    codes = np.empty((B, H, Lp, d), dtype=np.uint8)
    scales = np.empty((B, H, nb), dtype=np.float32)
    sm = None if smooth is None else np.ascontiguousarray(smooth, dtype=np.float32).reshape(B * H, d)
    _load().oracle_quantize_fp8(B, H, L, Lp, d, blk, _ptr(a), dt, _ptr(sm) if sm is not None else None,
                                _ptr(codes), _ptr(scales))
    return codes, scales


def dequantize_fp8(codes: np.ndarray, scales: np.ndarray, blk: int) -> np.ndarray:
    """codes [B,H,Lp,d] * their block's scale -> fp64."""
    B, H, Lp, d = codes.shape
    s = np.repeat(scales.astype(np.float64), blk, axis=2)[:, :, :Lp, None]
    return e4m3_decode(codes) * s


def attention_fp8(q_codes, q_scales, k_codes, k_scales, v, L: int, blk: int, row_ptr, col_idx,
                  scale: float = 0.0, units=None) -> np.ndarray:
    """The FP8 path: softmax attention over the kept blocks with Q and K dequantized from
    their codes and block scales (K as quantized, i.e. already smoothed), V as given."""
    qd = dequantize_fp8(q_codes, q_scales, blk)
    kd = dequantize_fp8(k_codes, k_scales, blk)
    va, dt = _as_input(v)
    vd = va.astype(np.float64) if dt == F64 or dt == F32 else \
        (va.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return attention(qd, kd, vd, L, blk, row_ptr, col_idx, scale, units)


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """e2m1 codes (low 4 bits of each entry) -> values (fp64)."""
    lib = _load()
    table = np.array([lib.oracle_e2m1_decode(c) for c in range(16)], dtype=np.float64)
    return table[np.asarray(codes) & 15]


def e2m1_encode(x: float) -> int:
    """One fp32 value -> e2m1 code (nearest, ties to the even code, saturating at +-6)."""
    return int(_load().oracle_e2m1_encode(float(np.float32(x))))


def nvfp4_sf_offset(r: int, kb: int, K: int) -> int:
    """Byte offset of the scale of (row r, 16-element block kb) in a K-column scale array."""
    return int(_load().oracle_nvfp4_sf_offset(r, kb, K))


def nvfp4_sf_bytes(rows: int, K: int) -> int:
    return (rows + 127) // 128 * 128 * (K // 16)


def nvfp4_quantize(x, amax=None):
    """[rows, K] (bf16 bits, fp32 or fp64) -> (codes uint8 [rows, K/2], sf uint8, tensor scale s).

    amax: the tensor's max |x| when x holds rows sampled from a larger tensor."""
    a, dt = _as_input(x)
    rows, K = a.shape
    if K % 64:
        raise ValueError("K must be a multiple of 64")
    codes = np.empty((rows, K // 2), dtype=np.uint8)
    sf = np.empty(nvfp4_sf_bytes(rows, K), dtype=np.uint8)
    s = _load().oracle_nvfp4_quantize(rows, K, _ptr(a), dt, -1.0 if amax is None else float(amax), _ptr(codes), _ptr(sf))
    return codes, sf, float(np.float32(s))


def nvfp4_dequantize(codes: np.ndarray, sf: np.ndarray, s: float) -> np.ndarray:
    """codes [rows, K/2] + scales + tensor scale -> fp64 [rows, K]."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((rows, K), dtype=np.float64)
    _load().oracle_nvfp4_dequantize(rows, K, _ptr(codes), _ptr(sf), ctypes.c_float(s), _ptr(out))
    return out


def nvfp4_gemm(a_codes, a_sf, a_s, b_codes, b_sf, b_s, bias=None) -> np.ndarray:
    """C[M, N] = A_dec @ B_dec^T + bias[N] in fp64, A [M, K] and B [N, K] in NVFP4."""
    c = nvfp4_dequantize(a_codes, a_sf, a_s) @ nvfp4_dequantize(b_codes, b_sf, b_s).T
    if bias is not None:
        c = c + np.asarray(bias, dtype=np.float64)[None, :]
    return c


def quantize_rows_fp8(rows: np.ndarray):
    """Per-row FP8 of a [n, d] matrix: each row one scale amax/448 and e4m3 codes (the FP8
    quantizer above with a block of one row)."""
    n, d = rows.shape
    codes, scales = quantize_fp8(np.ascontiguousarray(rows).reshape(1, 1, n, d), n, 1)
    return codes.reshape(n, d), scales.reshape(n)


def dequantize_rows_bf16(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """code * scale as an fp32 product, rounded to bf16 (ties to even); bf16 bits."""
    p = (e4m3_decode(codes) * scales.astype(np.float64)[:, None]).astype(np.float32)
    return bf16_round(p.astype(np.float64))


def ulysses_qkv(x_shards, heads: int, L: int, Lp: int):
    """Light-Ulysses forward exchange (page "知识卡片：600倍加速，720p视频实时生成！单卡也能带的动
    14B模型", 方法/产品要点, bullet Light-Ulysses 多卡并行; page "单卡 RTX 5090 跑 Wan2.2-A14B：
    720p 视频生成只要 3.8 秒", 四步拆解 item 4): G ranks each hold a contiguous shard of L/G
    tokens of the fused QKV activation, [L/G, 3, H, d]; after one all-to-all with an FP8
    payload rank r holds heads [r H/G, (r+1) H/G) of all L tokens.  Every (token, q/k/v,
    head) row of d values crosses as e4m3 codes with one scale and is restored to bf16.

    x_shards: G arrays of bf16 bits [L/G, 3, H, d].  Returns, per rank, bf16 bits
    [3, H/G, Lp, d] (q, k, v in the attention's layout, tokens t >= L zero)."""
    G = len(x_shards)
    Lr = L // G
    Hg = heads // G
    d = x_shards[0].shape[-1]
    out = []
    for r in range(G):
        dst = np.zeros((3, Hg, Lp, d), dtype=np.uint16)
        for i in range(G):
            rows = np.ascontiguousarray(x_shards[i][:, :, r * Hg:(r + 1) * Hg, :]).reshape(-1, d)
            deq = dequantize_rows_bf16(*quantize_rows_fp8(rows)).reshape(Lr, 3, Hg, d)
            dst[:, :, i * Lr:(i + 1) * Lr, :] = deq.transpose(1, 2, 0, 3)
        out.append(dst)
    return out


def ulysses_o(o_shards, heads: int, L: int):
    """The return exchange: rank r holds the attention output of heads [r H/G, (r+1) H/G)
    for all tokens, [H/G, Lp, d]; afterwards every rank holds all heads of its own token
    shard, [L/G, H, d], each (token, head) row having crossed as FP8 like the forward."""
    G = len(o_shards)
    Lr = L // G
    Hg = heads // G
    d = o_shards[0].shape[-1]
    out = []
    for r in range(G):
        dst = np.zeros((Lr, heads, d), dtype=np.uint16)
        for i in range(G):
            rows = np.ascontiguousarray(o_shards[i][:, r * Lr:(r + 1) * Lr, :].transpose(1, 0, 2)).reshape(-1, d)
            deq = dequantize_rows_bf16(*quantize_rows_fp8(rows)).reshape(Lr, Hg, d)
            dst[:, i * Hg:(i + 1) * Hg, :] = deq
        out.append(dst)
    return out


def score_row(qmean_bh: np.ndarray, kmean_bh: np.ndarray, i: int):
    """Scores s_j = <qmean_i, kmean_j> and a_j = sum |products| for one query block."""
    qm = np.ascontiguousarray(qmean_bh, dtype=np.float64)
    km = np.ascontiguousarray(kmean_bh, dtype=np.float64)
    nb, d = km.shape
    s = np.empty(nb, dtype=np.float64)
    a = np.empty(nb, dtype=np.float64)
    _load().oracle_score_row(nb, d, _ptr(qm), _ptr(km), int(i), _ptr(s), _ptr(a))
    return s, a


def select(qmean: np.ndarray, kmean: np.ndarray, k: int, want_kth: bool = False):
    """Diagonal + top-(k-1) per query block, ascending.  Returns col_idx [B,H,nb,k]
    (int32) and, if asked, the per-row score of the last kept non-diagonal block."""
    qm = np.ascontiguousarray(qmean, dtype=np.float64)
    km = np.ascontiguousarray(kmean, dtype=np.float64)
    B, H, nb, d = qm.shape
    col = np.empty((B, H, nb, k), dtype=np.int32)
    kth = np.empty((B, H, nb), dtype=np.float64) if want_kth else None
    rc = _load().oracle_select(B, H, nb, d, int(k), _ptr(qm), _ptr(km), _ptr(col),
                               _ptr(kth) if want_kth else None)
    if rc != 0:
        raise ValueError(f"oracle_select failed (rc={rc}, k={k}, nb={nb})")
    return (col, kth) if want_kth else col


def uniform_row_ptr(B: int, H: int, nb: int, k: int) -> np.ndarray:
    return (np.arange(B * H * nb + 1, dtype=np.int64) * k).astype(np.int32)


def attention(q, k, v, L: int, blk: int, row_ptr: np.ndarray, col_idx: np.ndarray,
              scale: float = 0.0, units=None) -> np.ndarray:
    """Softmax attention over the kept blocks, fp64.

    units: None for every (b,h,query block), else a list of unit ids bh*nb + i.
    Returns [B,H,Lp,d] (units=None) or [len(units), blk, d]."""
    qa, dt = _as_input(q)
    ka, dt2 = _as_input(k)
    va, dt3 = _as_input(v)
    if not (dt == dt2 == dt3):
        raise TypeError("q, k, v must share a dtype")
    B, H, Lp, d = qa.shape
    nb = Lp // blk
    rp = np.ascontiguousarray(row_ptr, dtype=np.int32).reshape(-1)
    ci = np.ascontiguousarray(col_idx, dtype=np.int32).reshape(-1)
    if units is None:
        out = np.empty((B, H, Lp, d), dtype=np.float64)
        n_units, up = B * H * nb, None
    else:
        ua = np.ascontiguousarray(units, dtype=np.int64)
        out = np.empty((len(ua), blk, d), dtype=np.float64)
        n_units, up = len(ua), _ptr(ua)
    rc = _load().oracle_attention(B, H, L, Lp, d, blk, _ptr(qa), _ptr(ka), _ptr(va), dt,
                                  _ptr(rp), _ptr(ci), float(scale), n_units, up, _ptr(out))
    if rc != 0:
        raise MemoryError("oracle_attention failed")
    return out


def keep_blocks(nb: int, keep_fraction: float) -> int:
    """k = round-half-up(keep * nb), clamped to [1, nb] (the reading of 'keep about
    10-20% of the blocks' as a per-query-block count)."""
    k = int(np.floor(keep_fraction * nb + 0.5))
    return max(1, min(nb, k))


def forward(q, k, v, L: int, blk: int, k_keep: int, scale: float = 0.0):
    """pool -> select -> attend.  Returns (out [B,H,Lp,d], col_idx, qmean, kmean)."""
    qm = pool(q, L, blk)
    km = pool(k, L, blk)
    col = select(qm, km, k_keep)
    B, H, nb, _ = qm.shape
    rp = uniform_row_ptr(B, H, nb, k_keep)
    out = attention(q, k, v, L, blk, rp, col, scale)
    return out, col, qm, km
