"""BitNest nested W4/W8 linear layer: the CPU oracle (ctypes binding).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
path (``w8_quantized_linear_b200``) never imports, links or calls it, and it
shares no code with the CUDA library: the C source in this folder is a plain,
slow, loop-by-loop statement of the "BitNest-Llama-3-8B" model card's
formulas (section "Files" and the model table) in fp32 (activation
quantiser) and fp64 (layer output).

Every function takes and returns numpy arrays on the host.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, exhaustive identities, library routines (numpy fp32
division and round-half-even, numpy integer and fp64 matmul) and the
hand-worked fixtures under ``tests/golden/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitnest_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DRAFT = 0
TARGET = 1
GROUP = 128

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FP contraction, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = [
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
            "-fno-fast-math", "-ffp-contract=off", "-fexcess-precision=standard",
            _SRC, "-o", _LIB + ".tmp", "-lm",
        ]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    I = ctypes.c_int
    lib.oracle_num_threads.restype = I
    lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_half_to_double.restype = ctypes.c_double
    lib.oracle_float_to_half.argtypes = [ctypes.c_float]
    lib.oracle_float_to_half.restype = ctypes.c_uint16
    lib.oracle_pack_weights.argtypes = [P, I64, I64, P, P, P]
    lib.oracle_nested_attention.argtypes = [I, P, I64, I64, I64, I64, P, P, P, P, P, P, P]
    lib.oracle_h28.argtypes = [I, I]
    lib.oracle_h28.restype = I
    lib.oracle_hadamard_entry.argtypes = [I64, I64, I64]
    lib.oracle_hadamard_entry.restype = I
    lib.oracle_hadamard_rotate.argtypes = [P, I64, I64, P]
    lib.oracle_quantize_f32.argtypes = [P, I64, I64, P, P]
    lib.oracle_pack_plane.argtypes = [P, I64, I64, P]
    lib.oracle_unpack_plane.argtypes = [P, I64, I64, P]
    lib.oracle_dequant.argtypes = [I, P, P, P, I64, I64, P]
    lib.oracle_quantize.argtypes = [P, I64, I64, I, P, P]
    lib.oracle_group_sums.argtypes = [I, P, P, P, I64, I64, I64, P]
    lib.oracle_group_sums.restype = I64
    lib.oracle_linear.argtypes = [I, P, P, P, P, P, I64, I64, I64, I, P, P]
    lib.oracle_linear_subset.argtypes = [I, P, P, P, P, P, I64, I64, I64, I, P, P, I64, P, I64, P]
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _half_bits(a):
    """fp16 array (or its uint16 bit pattern) -> contiguous uint16 bits."""
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    return np.ascontiguousarray(a, dtype=np.uint16)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def half_to_double(bits: int) -> float:
    return float(_load().oracle_half_to_double(int(bits) & 0xFFFF))


def float_to_half_bits(f) -> np.ndarray:
    """fp32 values -> fp16 bit patterns (round to nearest, ties to even)."""
    f = np.ascontiguousarray(np.asarray(f, np.float32))
    lib = _load()
    out = np.array([lib.oracle_float_to_half(float(v)) for v in f.ravel()], np.uint16)
    return out.reshape(f.shape)


def pack_weights(w):
    """fp16 weights [N, K] -> (uh uint8 [N, K], ul uint8 [N, K], scale fp16
    bits [N, K/128]): round-to-nearest 4-bit high nibble with scale
    max|W| / 7 per row and group, closed-form residual low nibble."""
    wb = _half_bits(w)
    N, K = wb.shape
    uh = np.empty((N, K), np.uint8)
    ul = np.empty((N, K), np.uint8)
    sc = np.empty((N, K // GROUP), np.uint16)
    _load().oracle_pack_weights(_ptr(wb), N, K, _ptr(uh), _ptr(ul), _ptr(sc))
    return uh, ul, sc


def kv_pack(kv):
    """fp16 K or V rows [T * Hkv, D] -> (hi, lo planes [T * Hkv, D/2], fp16
    scale bits [T * Hkv, D/128]): the runtime nesting of the cache (the
    weights' packing rule, one group of 128 per row segment)."""
    uh, ul, sc = pack_weights(kv)
    return pack_plane(uh), pack_plane(ul), sc


def nested_attention(mode: int, q, k_planes, v_planes, Hkv: int) -> np.ndarray:
    """Decode attention of one token over a nested KV cache, fp64 [H, D].
    q fp16 [H, D]; k_planes / v_planes = kv_pack(...) of [T * Hkv, D] rows
    (row t * Hkv + j: token t, KV head j); draft reads hi, target hi and lo."""
    qb = _half_bits(q)
    H, D = qb.shape
    k_hi, k_lo, k_sc = (_c(a, t) for a, t in zip(k_planes, (np.uint8, np.uint8, np.uint16)))
    v_hi, v_lo, v_sc = (_c(a, t) for a, t in zip(v_planes, (np.uint8, np.uint8, np.uint16)))
    T = k_hi.shape[0] // Hkv
    out = np.empty((H, D), np.float64)
    _load().oracle_nested_attention(mode, _ptr(qb), H, Hkv, D, T, _ptr(k_hi), _ptr(k_lo),
                                    _ptr(k_sc), _ptr(v_hi), _ptr(v_lo), _ptr(v_sc), _ptr(out))
    return out


def h28() -> np.ndarray:
    """The order-28 Hadamard factor (Paley construction I over GF(27))."""
    lib = _load()
    return np.array([[lib.oracle_h28(i, j) for j in range(28)] for i in range(28)], np.int64)


def hadamard_matrix(K: int) -> np.ndarray:
    """H [K, K] (+-1) of the rotation; small K only (entry by entry)."""
    lib = _load()
    return np.array([[lib.oracle_hadamard_entry(K, i, j) for j in range(K)] for i in range(K)],
                    np.int64)


def hadamard_rotate(x) -> np.ndarray:
    """fp16 [M, K] -> fp64 x H / sqrt(K) (K a power of two or 28 times one)."""
    xb = _half_bits(x)
    M, K = xb.shape
    out = np.empty((M, K), np.float64)
    _load().oracle_hadamard_rotate(_ptr(xb), M, K, _ptr(out))
    return out


def quantize_f32(x):
    """fp32 [M, K] -> (q int8 [M, K], xs fp32 [M]): the per-token quantiser."""
    x = _c(x, np.float32)
    M, K = x.shape
    q = np.empty((M, K), np.int8)
    xs = np.empty((M,), np.float32)
    _load().oracle_quantize_f32(_ptr(x), M, K, _ptr(q), _ptr(xs))
    return q, xs


def hadamard_quantize(x):
    """The down_proj input path: rotate (fp64), round to fp32, quantise per
    token.  Returns (q, xs, x_rot fp64)."""
    xr = hadamard_rotate(x)
    q, xs = quantize_f32(xr.astype(np.float32))
    return q, xs, xr


def pack_plane(u: np.ndarray) -> np.ndarray:
    """Unpacked nibbles uint8 [N, K] -> plane uint8 [N, K/2]."""
    u = _c(u, np.uint8)
    N, K = u.shape
    out = np.empty((N, K // 2), np.uint8)
    _load().oracle_pack_plane(_ptr(u), N, K, _ptr(out))
    return out


def unpack_plane(plane: np.ndarray, K: int) -> np.ndarray:
    """Plane uint8 [N, K/2] -> unpacked nibbles uint8 [N, K]."""
    plane = _c(plane, np.uint8)
    N = plane.shape[0]
    out = np.empty((N, K), np.uint8)
    _load().oracle_unpack_plane(_ptr(plane), N, K, _ptr(out))
    return out


def dequant(mode: int, hi, lo, scale, K: int) -> np.ndarray:
    """Dequantised weight W fp64 [N, K] (draft or target formula)."""
    hi = _c(hi, np.uint8)
    lo = _c(lo, np.uint8) if mode == TARGET else None
    scale = _half_bits(scale)
    N = hi.shape[0]
    W = np.empty((N, K), np.float64)
    _load().oracle_dequant(mode, _ptr(hi), _ptr(lo), _ptr(scale), N, K, _ptr(W))
    return W


def quantize(x, group: int = 0):
    """fp16 activations [M, K] -> (q int8 [M, K], xs fp32 [M] or [M, K/128])."""
    xb = _half_bits(x)
    M, K = xb.shape
    q = np.empty((M, K), np.int8)
    xs = np.empty((M,) if group == 0 else (M, K // GROUP), np.float32)
    _load().oracle_quantize(_ptr(xb), M, K, int(group), _ptr(q), _ptr(xs))
    return q, xs


def group_sums(mode: int, hi, lo, q, K: int) -> np.ndarray:
    """int32 S [M, N, K/128] of q times the integer weight code, per group."""
    hi = _c(hi, np.uint8)
    lo = _c(lo, np.uint8) if mode == TARGET else None
    q = _c(q, np.int8)
    M, N = q.shape[0], hi.shape[0]
    S = np.empty((M, N, K // GROUP), np.int32)
    over = _load().oracle_group_sums(mode, _ptr(hi), _ptr(lo), _ptr(q), M, N, K, _ptr(S))
    if over:
        raise OverflowError(f"{over} group sums do not fit int32")
    return S


def linear(mode: int, hi, lo, scale, q, xs, K: int, act_group: int = 0, bias=None,
           toks=None, rows=None) -> np.ndarray:
    """fp64 y [M, N] (or [len(toks), len(rows)] for a subset)."""
    hi = _c(hi, np.uint8)
    lo = _c(lo, np.uint8) if mode == TARGET else None
    scale = _half_bits(scale)
    q = _c(q, np.int8)
    xs = _c(xs, np.float32)
    bias = _half_bits(bias)
    M, N = q.shape[0], hi.shape[0]
    lib = _load()
    if toks is None and rows is None:
        y = np.empty((M, N), np.float64)
        lib.oracle_linear(mode, _ptr(hi), _ptr(lo), _ptr(scale), _ptr(q), _ptr(xs), M, N, K,
                          int(act_group), _ptr(bias), _ptr(y))
        return y
    toks = np.ascontiguousarray(np.arange(M) if toks is None else toks, dtype=np.int64)
    rows = np.ascontiguousarray(np.arange(N) if rows is None else rows, dtype=np.int64)
    y = np.empty((len(toks), len(rows)), np.float64)
    lib.oracle_linear_subset(mode, _ptr(hi), _ptr(lo), _ptr(scale), _ptr(q), _ptr(xs), M, N, K,
                             int(act_group), _ptr(bias), _ptr(toks), len(toks), _ptr(rows),
                             len(rows), _ptr(y))
    return y


def max_normalised_error(y, y_ref) -> float:
    """max |y - y_ref| / (|y_ref| + 1e-3 * rms(y_ref)), elementwise."""
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    if y_ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(y_ref * y_ref)))
    den = np.abs(y_ref) + 1e-3 * rms
    den = np.where(den == 0, 1.0, den)
    return float(np.max(np.abs(y - y_ref) / den))
