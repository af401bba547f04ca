"""Seeded synthetic inputs for the nested W4/W8 linear layer.

This module holds no arithmetic of the method: it only draws random numbers.
Both the CUDA path's callers and the CPU oracle's callers take their inputs
from here, and nothing else is shared between the two.

Generator: counter-based SplitMix64 (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014; the 64-bit finaliser with
constants 0xBF58476D1CE4E5B9 / 0x94D049BB133111EB).  Output i of stream
(seed, stream) is mix64(key + (i + 1) * 0x9E3779B97F4A7C15) with
key = mix64(seed * 2^16 + stream), so any element can be drawn on its own:
rows of a large matrix are generated without generating the rest.

Distributions (the workloads of the bit-nested decode and prefill layers):
  - nibbles   : uniform integers in [0, 15], 16 per 64-bit output;
  - scales    : fp16(1e-4 + 0.005 * |z|), z ~ N(0, 1), one per (row, 128-group);
  - activations: fp16(z), z ~ N(0, 1), with 4 seeded outlier channels x20;
  - z ~ N(0, 1) by Box-Muller in fp64 from two 53-bit uniforms in (0, 1].
"""
from __future__ import annotations

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
M1 = np.uint64(0xBF58476D1CE4E5B9)
M2 = np.uint64(0x94D049BB133111EB)

# seed bases (a projection's id is added)
SEED_WEIGHTS = 1000
SEED_SCALES = 2000
SEED_ACTS = 3000
SEED_OUTLIERS = 4000

STREAM_HI = 0
STREAM_LO = 1


def _mix64(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * M1
        z = (z ^ (z >> np.uint64(27))) * M2
        return z ^ (z >> np.uint64(31))


def _key(seed: int, stream: int) -> np.uint64:
    v = np.array([(int(seed) << 16) + int(stream)], dtype=np.uint64)
    return _mix64(v)[0]


def u64(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Outputs start .. start+count-1 of stream (seed, stream)."""
    idx = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = _key(seed, stream) + (idx + np.uint64(1)) * GOLDEN
    return _mix64(z)


def uniform01(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """fp64 uniforms in (0, 1]: ((u >> 11) + 1) * 2^-53."""
    u = u64(seed, stream, start, count)
    return ((u >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def normal(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Element i uses uniforms 2i and 2i+1 of the stream (Box-Muller)."""
    u = uniform01(seed, stream, 2 * start, 2 * count).reshape(count, 2)
    return np.sqrt(-2.0 * np.log(u[:, 0])) * np.cos(2.0 * np.pi * u[:, 1])


def nibbles(seed: int, stream: int, N: int, K: int, row0: int = 0, nrows: int | None = None
            ) -> np.ndarray:
    """Unpacked nibbles uint8 [nrows, K], uniform in [0, 15]; rows row0.. of an [N, K] matrix.

    Element (n, k) is bits 4*(i % 16) .. +3 of output i // 16, i = n*K + k.
    """
    if nrows is None:
        nrows = N - row0
    first = row0 * K
    count = nrows * K
    if count == 0:
        return np.zeros((nrows, K), np.uint8)
    o0 = first // 16
    o1 = (first + count + 15) // 16
    words = u64(seed, stream, o0, o1 - o0)
    b = words.view(np.uint8)  # little-endian: byte t of word = bits 8t..8t+7
    nib = np.empty(b.size * 2, np.uint8)
    nib[0::2] = b & 0xF
    nib[1::2] = b >> 4
    off = first - o0 * 16
    return nib[off:off + count].reshape(nrows, K).copy()


def group_scales(seed: int, N: int, K: int, row0: int = 0, nrows: int | None = None
                 ) -> np.ndarray:
    """fp16 [nrows, K/128] = fp16(1e-4 + 0.005 |z|)."""
    if nrows is None:
        nrows = N - row0
    G = K // 128
    z = normal(seed, 0, row0 * G, nrows * G)
    return (1e-4 + 0.005 * np.abs(z)).astype(np.float16).reshape(nrows, G)


def outlier_channels(K: int, count: int = 4, seed: int = SEED_OUTLIERS) -> np.ndarray:
    """`count` distinct channel indices in [0, K), drawn from the seed."""
    chosen: list[int] = []
    i = 0
    while len(chosen) < min(count, K):
        c = int(u64(seed, 0, i, 1)[0] % np.uint64(K))
        if c not in chosen:
            chosen.append(c)
        i += 1
    return np.array(sorted(chosen), np.int64)


def activations(seed: int, M: int, K: int, n_outliers: int = 4, factor: float = 20.0,
                outlier_seed: int = SEED_OUTLIERS) -> np.ndarray:
    """fp16 [M, K]: N(0,1) with `n_outliers` channels multiplied by `factor`."""
    z = normal(seed, 0, 0, M * K).reshape(M, K)
    if n_outliers:
        z[:, outlier_channels(K, n_outliers, outlier_seed)] *= factor
    return z.astype(np.float16)


def projection_inputs(proj_id: int, M: int, N: int, K: int):
    """The standard seeded set for one projection: (uh, ul, scale, x)."""
    uh = nibbles(SEED_WEIGHTS + proj_id, STREAM_HI, N, K)
    ul = nibbles(SEED_WEIGHTS + proj_id, STREAM_LO, N, K)
    s = group_scales(SEED_SCALES + proj_id, N, K)
    x = activations(SEED_ACTS + proj_id, M, K)
    return uh, ul, s, x


# Llama-3-8B-shaped projections (N, K) and the activation grouping o_proj uses.
LLAMA3_8B_PROJECTIONS = {
    "q_proj": (4096, 4096, 0),
    "k_proj": (1024, 4096, 0),
    "v_proj": (1024, 4096, 0),
    "o_proj": (4096, 4096, 128),
    "gate_proj": (14336, 4096, 0),
    "up_proj": (14336, 4096, 0),
    "down_proj": (4096, 14336, 0),
}
PROJ_IDS = {name: i for i, name in enumerate(LLAMA3_8B_PROJECTIONS)}
