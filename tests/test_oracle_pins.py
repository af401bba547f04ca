"""Pins of the CPU oracle to facts fixed outside it (no GPU).

Each test ties one oracle routine to something it does not compute itself:
the page's worked layout, hand-worked quantiser cases, an exhaustive
identity, a closed form, a library routine (numpy fp32 division and
round-half-even, numpy integer / fp64 matmul) or brute force on tiny shapes.
Formulas cited are those of the BitNest-Llama-3-8B model card, section
"Files" (plane layout and the draft / target dequantisation) and its model
table (group size 128; symmetric int8 activations, per token, per 128-group
for o_proj).
"""
import os

import numpy as np
import pytest

from w8_quantized_linear_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- layout
def _read_layout():
    cases = []
    with open(os.path.join(GOLDEN, "plane_layout.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            left, right = line.split("|")
            nib = [int(t, 16) for t in left.split()]
            byt = [int(t, 16) for t in right.split()]
            cases.append((np.array(nib, np.uint8), np.array(byt, np.uint8)))
    return cases


def test_pack_matches_page_layout(oracle_mod):
    for nib, byt in _read_layout():
        K = nib.size
        got = oracle_mod.pack_plane(nib.reshape(1, K))
        assert got.tolist() == [byt.tolist()]
        back = oracle_mod.unpack_plane(byt.reshape(1, K // 2), K)
        assert back.tolist() == [nib.tolist()]


def test_pack_unpack_exhaustive(oracle_mod):
    # every byte value unpacks to two nibbles that pack back to it
    plane = np.arange(256, dtype=np.uint8).reshape(1, 256)
    u = oracle_mod.unpack_plane(plane, 512)
    assert u.max() <= 15
    assert np.array_equal(oracle_mod.pack_plane(u), plane)
    # column 2j is the low nibble, 2j+1 the high nibble
    assert np.array_equal(u[0, 0::2], np.arange(256) & 15)
    assert np.array_equal(u[0, 1::2], np.arange(256) >> 4)


def test_pack_multirow_random(oracle_mod):
    u = synth.nibbles(7, 0, 5, 256)
    p = oracle_mod.pack_plane(u)
    assert p.shape == (5, 128)
    assert np.array_equal(oracle_mod.unpack_plane(p, 256), u)


# ------------------------------------------------------- weight formulas
def _all_pairs_planes():
    """One row holding every (hi, lo) nibble pair, column c = 16*h + l."""
    h = np.repeat(np.arange(16, dtype=np.uint8), 16)
    l = np.tile(np.arange(16, dtype=np.uint8), 16)
    return h, l


def test_target_code_identity_all_256_pairs(oracle_mod):
    """16(h-8)+(l-8) equals the unsigned byte (h<<4|l) minus 136, for all pairs."""
    h, l = _all_pairs_planes()
    K = 256
    hi = oracle_mod.pack_plane(h.reshape(1, K))
    lo = oracle_mod.pack_plane(l.reshape(1, K))
    one = np.full((1, K // 128), 0x3C00, np.uint16)  # fp16 1.0
    Wt = oracle_mod.dequant(oracle_mod.TARGET, hi, lo, one, K)[0]
    byte = (h.astype(np.int64) << 4) | l
    assert np.array_equal(Wt * 16, (byte - 136).astype(np.float64))
    assert (Wt * 16).min() == -136 and (Wt * 16).max() == 119
    assert len(np.unique(Wt)) == 256
    Wd = oracle_mod.dequant(oracle_mod.DRAFT, hi, None, one, K)[0]
    assert np.array_equal(Wd, h.astype(np.float64) - 8)


def test_dequant_scale_applies_per_group(oracle_mod):
    K = 384
    u = np.full((2, K), 9, np.uint8)  # code +1
    hi = oracle_mod.pack_plane(u)
    scale = np.array([[1.0, 2.0, 0.5], [4.0, 0.25, 8.0]], np.float16)
    W = oracle_mod.dequant(oracle_mod.DRAFT, hi, None, scale, K)
    expect = np.repeat(scale.astype(np.float64), 128, axis=1)
    assert np.array_equal(W, expect)


# ---------------------------------------------------------- fp16 decoding
def test_half_decoding_matches_numpy(oracle_mod):
    bits = np.arange(0, 65536, 97, dtype=np.uint16)
    bits = bits[(bits & 0x7C00) != 0x7C00]  # finite values only
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle_mod.half_to_double(int(b)) for b in bits])
    assert np.array_equal(got, ref)
    for b in (0x0001, 0x03FF, 0x0400, 0x7BFF, 0x8001, 0x3C00, 0xBC00):
        assert oracle_mod.half_to_double(b) == float(np.array([b], np.uint16).view(np.float16)[0])


# -------------------------------------------------------------- quantiser
def _read_quant_cases():
    cases = []
    cur = None
    with open(os.path.join(GOLDEN, "quantize_cases.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tok = line.split()
            if tok[0] == "case":
                kv = dict(t.split("=") for t in tok[2:])
                cur = {"name": tok[1], "group": int(kv["group"]), "K": int(kv["K"])}
                cases.append(cur)
            elif tok[0] in ("x", "q"):
                arr = np.zeros(cur["K"], np.float64)
                for t in tok[1:]:
                    i, v = t.split(":")
                    arr[int(i)] = float(v)
                cur[tok[0]] = arr
            elif tok[0] == "s":
                cur["s"] = np.array([float(t) for t in tok[1:]], np.float32)
    return cases


@pytest.mark.parametrize("case", _read_quant_cases(), ids=lambda c: c["name"])
def test_quantize_golden(oracle_mod, case):
    x = case["x"].astype(np.float16).reshape(1, -1)
    assert np.array_equal(x.astype(np.float64)[0], case["x"])  # fixture exact in fp16
    q, xs = oracle_mod.quantize(x, case["group"])
    assert q[0].astype(np.int64).tolist() == case["q"].astype(np.int64).tolist()
    assert np.array_equal(xs.reshape(-1), case["s"])


def test_quantize_subnormal_extreme(oracle_mod):
    x = np.array([[2.0 ** -24, -(2.0 ** -24), 0.0]], np.float16)
    q, xs = oracle_mod.quantize(x, 0)
    assert q.tolist() == [[127, -127, 0]]
    assert xs[0] == np.float32(2.0 ** -24) / np.float32(127)


def _numpy_fp32_quantize(x16, group):
    """The same definition through numpy's IEEE fp32 division and np.rint."""
    x = x16.astype(np.float32)
    M, K = x.shape
    span = K if group == 0 else group
    xr = x.reshape(M, K // span, span)
    amax = np.max(np.abs(xr), axis=2)
    s = (amax / np.float32(127)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.rint(xr / s[:, :, None])
    r = np.where(s[:, :, None] == 0, 0, r)
    q = np.clip(r, -127, 127).astype(np.int8).reshape(M, K)
    return q, (s.reshape(M) if group == 0 else s)


@pytest.mark.parametrize("group", [0, 128])
def test_quantize_matches_numpy_fp32(oracle_mod, group):
    x = synth.activations(11, 9, 1024)
    # add exact-tie values: multiples of 0.5 scaled into range
    x[3, :] = (np.arange(1024) % 255 - 127).astype(np.float16) * np.float16(0.5)
    x[4, :] = 0
    q, xs = oracle_mod.quantize(x, group)
    qr, sr = _numpy_fp32_quantize(x, group)
    assert np.array_equal(q, qr)
    assert np.array_equal(xs, sr)
    assert q.min() >= -127 and q.max() <= 127


def test_quantize_per_group_equals_per_token_on_slices(oracle_mod):
    x = synth.activations(12, 3, 512)
    qg, sg = oracle_mod.quantize(x, 128)
    for g in range(4):
        qt, st = oracle_mod.quantize(x[:, g * 128:(g + 1) * 128], 0)
        assert np.array_equal(qg[:, g * 128:(g + 1) * 128], qt)
        assert np.array_equal(sg[:, g], st)


# ------------------------------------------------------------- group sums
def _tiny_problem(seed, M, N, K):
    uh = synth.nibbles(seed, 0, N, K)
    ul = synth.nibbles(seed, 1, N, K)
    q = (synth.u64(seed, 2, 0, M * K) % np.uint64(255)).astype(np.int64) - 127
    return uh, ul, q.astype(np.int8).reshape(M, K)


@pytest.mark.parametrize("M,N,K", [(1, 1, 128), (2, 3, 256), (5, 2, 384), (3, 5, 128)])
def test_group_sums_equal_integer_matmul(oracle_mod, M, N, K):
    uh, ul, q = _tiny_problem(M * 100 + N * 10 + K, M, N, K)
    hi, lo = oracle_mod.pack_plane(uh), oracle_mod.pack_plane(ul)
    G = K // 128
    q64 = q.astype(np.int64)
    # draft: the integer matmul of q with (uh - 8), one matmul per group
    cd = uh.astype(np.int64) - 8
    # target, through the unsigned-byte form of the code (a different expression)
    ct = ((uh.astype(np.int64) << 4) | ul) - 136
    Sd = oracle_mod.group_sums(oracle_mod.DRAFT, hi, None, q, K)
    St = oracle_mod.group_sums(oracle_mod.TARGET, hi, lo, q, K)
    for g in range(G):
        sl = slice(g * 128, (g + 1) * 128)
        assert np.array_equal(Sd[:, :, g], q64[:, sl] @ cd[:, sl].T)
        assert np.array_equal(St[:, :, g], q64[:, sl] @ ct[:, sl].T)


def test_group_sums_extreme_bounds(oracle_mod):
    K = 128
    q = np.full((2, K), 127, np.int8)
    q[1] = -127
    zero = oracle_mod.pack_plane(np.zeros((1, K), np.uint8))
    full = oracle_mod.pack_plane(np.full((1, K), 15, np.uint8))
    # all hi = lo = 0: code -136 everywhere -> +-128*127*136
    St = oracle_mod.group_sums(oracle_mod.TARGET, zero, zero, q, K)
    assert St[:, 0, 0].tolist() == [-128 * 127 * 136, 128 * 127 * 136]
    Sd = oracle_mod.group_sums(oracle_mod.DRAFT, full, None, q, K)
    assert Sd[:, 0, 0].tolist() == [128 * 127 * 7, -128 * 127 * 7]


def test_closed_form_unit_case(oracle_mod):
    """hi = 9, lo = 8, q = 1, s = 1, xs = 1: both models give 128 per group."""
    K = 256
    hi = oracle_mod.pack_plane(np.full((1, K), 9, np.uint8))
    lo = oracle_mod.pack_plane(np.full((1, K), 8, np.uint8))
    q = np.ones((1, K), np.int8)
    xs = np.ones(1, np.float32)
    s = np.full((1, 2), 1.0, np.float16)
    for mode in (oracle_mod.DRAFT, oracle_mod.TARGET):
        y = oracle_mod.linear(mode, hi, lo, s, q, xs, K)
        assert y.tolist() == [[256.0]]
        S = oracle_mod.group_sums(mode, hi, lo, q, K)
        assert S.reshape(-1).tolist() == ([128, 128] if mode == 0 else [2048, 2048])


# -------------------------------------------------------------- layer output
@pytest.mark.parametrize("M,N,K", [(1, 1, 128), (2, 3, 256), (3, 5, 128), (5, 2, 256)])
@pytest.mark.parametrize("act_group", [0, 128])
def test_linear_dense_bruteforce(oracle_mod, M, N, K, act_group):
    """fp64 dense matmul of the dequantised operands built from the unpacked nibbles."""
    seed = 500 + M + N + K
    uh, ul, _ = _tiny_problem(seed, M, N, K)
    s = synth.group_scales(seed, N, K)
    x = synth.activations(seed, M, K, n_outliers=min(4, K))
    q, xs = oracle_mod.quantize(x, act_group)
    hi, lo = oracle_mod.pack_plane(uh), oracle_mod.pack_plane(ul)
    sd = np.repeat(s.astype(np.float64), 128, axis=1)
    xsd = xs.astype(np.float64)[:, None] if act_group == 0 else np.repeat(xs.astype(np.float64), 128, axis=1)
    xdeq = q.astype(np.float64) * xsd
    W_draft = (uh.astype(np.float64) - 8) * sd
    W_target = ((uh.astype(np.float64) - 8) * 16 + (ul.astype(np.float64) - 8)) * sd / 16
    yd = oracle_mod.linear(oracle_mod.DRAFT, hi, lo, s, q, xs, K, act_group)
    yt = oracle_mod.linear(oracle_mod.TARGET, hi, lo, s, q, xs, K, act_group)
    np.testing.assert_allclose(yd, xdeq @ W_draft.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(yt, xdeq @ W_target.T, rtol=1e-12, atol=1e-12)


def test_linear_unit_scales_is_integer_matmul(oracle_mod):
    M, N, K = 4, 6, 256
    uh, ul, q = _tiny_problem(77, M, N, K)
    hi, lo = oracle_mod.pack_plane(uh), oracle_mod.pack_plane(ul)
    s = np.ones((N, K // 128), np.float16)
    xs = np.ones(M, np.float32)
    yd = oracle_mod.linear(oracle_mod.DRAFT, hi, lo, s, q, xs, K)
    yt = oracle_mod.linear(oracle_mod.TARGET, hi, lo, s, q, xs, K)
    q64 = q.astype(np.int64)
    assert np.array_equal(yd, (q64 @ (uh.astype(np.int64) - 8).T).astype(np.float64))
    ct = ((uh.astype(np.int64) << 4) | ul) - 136
    assert np.array_equal(yt * 16, (q64 @ ct.T).astype(np.float64))


def test_linear_equals_scaled_group_sums(oracle_mod):
    """y = sum_g xs * s[n,g] * S[m,n,g] (/16 for the target), as the formulas factor."""
    M, N, K = 3, 4, 512
    uh, ul, _ = _tiny_problem(91, M, N, K)
    s = synth.group_scales(91, N, K)
    x = synth.activations(91, M, K)
    hi, lo = oracle_mod.pack_plane(uh), oracle_mod.pack_plane(ul)
    for act_group in (0, 128):
        q, xs = oracle_mod.quantize(x, act_group)
        xs2 = xs[:, None] if act_group == 0 else xs
        for mode, div in ((oracle_mod.DRAFT, 1.0), (oracle_mod.TARGET, 16.0)):
            S = oracle_mod.group_sums(mode, hi, lo, q, K).astype(np.float64)
            y = np.einsum("mng,ng,mg->mn", S, s.astype(np.float64),
                          np.broadcast_to(xs2.astype(np.float64), (M, K // 128))) / div
            np.testing.assert_allclose(oracle_mod.linear(mode, hi, lo, s, q, xs, K, act_group),
                                       y, rtol=1e-12, atol=1e-9)


def test_lo_eight_draft_equals_target(oracle_mod):
    M, N, K = 4, 7, 384
    uh, _, _ = _tiny_problem(5, M, N, K)
    ul = np.full((N, K), 8, np.uint8)
    s = synth.group_scales(5, N, K)
    q, xs = oracle_mod.quantize(synth.activations(5, M, K), 0)
    hi, lo = oracle_mod.pack_plane(uh), oracle_mod.pack_plane(ul)
    yd = oracle_mod.linear(oracle_mod.DRAFT, hi, lo, s, q, xs, K)
    yt = oracle_mod.linear(oracle_mod.TARGET, hi, lo, s, q, xs, K)
    assert np.array_equal(yd, yt)
    assert np.array_equal(oracle_mod.group_sums(1, hi, lo, q, K),
                          16 * oracle_mod.group_sums(0, hi, lo, q, K))


def test_linear_bias_and_subset(oracle_mod):
    M, N, K = 3, 5, 256
    uh, ul, _ = _tiny_problem(8, M, N, K)
    s = synth.group_scales(8, N, K)
    q, xs = oracle_mod.quantize(synth.activations(8, M, K), 0)
    hi, lo = oracle_mod.pack_plane(uh), oracle_mod.pack_plane(ul)
    bias = np.array([1.0, -2.0, 0.5, 0.0, 3.25], np.float16)
    y0 = oracle_mod.linear(1, hi, lo, s, q, xs, K)
    yb = oracle_mod.linear(1, hi, lo, s, q, xs, K, bias=bias)
    assert np.array_equal(yb, y0 + bias.astype(np.float64)[None, :])
    sub = oracle_mod.linear(1, hi, lo, s, q, xs, K, toks=[2, 0], rows=[4, 1, 3])
    assert np.array_equal(sub, y0[[2, 0]][:, [4, 1, 3]])


def test_normalised_error_metric():
    import oracle

    y_ref = np.array([1.0, -2.0, 0.0, 4.0])
    rms = np.sqrt(np.mean(y_ref ** 2))
    y = y_ref + np.array([0, 0, 1e-3 * 1e-3 * rms, 0])
    assert oracle.max_normalised_error(y, y_ref) == pytest.approx(1e-3, rel=1e-9)
    assert oracle.max_normalised_error(y_ref, y_ref) == 0.0


# ------------------------------------------------------- fp16 encoding
def test_float_to_half_exhaustive_round_trip(oracle_mod):
    """Every finite fp16 value, widened to fp32, encodes back to itself."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    bits = bits[(bits & 0x7C00) != 0x7C00]
    f32 = bits.view(np.float16).astype(np.float32)
    assert np.array_equal(oracle_mod.float_to_half_bits(f32), bits)


def test_float_to_half_matches_numpy(oracle_mod):
    """Rounding (ties to even, subnormals, overflow) against numpy's fp16 cast."""
    rng = np.random.default_rng(11)
    mags = np.concatenate([10.0 ** rng.uniform(-9, 5, 4000), [65504, 65519.99, 65520, 70000,
                                                              2.0 ** -25, 2.0 ** -24 * 1.5]])
    f = (mags * rng.choice([-1, 1], mags.size)).astype(np.float32)
    # exact midpoints between neighbouring fp16 values: ties go to the even one
    h = rng.integers(0x0001, 0x7BFE, 500).astype(np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    f = np.concatenate([f, ((lo + hi) / 2).astype(np.float32)])
    with np.errstate(over="ignore"):
        ref = f.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle_mod.float_to_half_bits(f), ref)


# -------------------------------------------------- packer from weights
def _read_pack_cases():
    cases, cur = [], None
    with open(os.path.join(GOLDEN, "pack_weights_cases.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tok = line.split()
            if tok[0] == "case":
                K = int(tok[2].split("=")[1])
                cur = {"name": tok[1], "w": np.zeros(K), "uh": np.full(K, 8), "ul": np.full(K, 8)}
                cases.append(cur)
            elif tok[0] in ("w", "uh", "ul"):
                for t in tok[1:]:
                    i, v = t.split(":")
                    cur[tok[0]][int(i)] = float(v)
            elif tok[0] == "s":
                cur["s"] = int(tok[1], 16)
    return cases


@pytest.mark.parametrize("case", _read_pack_cases(), ids=lambda c: c["name"])
def test_pack_weights_golden(oracle_mod, case):
    w = case["w"].astype(np.float16).reshape(1, -1)
    assert np.array_equal(w.astype(np.float64)[0], case["w"])  # fixture exact in fp16
    uh, ul, sc = oracle_mod.pack_weights(w)
    assert uh[0].tolist() == case["uh"].astype(int).tolist()
    assert ul[0].tolist() == case["ul"].astype(int).tolist()
    assert int(sc[0, 0]) == case["s"]


def test_pack_weights_recovers_codes_on_the_grid(oracle_mod):
    """Weights exactly on the target grid (16 c4 + cl) s / 16, with the group
    maximum 7 s: the packer returns those codes and that scale."""
    rng = np.random.default_rng(3)
    N, K = 6, 512
    s = 2.0 ** -6
    c4 = rng.integers(-6, 7, (N, K))
    cl = rng.integers(-7, 8, (N, K))
    c4[:, ::128] = rng.choice([-7, 7], (N, K // 128))  # one element at +-7 s per group
    cl[:, ::128] = 0
    w = ((16 * c4 + cl) * s / 16).astype(np.float16)
    assert np.array_equal(w.astype(np.float64), (16 * c4 + cl) * s / 16)
    uh, ul, sc = oracle_mod.pack_weights(w)
    assert np.array_equal(uh.astype(int), c4 + 8)
    assert np.array_equal(ul.astype(int), cl + 8)
    assert np.all(sc == np.float16(s).view(np.uint16))


def test_pack_weights_error_bounds(oracle_mod):
    """Random weights: the draft is within s/2 of W, the target within s/16
    (s/32 where the residual is not clipped), per element."""
    rng = np.random.default_rng(4)
    N, K = 8, 1024
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    w[1, :128] = 0  # an all-zero group
    uh, ul, sc = oracle_mod.pack_weights(w)
    hi, lo = oracle_mod.pack_plane(uh), oracle_mod.pack_plane(ul)
    W = w.astype(np.float64)
    s = np.repeat(sc.view(np.float16).astype(np.float64), 128, axis=1)
    d4 = np.abs(oracle_mod.dequant(0, hi, None, sc, K) - W)
    d8 = np.abs(oracle_mod.dequant(1, hi, lo, sc, K) - W)
    assert np.all(d4 <= s * 0.5 * (1 + 2.0 ** -20))
    assert np.all(d8 <= s / 16 * (1 + 2.0 ** -20))
    unclipped = ul < 15
    assert np.all(d8[unclipped] <= s[unclipped] / 32 * (1 + 2.0 ** -20))
    assert sc[1, 0] == 0 and np.all(uh[1, :128] == 8) and np.all(ul[1, :128] == 8)


# ------------------------------------------------- Hadamard rotation (R4)
def test_h28_is_a_skew_hadamard_matrix(oracle_mod):
    """Paley construction I: entries +-1, H H^T = 28 I, and H - I skew-symmetric."""
    H = oracle_mod.h28()
    assert set(np.unique(H).tolist()) == {-1, 1}
    assert np.array_equal(H @ H.T, 28 * np.eye(28, dtype=np.int64))
    S = H - np.eye(28, dtype=np.int64)
    assert np.array_equal(S.T, -S)


@pytest.mark.parametrize("b", range(1, 8))
def test_sylvester_factor_matches_scipy(oracle_mod, b):
    scipy_linalg = pytest.importorskip("scipy.linalg")
    assert np.array_equal(oracle_mod.hadamard_matrix(2 ** b), scipy_linalg.hadamard(2 ** b))


@pytest.mark.parametrize("p", [1, 2, 4])
def test_order_28_p_is_the_kronecker_product(oracle_mod, p):
    """Index i = i28 * p + i': the order-28 factor outer (numpy's kron)."""
    scipy_linalg = pytest.importorskip("scipy.linalg")
    H = oracle_mod.hadamard_matrix(28 * p)
    assert np.array_equal(H, np.kron(oracle_mod.h28(), scipy_linalg.hadamard(p)))
    assert np.array_equal(H @ H.T, 28 * p * np.eye(28 * p, dtype=np.int64))


@pytest.mark.parametrize("K", [128, 112, 224])
def test_rotation_is_x_times_h_over_sqrt_k(oracle_mod, K):
    """Small K: the oracle's rotation against numpy's fp64 matmul with H."""
    x = synth.activations(4242 + K, 3, K)
    H = oracle_mod.hadamard_matrix(K).astype(np.float64)
    ref = x.astype(np.float64) @ H / np.sqrt(K)
    assert np.allclose(oracle_mod.hadamard_rotate(x), ref, rtol=1e-13, atol=1e-13)


def test_rotation_preserves_the_norm_at_down_proj_size(oracle_mod):
    """K = 14336 = 28 * 512: orthogonal (Parseval), and a one-hot input gives
    a row of H / sqrt(K)."""
    K = 14336
    x = synth.activations(4343, 1, K)
    xr = oracle_mod.hadamard_rotate(x)
    n0 = np.sum(x.astype(np.float64) ** 2)
    assert abs(np.sum(xr ** 2) - n0) <= 1e-10 * n0
    e = np.zeros((1, K), np.float16)
    e[0, 1000] = 1.0
    row = oracle_mod.hadamard_rotate(e)[0] * np.sqrt(K)
    i28, ip = divmod(1000, 512)
    scipy_linalg = pytest.importorskip("scipy.linalg")
    ref = np.kron(oracle_mod.h28()[i28], scipy_linalg.hadamard(512)[ip])
    assert np.allclose(row, ref, atol=1e-12)


def test_quantize_f32_matches_numpy_and_fp16_path(oracle_mod):
    """fp32 quantiser: numpy fp32 division and round-half-even; on fp16
    values it equals the fp16 quantiser."""
    x16 = synth.activations(4444, 5, 1024)
    q, xs = oracle_mod.quantize_f32(x16.astype(np.float32))
    q16, xs16 = oracle_mod.quantize(x16, 0)
    assert np.array_equal(q, q16) and np.array_equal(xs, xs16)
    x = (np.random.default_rng(5).standard_normal((4, 777)) * 3).astype(np.float32)
    amax = np.max(np.abs(x), axis=1)
    s = (amax / np.float32(127.0)).astype(np.float32)
    ref = np.clip(np.rint(x / s[:, None]), -127, 127).astype(np.int8)
    q, xs = oracle_mod.quantize_f32(x)
    assert np.array_equal(xs, s) and np.array_equal(q, ref)


# ------------------------------------- nested KV cache: decode attention
def _kv_case(seed, H, Hkv, D, T):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((H, D)).astype(np.float16)
    k = (rng.standard_normal((T * Hkv, D)) * 0.7).astype(np.float16)
    v = rng.standard_normal((T * Hkv, D)).astype(np.float16)
    return q, k, v


@pytest.mark.parametrize("H,Hkv,D,T", [(4, 2, 128, 7), (8, 8, 128, 3), (32, 8, 128, 33),
                                       (2, 1, 256, 5)])
@pytest.mark.parametrize("mode", [0, 1])
def test_nested_attention_is_softmax_attention_on_the_dequantised_cache(oracle_mod, H, Hkv, D, T,
                                                                       mode):
    """numpy's softmax attention over the (separately pinned) dequantised
    cache, heads grouped as h // (H / Hkv)."""
    q, k, v = _kv_case(H + T, H, Hkv, D, T)
    kp, vp = oracle_mod.kv_pack(k), oracle_mod.kv_pack(v)
    K = oracle_mod.dequant(mode, kp[0], kp[1], kp[2], D).reshape(T, Hkv, D)
    V = oracle_mod.dequant(mode, vp[0], vp[1], vp[2], D).reshape(T, Hkv, D)
    ref = np.empty((H, D))
    for h in range(H):
        j = h // (H // Hkv)
        sc = K[:, j, :] @ q[h].astype(np.float64) / np.sqrt(D)
        p = np.exp(sc - sc.max())
        ref[h] = (p / p.sum()) @ V[:, j, :]
    got = oracle_mod.nested_attention(mode, q, kp, vp, Hkv)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_nested_attention_closed_forms(oracle_mod):
    """One cached token: every head returns its KV head's value row.  A zero
    query: uniform weights, the mean of the value rows."""
    H, Hkv, D = 4, 2, 128
    q, k, v = _kv_case(1, H, Hkv, D, 1)
    kp, vp = oracle_mod.kv_pack(k), oracle_mod.kv_pack(v)
    V = oracle_mod.dequant(1, vp[0], vp[1], vp[2], D)
    out = oracle_mod.nested_attention(1, q, kp, vp, Hkv)
    for h in range(H):
        assert np.array_equal(out[h], V[h // 2])
    T = 6
    _, k, v = _kv_case(2, H, Hkv, D, T)
    kp, vp = oracle_mod.kv_pack(k), oracle_mod.kv_pack(v)
    V = oracle_mod.dequant(0, vp[0], None, vp[2], D).reshape(T, Hkv, D)
    out = oracle_mod.nested_attention(0, np.zeros((H, D), np.float16), kp, vp, Hkv)
    for h in range(H):
        assert np.allclose(out[h], V[:, h // 2, :].mean(axis=0), rtol=1e-13, atol=1e-13)


def test_nested_attention_draft_equals_target_when_lo_is_eight(oracle_mod):
    H, Hkv, D, T = 8, 2, 128, 9
    q, k, v = _kv_case(3, H, Hkv, D, T)
    kp, vp = list(oracle_mod.kv_pack(k)), list(oracle_mod.kv_pack(v))
    eight = oracle_mod.pack_plane(np.full((T * Hkv, D), 8, np.uint8))
    kp[1], vp[1] = eight, eight
    d = oracle_mod.nested_attention(0, q, kp, vp, Hkv)
    t = oracle_mod.nested_attention(1, q, kp, vp, Hkv)
    assert np.array_equal(d, t)
