"""GPU parity of the tcgen05 tensor-core path against the CPU oracle.

Same bar as the decode GEMV: the int32 per-group sums equal the oracle's
bit for bit; y satisfies max|y - y_ref| / (|y_ref| + 1e-3 rms(y_ref)) <= 1e-3.
Shapes span several 128-row weight tiles and token tiles with ragged tails
in both, and the Llama-3-8B-shaped prefill (M = 2048) on sampled outputs.
"""
import numpy as np
import pytest

import oracle
import w8_quantized_linear_b200 as bn
from w8_quantized_linear_b200 import synth

pytestmark = pytest.mark.gpu
TOL = 1e-3

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from test_gpu_parity import DEV, Problem, dev, host  # noqa: E402


@pytest.fixture(autouse=True)
def _no_wait_timeouts():
    bn.device_wait_timeout(reset=True)
    yield
    torch.cuda.synchronize()
    assert bn.device_wait_timeout(reset=True) == 0


SHAPES = [(1, 1, 128), (9, 100, 256), (16, 128, 1024), (17, 129, 384), (33, 300, 1152),
          (64, 256, 512), (100, 200, 4096), (128, 128, 128), (129, 257, 1024),
          (300, 130, 640), (512, 128, 256), (520, 300, 384), (1000, 129, 1152)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("mode", [0, 1])
def test_tc_group_sums_bit_exact(M, N, K, mode):
    p = Problem(M, N, K, seed=M + 3 * N)
    S = bn.debug_group_sums(mode, p.d_hi, p.d_lo, p.d_xq, p.d_xsum, path=bn.PATH_TC)
    torch.cuda.synchronize()
    assert np.array_equal(host(S), oracle.group_sums(mode, p.hi, p.lo, p.q, K))


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("act_group", [0, 128])
def test_tc_output(M, N, K, mode, act_group):
    p = Problem(M, N, K, seed=N + K + M, act_group=act_group)
    y = p.y_gpu(mode, path=bn.PATH_TC)
    assert oracle.max_normalised_error(y, p.y_ref(mode)) <= TOL


def test_tc_bias():
    p = Problem(20, 150, 512, seed=4, bias=True)
    for mode in (0, 1):
        assert oracle.max_normalised_error(p.y_gpu(mode, bn.PATH_TC), p.y_ref(mode)) <= TOL


@pytest.mark.parametrize("M", [5, 40, 128])
def test_tc_draft_equals_target_when_lo_is_eight(M):
    p = Problem(M, 257, 1024, seed=6, lo_eight=True)
    assert np.array_equal(p.y_gpu(0, bn.PATH_TC), p.y_gpu(1, bn.PATH_TC))


@pytest.mark.parametrize("M", [1, 4, 8])
def test_tc_and_gemv_agree(M):
    p = Problem(M, 384, 2048, seed=11)
    for mode in (0, 1):
        y_tc = p.y_gpu(mode, bn.PATH_TC)
        y_gv = p.y_gpu(mode, bn.PATH_GEMV)
        ref = p.y_ref(mode)
        assert oracle.max_normalised_error(y_tc, ref) <= TOL
        assert oracle.max_normalised_error(y_gv, ref) <= TOL
        S_tc = bn.debug_group_sums(mode, p.d_hi, p.d_lo, p.d_xq, p.d_xsum, path=bn.PATH_TC)
        S_gv = bn.debug_group_sums(mode, p.d_hi, p.d_lo, p.d_xq, p.d_xsum, path=bn.PATH_GEMV)
        assert torch.equal(S_tc, S_gv)


@pytest.mark.parametrize("name", list(synth.LLAMA3_8B_PROJECTIONS))
def test_llama3_prefill_sampled(name):
    """Target W8A8 at M = 2048 on the full Llama-3-8B-shaped projection; the
    oracle evaluates a sample of rows x tokens and the exact sums of a sample."""
    N, K, act_group = synth.LLAMA3_8B_PROJECTIONS[name]
    M = 2048
    pid = synth.PROJ_IDS[name]
    uh = synth.nibbles(synth.SEED_WEIGHTS + pid, synth.STREAM_HI, N, K)
    ul = synth.nibbles(synth.SEED_WEIGHTS + pid, synth.STREAM_LO, N, K)
    s = synth.group_scales(synth.SEED_SCALES + pid, N, K)
    x = synth.activations(synth.SEED_ACTS + pid, M, K)
    d_hi, d_lo = bn.pack_planes(dev(uh), dev(ul))
    d_xq, d_xs, d_xsum = bn.quantize_act(dev(x), act_group)
    y = host(bn.linear(1, d_hi, d_lo, dev(s), d_xq, d_xs, d_xsum, act_group))
    torch.cuda.synchronize()
    rng = np.random.default_rng(pid)
    rows = np.unique(np.concatenate([[0, 127, 128, N - 1], rng.choice(N, 60, replace=False)]))
    toks = np.unique(np.concatenate([[0, 127, 128, M - 1], rng.choice(M, 28, replace=False)]))
    hi_r, lo_r = oracle.pack_plane(uh[rows]), oracle.pack_plane(ul[rows])
    q, xs = oracle.quantize(x, act_group)
    y_ref = oracle.linear(1, hi_r, lo_r, s[rows], q[toks], xs[toks], K, act_group)
    assert oracle.max_normalised_error(y[np.ix_(toks, rows)], y_ref) <= TOL
    # the exact int32 sums of a few weight tiles
    S = bn.debug_group_sums(1, d_hi[:256], d_lo[:256], d_xq, d_xsum)
    S = host(S)
    S_ref = oracle.group_sums(1, oracle.pack_plane(uh[:256]), oracle.pack_plane(ul[:256]),
                              q[toks], K)
    assert np.array_equal(S[toks], S_ref)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("act_group", [0, 128])
def test_tc_persistent_tiles(mode, act_group):
    """More tiles (32 row tiles x 5 token tiles, both ragged) than SMs: every
    CTA walks several tiles; outputs and exact sums over the whole problem."""
    M, N, K = 600, 4000, 256
    p = Problem(M, N, K, seed=77 + mode, act_group=act_group)
    y = p.y_gpu(mode, path=bn.PATH_TC)
    assert oracle.max_normalised_error(y, p.y_ref(mode)) <= TOL
    if act_group == 0:
        S = bn.debug_group_sums(mode, p.d_hi, p.d_lo, p.d_xq, p.d_xsum, path=bn.PATH_TC)
        torch.cuda.synchronize()
        assert np.array_equal(host(S), oracle.group_sums(mode, p.hi, p.lo, p.q, K))


# ------------------------------------------------------------------ split K
SPLIT_SHAPES = [(1, 100, 4096), (16, 300, 1024), (33, 129, 2048), (100, 1000, 1152),
                (128, 256, 14336)]


@pytest.mark.parametrize("M,N,K", SPLIT_SHAPES)
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("act_group", [0, 128])
def test_tc_split_k_matches_oracle(M, N, K, mode, act_group):
    """Too few (row tile, token tile) pairs to fill the GPU: the tensor-core
    path splits K through the scratch (ragged K ranges, ragged tiles).  y
    matches the oracle, and a second call on the same scratch (whose
    counters the first left at zero) gives the same bits."""
    p = Problem(M, N, K, seed=31 * M + N, act_group=act_group, bias=(M == 33))
    nbytes = bn.linear_ws_bytes(mode, M, N, K, bn.PATH_TC)
    assert nbytes > 0
    ws = bn.workspace(nbytes, DEV)
    args = (mode, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum, ws, act_group, p.d_bias)
    y1 = bn.linear_ws(*args, path=bn.PATH_TC)
    y2 = bn.linear_ws(*args, path=bn.PATH_TC)
    torch.cuda.synchronize()
    assert oracle.max_normalised_error(host(y1), p.y_ref(mode)) <= TOL
    assert torch.equal(y1, y2)
    assert int(torch.count_nonzero(ws[:8192])) == 0  # the arrival counters, left at zero


def test_tc_split_k_llama3_down_proj_sampled():
    """down_proj (N = 4096, K = 14336) at 16 and 128 tokens, where the split
    applies: sampled rows against the oracle, and the unsplit call agrees."""
    name = "down_proj"
    N, K, act_group = synth.LLAMA3_8B_PROJECTIONS[name]
    pid = synth.PROJ_IDS[name]
    uh = synth.nibbles(synth.SEED_WEIGHTS + pid, synth.STREAM_HI, N, K)
    ul = synth.nibbles(synth.SEED_WEIGHTS + pid, synth.STREAM_LO, N, K)
    s = synth.group_scales(synth.SEED_SCALES + pid, N, K)
    d_hi, d_lo = bn.pack_planes(dev(uh), dev(ul))
    rows = np.unique(np.concatenate([[0, 127, 128, N - 1],
                                     np.random.default_rng(5).choice(N, 40, replace=False)]))
    hi_r, lo_r = oracle.pack_plane(uh[rows]), oracle.pack_plane(ul[rows])
    for M in (16, 128):
        x = synth.activations(synth.SEED_ACTS + pid + M, M, K)
        q, xs = oracle.quantize(x, act_group)
        d_xq, d_xs, d_xsum = bn.quantize_act(dev(x), act_group)
        for mode in (0, 1):
            ws = bn.workspace(bn.linear_ws_bytes(mode, M, N, K, bn.PATH_TC), DEV)
            y = bn.linear_ws(mode, d_hi, d_lo, dev(s), d_xq, d_xs, d_xsum, ws, act_group,
                             path=bn.PATH_TC)
            y0 = bn.linear(mode, d_hi, d_lo, dev(s), d_xq, d_xs, d_xsum, act_group,
                           path=bn.PATH_TC)
            torch.cuda.synchronize()
            y_ref = oracle.linear(mode, hi_r, lo_r if mode else None, s[rows], q, xs, K,
                                  act_group)
            assert oracle.max_normalised_error(host(y)[:, rows], y_ref) <= TOL
            assert oracle.max_normalised_error(host(y), host(y0).astype(np.float64)) <= TOL


def test_tc_without_split_needs_no_scratch():
    """Enough tiles: no scratch is needed and linear_ws is linear."""
    M, N, K = 300, 2000, 256
    assert bn.linear_ws_bytes(1, M, N, K, bn.PATH_TC) == 0
    p = Problem(M, N, K, seed=5)
    y = bn.linear_ws(1, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum, None, path=bn.PATH_TC)
    y0 = bn.linear(1, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum, path=bn.PATH_TC)
    torch.cuda.synchronize()
    assert torch.equal(y, y0)


def test_tc_split_k_scratch_shared_by_shapes():
    """One scratch for calls of different shapes in turn (each split differs):
    every result equals that of a fresh scratch, so no call disturbs the
    counters another shape relies on."""
    shapes = [(16, 300, 1024), (128, 256, 14336), (8, 4096, 14336), (33, 129, 2048)]
    probs = [Problem(M, N, K, seed=M + N) for M, N, K in shapes]
    need = max(bn.linear_ws_bytes(1, M, N, K, bn.PATH_TC) for M, N, K in shapes)
    shared = bn.workspace(need, DEV)
    for rnd in range(2):
        for p in probs:
            args = (1, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum)
            y = bn.linear_ws(*args, shared, path=bn.PATH_TC)
            fresh = bn.workspace(bn.linear_ws_bytes(1, p.M, p.N, p.K, bn.PATH_TC), DEV)
            y0 = bn.linear_ws(*args, fresh, path=bn.PATH_TC)
            torch.cuda.synchronize()
            assert torch.equal(y, y0), (rnd, p.M, p.N, p.K)
    assert int(torch.count_nonzero(shared[:8192])) == 0


# ---------------------------------------------- without caller group sums
XS_SHAPES = [(5, 37, 1024), (16, 128, 1024), (33, 300, 1152), (128, 257, 512),
             (600, 300, 384), (1030, 150, 640)]


@pytest.mark.parametrize("M,N,K", XS_SHAPES)
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("act_group", [0, 128])
def test_tc_without_group_sums(M, N, K, mode, act_group):
    """xsum = NULL: the tensor-core kernel forms each token's group sums from
    the activation tile it loaded.  y equals the call with the quantiser's
    sums bit for bit and the oracle within the bar; the exact group sums too."""
    p = Problem(M, N, K, seed=13 * M + N, act_group=act_group)
    y0 = bn.linear(mode, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum, act_group,
                   path=bn.PATH_TC)
    y1 = bn.linear(mode, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, None, act_group, path=bn.PATH_TC)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    assert oracle.max_normalised_error(host(y1), p.y_ref(mode)) <= TOL
    if act_group == 0:
        S = bn.debug_group_sums(mode, p.d_hi, p.d_lo, p.d_xq, None, path=bn.PATH_TC)
        torch.cuda.synchronize()
        assert np.array_equal(host(S), oracle.group_sums(mode, p.hi, p.lo, p.q, K))


def test_tc_split_k_without_group_sums():
    """Split K and no caller sums together, on caller scratch."""
    M, N, K = 16, 300, 1024
    p = Problem(M, N, K, seed=8)
    for mode in (0, 1):
        ws = bn.workspace(bn.linear_ws_bytes(mode, M, N, K, bn.PATH_TC), DEV)
        y = bn.linear_ws(mode, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, None, ws, path=bn.PATH_TC)
        torch.cuda.synchronize()
        assert oracle.max_normalised_error(host(y), p.y_ref(mode)) <= TOL
        assert int(torch.count_nonzero(ws[:8192])) == 0


def test_llama3_gate_prefill_without_group_sums():
    """gate_proj at M = 2048 (tiles of 256 tokens) with xsum = NULL: the
    same bits as with the quantiser's sums; sampled outputs against the oracle."""
    name = "gate_proj"
    N, K, act_group = synth.LLAMA3_8B_PROJECTIONS[name]
    M = 2048
    pid = synth.PROJ_IDS[name]
    uh = synth.nibbles(synth.SEED_WEIGHTS + pid, synth.STREAM_HI, N, K)
    ul = synth.nibbles(synth.SEED_WEIGHTS + pid, synth.STREAM_LO, N, K)
    s = synth.group_scales(synth.SEED_SCALES + pid, N, K)
    x = synth.activations(synth.SEED_ACTS + pid + 1, M, K)
    d_hi, d_lo = bn.pack_planes(dev(uh), dev(ul))
    d_s = dev(s)
    d_xq, d_xs, d_xsum = bn.quantize_act(dev(x), act_group)
    y0 = bn.linear(1, d_hi, d_lo, d_s, d_xq, d_xs, d_xsum, act_group)
    y1 = bn.linear(1, d_hi, d_lo, d_s, d_xq, d_xs, None, act_group)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    rng = np.random.default_rng(pid + 1)
    rows = np.unique(np.concatenate([[0, 127, 128, N - 1], rng.choice(N, 40, replace=False)]))
    toks = np.unique(np.concatenate([[0, 255, 256, M - 1], rng.choice(M, 20, replace=False)]))
    q, xs = oracle.quantize(x, act_group)
    y_ref = oracle.linear(1, oracle.pack_plane(uh[rows]), oracle.pack_plane(ul[rows]), s[rows],
                          q[toks], xs[toks], K, act_group)
    assert oracle.max_normalised_error(host(y1)[np.ix_(toks, rows)], y_ref) <= TOL
