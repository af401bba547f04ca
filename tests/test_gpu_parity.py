"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bar (from the layer's definition): plane bytes, int8 activation codes, fp32
activation scales, activation group sums and the int32 per-group weight sums
are bit-exact; the fp32 output y satisfies
    max |y - y_ref| / (|y_ref| + 1e-3 * rms(y_ref)) <= 1e-3
against the oracle's fp64 output.  Inputs are the seeded synthetic workloads
(uniform nibbles, fp16 scales 1e-4 + 0.005|z|, N(0,1) activations with four
x20 outlier channels).
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

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from w8_quantized_linear_b200 import build

    build.build()
    oracle.build()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def host(t):
    return t.detach().cpu().numpy()


class Problem:
    """Seeded problem: host copies for the oracle, device copies for CUDA."""

    def __init__(self, M, N, K, seed=0, act_group=0, lo_eight=False, bias=False):
        self.M, self.N, self.K, self.act_group = M, N, K, act_group
        self.uh = synth.nibbles(1000 + seed, 0, N, K)
        self.ul = np.full((N, K), 8, np.uint8) if lo_eight else synth.nibbles(1000 + seed, 1, N, K)
        self.s = synth.group_scales(2000 + seed, N, K)
        self.x = synth.activations(3000 + seed, M, K) if M else np.zeros((0, K), np.float16)
        self.bias = (synth.normal(5000 + seed, 0, 0, N).astype(np.float16) if bias else None)
        # oracle side
        self.hi = oracle.pack_plane(self.uh)
        self.lo = oracle.pack_plane(self.ul)
        self.q, self.xs = oracle.quantize(self.x, act_group)
        # device side: the CUDA path packs and quantises on its own
        self.d_hi, self.d_lo = bn.pack_planes(dev(self.uh), dev(self.ul))
        self.d_s = dev(self.s)
        self.d_x = dev(self.x)
        self.d_bias = dev(self.bias) if bias else None
        self.d_xq, self.d_xs, self.d_xsum = bn.quantize_act(self.d_x, act_group)

    def y_gpu(self, mode, path=bn.PATH_AUTO):
        y = bn.linear(mode, self.d_hi, self.d_lo, self.d_s, self.d_xq, self.d_xs, self.d_xsum,
                      self.act_group, self.d_bias, path=path)
        torch.cuda.synchronize()
        return host(y)

    def y_ref(self, mode, toks=None, rows=None):
        return oracle.linear(mode, self.hi, self.lo, self.s, self.q, self.xs, self.K,
                             self.act_group, self.bias, toks=toks, rows=rows)


# ------------------------------------------------------------- boundary ops
@pytest.mark.parametrize("N,K", [(1, 128), (7, 256), (64, 1152), (300, 4096)])
def test_pack_planes_bit_exact(N, K):
    u = synth.nibbles(42, 0, N, K)
    u_dirty = u | (synth.nibbles(43, 0, N, K) << 4)  # high bits must be ignored
    hi, _ = bn.pack_planes(dev(u_dirty))
    torch.cuda.synchronize()
    assert np.array_equal(host(hi), oracle.pack_plane(u))


@pytest.mark.parametrize("M,K", [(1, 128), (1, 4096), (4, 14336), (5, 1152), (33, 1024),
                                 (129, 256), (2048, 4096), (16, 2048), (2, 1024), (3, 768),
                                 (7, 512)])
@pytest.mark.parametrize("act_group", [0, 128])
def test_quantize_bit_exact(M, K, act_group):
    x = synth.activations(3100 + M, M, K)
    x[0, :] = 0  # an all-zero token
    if M > 2:
        x[2, : K // 2] = (np.arange(K // 2) % 255 - 127).astype(np.float16) * np.float16(0.5)
    q, xs = oracle.quantize(x, act_group)
    d_xq, d_xs, d_xsum = bn.quantize_act(dev(x), act_group)
    torch.cuda.synchronize()
    assert np.array_equal(host(d_xq), q)
    assert np.array_equal(host(d_xs), xs)
    xsum_ref = q.astype(np.int64).reshape(M, K // 128, 128).sum(axis=2)
    assert np.array_equal(host(d_xsum), xsum_ref)
    assert np.array_equal(host(bn.act_group_sums(d_xq)), xsum_ref)


# ------------------------------------------------------------ group sums
SMALL = [(1, 1, 128), (1, 37, 1024), (2, 64, 1152), (3, 5, 256), (4, 512, 1024),
         (5, 33, 384), (6, 17, 2048), (7, 9, 4224), (8, 130, 1024)]
# two 8-token column blocks of the TMA GEMV's MMA (K a multiple of 1024)
WIDE = [(9, 70, 1024), (12, 33, 2048), (16, 130, 1024), (13, 2500, 4096), (16, 300, 4096)]


@pytest.mark.parametrize("M,N,K", SMALL + WIDE)
@pytest.mark.parametrize("mode", [0, 1])
def test_gemv_group_sums_bit_exact(M, N, K, mode):
    p = Problem(M, N, K, seed=M * 7 + N)
    S_ref = oracle.group_sums(mode, p.hi, p.lo, p.q, K)
    S = bn.debug_group_sums(mode, p.d_hi, p.d_lo, p.d_xq, p.d_xsum, path=bn.PATH_GEMV)
    torch.cuda.synchronize()
    assert np.array_equal(host(S), S_ref)


# ---------------------------------------------------------------- outputs
@pytest.mark.parametrize("M,N,K", SMALL + WIDE + [(4, 300, 14336), (1, 1024, 4096)])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("act_group", [0, 128])
def test_gemv_output(M, N, K, mode, act_group):
    p = Problem(M, N, K, seed=N + K, act_group=act_group)
    y = p.y_gpu(mode, path=bn.PATH_GEMV)
    assert oracle.max_normalised_error(y, p.y_ref(mode)) <= TOL


def test_gemv_bias():
    p = Problem(3, 100, 512, seed=9, bias=True)
    for mode in (0, 1):
        assert oracle.max_normalised_error(p.y_gpu(mode, bn.PATH_GEMV), p.y_ref(mode)) <= TOL


@pytest.mark.parametrize("M", [1, 4, 8, 11, 16])
def test_draft_equals_target_when_lo_is_eight(M):
    p = Problem(M, 257, 2048, seed=3, lo_eight=True)
    yd = p.y_gpu(0, bn.PATH_GEMV)
    yt = p.y_gpu(1, bn.PATH_GEMV)
    assert np.array_equal(yd, yt)


def test_empty_problems_are_noops():
    y = torch.full((0, 16), 7.0, device=DEV)
    p = Problem(1, 16, 128)
    xq = torch.empty((0, 128), dtype=torch.int8, device=DEV)
    xs = torch.empty((0,), dtype=torch.float32, device=DEV)
    xsum = torch.empty((0, 1), dtype=torch.int32, device=DEV)
    # zero tokens: nothing launched, nothing written
    bn.linear(1, p.d_hi, p.d_lo, p.d_s, xq, xs, xsum, out=y)
    torch.cuda.synchronize()


# ------------------------------------------- full-size projections, sampled
def _sample_rows(N, count=48, seed=0):
    rng = np.random.default_rng(seed)
    rows = set([0, 1, N - 2, N - 1]) | set(rng.choice(N, size=min(N, count), replace=False).tolist())
    return np.array(sorted(rows), np.int64)


@pytest.mark.parametrize("name", list(synth.LLAMA3_8B_PROJECTIONS))
def test_llama3_projection_decode_sampled(name):
    """Draft at M=1 and target at M=4 on the full Llama-3-8B-shaped weights;
    the oracle evaluates sampled output rows."""
    N, K, act_group = synth.LLAMA3_8B_PROJECTIONS[name]
    pid = synth.PROJ_IDS[name]
    uh = synth.nibbles(synth.SEED_WEIGHTS + pid, synth.STREAM_HI, N, K)
    ul = synth.nibbles(synth.SEED_WEIGHTS + pid, synth.STREAM_LO, N, K)
    s = synth.group_scales(synth.SEED_SCALES + pid, N, K)
    d_hi, d_lo = bn.pack_planes(dev(uh), dev(ul))
    d_s = dev(s)
    rows = _sample_rows(N, seed=pid)
    hi_rows = oracle.pack_plane(uh[rows])
    lo_rows = oracle.pack_plane(ul[rows])
    for mode, M in ((0, 1), (1, 4)):
        x = synth.activations(synth.SEED_ACTS + pid, M, K)
        q, xs = oracle.quantize(x, act_group)
        d_xq, d_xs, d_xsum = bn.quantize_act(dev(x), act_group)
        y = host(bn.linear(mode, d_hi, d_lo, d_s, d_xq, d_xs, d_xsum, act_group))
        torch.cuda.synchronize()
        y_ref = oracle.linear(mode, hi_rows, lo_rows, s[rows], q, xs, K, act_group)
        assert oracle.max_normalised_error(y[:, rows], y_ref) <= TOL, (name, mode)
        # the exact integer sums of the sampled rows
        S = host(bn.debug_group_sums(mode, d_hi, d_lo, d_xq, d_xsum))
        assert np.array_equal(S[:, rows, :], oracle.group_sums(mode, hi_rows, lo_rows, q, K))


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (4, 1000, 2048), (3, 17, 14336), (8, 64, 1024),
                                   (16, 1000, 4096)])
@pytest.mark.parametrize("mode", [0, 1])
def test_gemv_overlap_launch(M, N, K, mode):
    """Programmatic dependent launch after the quantiser gives the same result."""
    p = Problem(M, N, K, seed=21 + M)
    xq, xs, xsum = bn.quantize_act(p.d_x, 0)
    y = bn.linear(mode, p.d_hi, p.d_lo, p.d_s, xq, xs, xsum,
                  path=bn.PATH_GEMV | bn.PATH_OVERLAP)
    torch.cuda.synchronize()
    assert oracle.max_normalised_error(host(y), p.y_ref(mode)) <= TOL
    assert bn.device_wait_timeout(reset=True) == 0


@pytest.mark.parametrize("M,N,K", [(1, 3, 1024), (2, 9, 2048), (5, 200, 1024), (8, 130, 3072)])
@pytest.mark.parametrize("mode", [0, 1])
def test_gemv_simple_kernel_for_odd_k(M, N, K, mode):
    """K not a multiple of 1024 takes the plain-load GEMV; K that is takes the
    TMA-ring GEMV: both agree with the oracle and with each other's sums."""
    for KK in (K, K + 128):
        p = Problem(M, N, KK, seed=KK + M)
        S = bn.debug_group_sums(mode, p.d_hi, p.d_lo, p.d_xq, p.d_xsum, path=bn.PATH_GEMV)
        torch.cuda.synchronize()
        assert np.array_equal(host(S), oracle.group_sums(mode, p.hi, p.lo, p.q, KK))
        assert oracle.max_normalised_error(p.y_gpu(mode, bn.PATH_GEMV), p.y_ref(mode)) <= TOL


# ------------------------------------------- fused quantiser + linear layer
@pytest.mark.parametrize("M,N,K", [(1, 37, 1024), (4, 300, 4096), (3, 129, 2048), (8, 64, 1024),
                                   (4, 200, 14336), (2, 50, 1152), (12, 130, 1024),
                                   (4, 2500, 2048), (1, 2500, 3072), (7, 2400, 1024)])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("act_group", [0, 128])
def test_quantize_linear_matches_oracle(M, N, K, mode, act_group):
    """One call: the codes, scales and group sums are the quantiser's, bit for
    bit; y matches the oracle, on the GEMV and the tensor-core paths (N > 2368
    gives the decode GEMV's CTAs more than one 16-row block each)."""
    p = Problem(M, N, K, seed=7 * M + N, act_group=act_group)
    for path in (bn.PATH_AUTO, bn.PATH_AUTO | bn.PATH_OVERLAP):
        y, (xq, xs, xsum) = bn.quantize_linear(mode, p.d_hi, p.d_lo, p.d_s, p.d_x, act_group,
                                               path=path)
        torch.cuda.synchronize()
        assert np.array_equal(host(xq), p.q)
        assert np.array_equal(host(xs), p.xs)
        assert np.array_equal(host(xsum), p.q.astype(np.int64).reshape(M, K // 128, 128).sum(2))
        assert oracle.max_normalised_error(host(y), p.y_ref(mode)) <= TOL
    assert bn.device_wait_timeout(reset=True) == 0


def _near_tie_activations(M, K, seed):
    """Rows whose values land near and exactly on half-integers of x / s:
    the quantiser's rounding is decided by the correctly rounded quotient."""
    rng = np.random.default_rng(seed)
    x = np.zeros((M, K), np.float16)
    for m in range(M):
        amax = np.float32(rng.uniform(0.5, 40.0))
        s = np.float32(amax) / np.float32(127.0)
        k = rng.integers(-126, 126, size=K).astype(np.float32) + np.float32(0.5)
        jitter = rng.choice(np.array([0.0, 1e-4, -1e-4, 3e-5, -3e-5, 1e-6], np.float32), size=K)
        x[m] = (k * (1.0 + jitter) * s).astype(np.float16)
        x[m, rng.integers(0, K)] = np.float16(amax)
    return x


@pytest.mark.parametrize("act_group", [0, 128])
def test_quantiser_near_ties_bit_exact(act_group):
    for M, K in ((1, 4096), (4, 14336), (3, 1152)):
        x = _near_tie_activations(M, K, seed=M + K + act_group)
        q, xs = oracle.quantize(x, act_group)
        d_xq, d_xs, _ = bn.quantize_act(dev(x), act_group)
        torch.cuda.synchronize()
        assert np.array_equal(host(d_xq), q)
        assert np.array_equal(host(d_xs), xs)
        if M <= 8:  # the one-call quantise + layer entry point
            p = Problem(M, 40, K, seed=3)
            _, (fq, fs, _) = bn.quantize_linear(0, p.d_hi, p.d_lo, p.d_s, dev(x), act_group)
            torch.cuda.synchronize()
            assert np.array_equal(host(fq), q)
            assert np.array_equal(host(fs), xs)


# ---------------------------------- the bench's own launch configuration
@pytest.mark.parametrize("members", [("gate_proj", "up_proj"), ("q_proj", "k_proj", "v_proj")],
                         ids=["gate_up_N28672", "qkv_N6144"])
def test_fused_layer_group_as_the_bench_launches_it(members):
    """The decode step's fused weights (rows of the member projections
    stacked: gate|up N = 28672, 13 row blocks per CTA; q|k|v N = 6144),
    draft M=1 and target M=4 through the one-call entry with programmatic
    dependent launch, as the bench times them; sampled rows against the
    oracle, codes bit-exact."""
    parts = [synth.LLAMA3_8B_PROJECTIONS[m] for m in members]
    K, g = parts[0][1], parts[0][2]
    uh = np.concatenate([synth.nibbles(synth.SEED_WEIGHTS + synth.PROJ_IDS[m], synth.STREAM_HI,
                                       synth.LLAMA3_8B_PROJECTIONS[m][0], K) for m in members])
    ul = np.concatenate([synth.nibbles(synth.SEED_WEIGHTS + synth.PROJ_IDS[m], synth.STREAM_LO,
                                       synth.LLAMA3_8B_PROJECTIONS[m][0], K) for m in members])
    s = np.concatenate([synth.group_scales(synth.SEED_SCALES + synth.PROJ_IDS[m],
                                           synth.LLAMA3_8B_PROJECTIONS[m][0], K) for m in members])
    N = uh.shape[0]
    d_hi, d_lo = bn.pack_planes(dev(uh), dev(ul))
    d_s = dev(s)
    rows = _sample_rows(N, count=64, seed=N)
    hi_r, lo_r = oracle.pack_plane(uh[rows]), oracle.pack_plane(ul[rows])
    for mode, M in ((0, 1), (1, 4)):
        x = synth.activations(synth.SEED_ACTS + N + mode, M, K)
        y, (xq, xs, _) = bn.quantize_linear(mode, d_hi, d_lo, d_s, dev(x), g,
                                            path=bn.PATH_AUTO | bn.PATH_OVERLAP)
        torch.cuda.synchronize()
        q, xs_ref = oracle.quantize(x, g)
        assert np.array_equal(host(xq), q) and np.array_equal(host(xs), xs_ref)
        y_ref = oracle.linear(mode, hi_r, lo_r if mode else None, s[rows], q, xs_ref, K, g)
        assert oracle.max_normalised_error(host(y)[:, rows], y_ref) <= TOL
    assert bn.device_wait_timeout(reset=True) == 0


# -------------------------------------------- without caller group sums
@pytest.mark.parametrize("M,N,K", [(1, 37, 1024), (4, 300, 4096), (8, 130, 1024),
                                   (3, 17, 14336), (5, 33, 384), (2, 2500, 2048)])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("act_group", [0, 128])
def test_gemv_without_group_sums(M, N, K, mode, act_group):
    """xsum = NULL (a caller holding only int8 codes): the decode GEMV forms
    the per-(token, group) sums from the codes it stages.  Exact group sums,
    y against the oracle, and the same bits as with the quantiser's sums."""
    p = Problem(M, N, K, seed=5 * M + N + K, act_group=act_group)
    y0 = bn.linear(mode, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, p.d_xsum, act_group,
                   path=bn.PATH_GEMV)
    y1 = bn.linear(mode, p.d_hi, p.d_lo, p.d_s, p.d_xq, p.d_xs, None, act_group,
                   path=bn.PATH_GEMV)
    S = bn.debug_group_sums(mode, p.d_hi, p.d_lo, p.d_xq, None, path=bn.PATH_GEMV)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    assert oracle.max_normalised_error(host(y1), p.y_ref(mode)) <= TOL
    assert np.array_equal(host(S), oracle.group_sums(mode, p.hi, p.lo, p.q, K))


@pytest.mark.parametrize("M,N,K", [(1, 300, 4096), (4, 200, 14336), (12, 130, 1024),
                                   (40, 300, 1152)])
@pytest.mark.parametrize("mode", [0, 1])
def test_quantize_linear_without_group_sums(M, N, K, mode):
    """The one-call entry with no xsum buffer: codes and scales bit-exact,
    y against the oracle on the GEMV and the tensor-core paths."""
    p = Problem(M, N, K, seed=3 * M + N)
    xq = torch.empty((M, K), dtype=torch.int8, device=DEV)
    xs = torch.empty((M,), dtype=torch.float32, device=DEV)
    for path in (bn.PATH_AUTO | bn.PATH_OVERLAP, bn.PATH_TC):
        y, _ = bn.quantize_linear(mode, p.d_hi, p.d_lo, p.d_s, p.d_x, act_out=(xq, xs, None),
                                  path=path)
        torch.cuda.synchronize()
        assert np.array_equal(host(xq), p.q) and np.array_equal(host(xs), p.xs)
        assert oracle.max_normalised_error(host(y), p.y_ref(mode)) <= TOL
    assert bn.device_wait_timeout(reset=True) == 0


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (4, 28672, 4096), (4, 4096, 14336),
                                   (8, 300, 1024), (2, 1024, 2048)])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("act_group", [0, 128])
def test_one_launch_quantise_and_apply_equals_two_steps(M, N, K, mode, act_group):
    """On the decode GEMV (with programmatic dependent launch) the one-call
    entry gives, bit for bit, the codes, scales, sums and output of the
    quantiser followed by the layer."""
    p = Problem(M, N, K, seed=11 * M + K, act_group=act_group)
    y1, (q1, s1, u1) = bn.quantize_linear(mode, p.d_hi, p.d_lo, p.d_s, p.d_x, act_group,
                                          path=bn.PATH_GEMV | bn.PATH_OVERLAP)
    q2, s2, u2 = bn.quantize_act(p.d_x, act_group)
    y2 = bn.linear(mode, p.d_hi, p.d_lo, p.d_s, q2, s2, u2, act_group, path=bn.PATH_GEMV)
    torch.cuda.synchronize()
    assert torch.equal(q1, q2) and torch.equal(s1, s2) and torch.equal(u1, u2)
    assert torch.equal(y1, y2)
    assert np.array_equal(host(q1), p.q)
    assert bn.device_wait_timeout(reset=True) == 0
