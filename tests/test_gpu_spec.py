"""GPU: speculative decoding rounds on a synthetic nested model
(bitnest_spec_rounds / bitnest_spec_greedy through the C ABI).

The method's invariant, exactly: the tokens the rounds emit equal the
target's own greedy decoding (same kernels, compared token for token).  Each
greedy step of the GPU is checked against the oracle given the same context
(the argmax of the oracle's fp64 logits, or one of two logits the oracle
cannot tell apart at fp32 rounding).  With lo planes of all 8 the draft is the
target and every draft token is accepted.  The statistics and the capacity
guard are checked as well."""
import numpy as np
import pytest

import oracle
from oracle import spec
import w8_quantized_linear_b200 as bn
from w8_quantized_linear_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from test_gpu_parity import DEV, dev, host  # noqa: E402


def build_model(seed, V=512, d=1024, L=3, lo_eight=False, from_weights=False):
    """The same model on the host (oracle) and the device (library)."""
    layers_h, layers_d = [], []

    def planes(rows, pid):
        if from_weights:  # planes packed from fp16 weights: the draft is close to the target
            w = (0.05 * synth.normal(8100 + seed * 10 + pid, 0, 0, rows * d)).reshape(rows, d)
            uh, ul, sb = oracle.pack_weights(w.astype(np.float16))
            s = sb.view(np.float16)
        else:
            uh = synth.nibbles(8000 + seed * 10 + pid, 0, rows, d)
            ul = synth.nibbles(8000 + seed * 10 + pid, 1, rows, d)
            s = synth.group_scales(8500 + seed * 10 + pid, rows, d)
        if lo_eight:
            ul = np.full_like(ul, 8)
        hi, lo = oracle.pack_plane(uh), oracle.pack_plane(ul)
        return (hi, lo, s), (dev(hi), dev(lo), dev(s))

    for l in range(L):
        h, dv = planes(d, l)
        layers_h.append(h)
        layers_d.append(dv)
    head_h, head_d = planes(V, 9)
    E = synth.normal(8900 + seed, 0, 0, V * d).reshape(V, d).astype(np.float16)
    return spec.Model(E, layers_h, head_h), bn.SpecModel(dev(E), layers_d, head_d)


def buffers(prompt, cap, vocab, dim, gamma):
    seq = torch.full((cap,), -1, dtype=torch.int32, device=DEV)
    seq[:len(prompt)] = torch.tensor(prompt, dtype=torch.int32)
    length = torch.tensor([len(prompt)], dtype=torch.int32, device=DEV)
    stats = torch.zeros(4, dtype=torch.int32, device=DEV)
    work = torch.empty(bn.spec_work_bytes(vocab, dim, gamma), dtype=torch.uint8, device=DEV)
    return seq, length, stats, work


def run_rounds(m, gamma, rounds, prompt):
    seq, length, stats, work = buffers(prompt, len(prompt) + rounds * (gamma + 1), m.vocab, m.dim,
                                       gamma)
    bn.spec_rounds(m, gamma, rounds, seq, length, stats, work)
    torch.cuda.synchronize()
    n = int(length.item())
    return host(seq)[:n].tolist(), host(stats).tolist()


def run_greedy(m, steps, prompt):
    seq, length, stats, work = buffers(prompt, len(prompt) + steps, m.vocab, m.dim, 0)
    bn.spec_greedy(m, steps, seq, length, stats, work)
    torch.cuda.synchronize()
    return host(seq)[:int(length.item())].tolist(), host(stats).tolist()


@pytest.mark.parametrize("seed", [0, 1])
@pytest.mark.parametrize("gamma", [1, 3])
@pytest.mark.parametrize("from_weights", [False, True])
def test_rounds_reproduce_the_target_greedy_output(seed, gamma, from_weights):
    _, m = build_model(seed, from_weights=from_weights)
    prompt = [7, 300]
    s, stats = run_rounds(m, gamma, 8, prompt)
    g, _ = run_greedy(m, len(s) - len(prompt), prompt)
    assert s == g
    rounds, appended, accepted, overflow = stats
    assert rounds == 8 and overflow == 0
    assert appended == len(s) - len(prompt) == rounds + accepted
    assert bn.device_wait_timeout(reset=True) == 0


def test_greedy_steps_match_the_oracle():
    """Each GPU greedy token is the oracle's argmax for the same context,
    unless the oracle's two best logits are within fp32 rounding of each
    other (then either is accepted)."""
    mh, m = build_model(2, V=256, d=1024, L=2)
    prompt = [11, 12]
    g, _ = run_greedy(m, 6, prompt)
    for i in range(len(prompt), len(g)):
        logits = spec.forward_logits(mh, oracle.TARGET, [g[i - 1]], [g[i - 2]])[0]
        order = np.argsort(-logits, kind="stable")
        tol = 1e-4 * float(np.sqrt(np.mean(logits * logits)))
        ok = {int(order[0])}
        if logits[order[0]] - logits[order[1]] <= tol:
            ok.add(int(order[1]))
        assert g[i] in ok, (i, g[i], order[:2], logits[order[:2]])


def test_every_draft_token_accepted_when_the_draft_is_the_target():
    _, m = build_model(3, lo_eight=True)
    s, stats = run_rounds(m, 3, 5, [1, 2])
    assert stats[2] == 15 and stats[1] == 20 and len(s) == 22


def test_capacity_guard_writes_nothing_past_cap():
    _, m = build_model(4, V=256, d=1024, L=1)
    prompt = [5, 6]
    gamma = 3
    seq, length, stats, work = buffers(prompt, len(prompt) + 2, m.vocab, m.dim, gamma)
    bn.spec_rounds(m, gamma, 3, seq, length, stats, work)
    torch.cuda.synchronize()
    st = host(stats).tolist()
    n = int(length.item())
    assert n <= seq.numel()
    if st[3]:  # a round needed more room than was left: it wrote nothing
        assert st[1] == n - len(prompt)
