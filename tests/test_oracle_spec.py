"""CPU pins of the speculative-decoding oracle (oracle/spec.py).

The round's acceptance rule against hand-worked cases; the method's
invariant (speculative output == the target's greedy output) on small random
nested models; its special cases (a draft length of 0 is one greedy step;
with lo planes of all 8 the draft equals the target and every draft token is
accepted); argmax tie-breaking; the input embedding's rounding."""
import os

import numpy as np
import pytest

import oracle
from oracle import spec
from w8_quantized_linear_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "spec_accept_cases.txt")


def _cases():
    out = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        d, v, k, e = (f.split() for f in line.split(";"))
        out.append(([int(t) for t in d], [int(t) for t in v], int(k[0]), [int(t) for t in e]))
    return out


@pytest.mark.parametrize("draft,verify,k,emitted", _cases())
def test_accept_hand_worked(draft, verify, k, emitted):
    assert spec.accept(draft, verify) == (k, emitted)


def test_accept_rejects_bad_lengths():
    with pytest.raises(ValueError):
        spec.accept([1, 2], [1, 2])


def test_argmax_takes_the_lowest_of_equal_maxima():
    assert list(spec.argmax_lowest(np.array([[1.0, 3.0, 3.0, 2.0], [5.0, 5.0, 5.0, 5.0]]))) == [1, 0]


def test_embedding_is_the_rounded_exact_sum():
    E = np.zeros((3, 128), np.float16)
    E[0, 0], E[1, 0] = 1.0, 2.0          # 1 + 0.5 * 2 = 2 exactly
    E[0, 1], E[1, 1] = 2048.0, 2.0       # 2048 + 1 = 2049: a tie between 2048 and 2050 -> 2048
    E[0, 2], E[1, 2] = 2048.0, 6.0       # 2048 + 3 = 2051: tie between 2050 and 2052 -> 2052
    m = spec.Model(E, [], None)
    x = spec.embed_inputs(m, [0], [1])
    assert x[0, 0] == 2.0 and x[0, 1] == 2048.0 and x[0, 2] == 2052.0


def tiny_model(seed, V=64, d=128, L=2, lo_eight=False):
    def planes(rows, pid):
        uh = synth.nibbles(7000 + seed * 10 + pid, 0, rows, d)
        ul = np.full((rows, d), 8, np.uint8) if lo_eight else synth.nibbles(7000 + seed * 10 + pid, 1, rows, d)
        return oracle.pack_plane(uh), oracle.pack_plane(ul), synth.group_scales(7500 + seed * 10 + pid, rows, d)
    E = synth.normal(7900 + seed, 0, 0, V * d).reshape(V, d).astype(np.float16)
    return spec.Model(E, [planes(d, l) for l in range(L)], planes(V, 9))


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("gamma", [1, 2, 3])
def test_speculative_output_equals_target_greedy(seed, gamma):
    m = tiny_model(seed)
    prompt = [3, 17]
    s_spec, _ = spec.spec_decode(m, prompt, gamma, rounds=4)
    s_greedy = spec.greedy(m, prompt, len(s_spec) - len(prompt))
    assert s_spec == s_greedy


def test_draft_length_zero_is_one_greedy_step():
    m = tiny_model(4)
    s, k, draft, verify = spec.spec_round(m, [5, 6], 0)
    assert k == 0 and draft == [] and s == spec.greedy(m, [5, 6], 1)


def test_draft_equals_target_when_lo_is_eight():
    m = tiny_model(5, lo_eight=True)
    s, accepted = spec.spec_decode(m, [1, 2], gamma=3, rounds=3)
    assert accepted == 9 and len(s) == 2 + 3 * 4
    assert s == spec.greedy(m, [1, 2], 12, mode=oracle.DRAFT)
