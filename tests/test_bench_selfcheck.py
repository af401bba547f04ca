"""The bench's self-check (CPU): the comparison that its oracle leg applies
to the GPU step's results accepts the oracle's own step and rejects a step
with one output element off by 1 %, one activation code changed or one
activation scale changed (the planted mistakes sit in copies of the oracle's
outputs)."""
import numpy as np
import pytest

import bench
import oracle


@pytest.fixture(scope="module")
def step():
    oracle.build()
    packed, acts = bench.oracle_step_inputs()
    outs = bench.oracle_step(packed, acts)
    results = {k: (y.astype(np.float32), q.copy(), xs.copy()) for k, (y, q, xs) in outs.items()}
    return outs, results


def test_every_group_and_pass_is_covered(step):
    outs, _ = step
    assert set(outs) == {(g, m) for g, _ in bench.LAYER_GROUPS for m in bench.DECODE_M}
    for (g, mode), (y, q, xs) in outs.items():
        N, K, ag = bench.group_shape(dict(bench.LAYER_GROUPS)[g])
        assert y.shape == (bench.DECODE_M[mode], N)
        assert q.shape == (bench.DECODE_M[mode], K)


def test_the_oracles_own_step_passes(step):
    outs, results = step
    assert bench.compare_step(outs, results) == "ok"


def _planted(results, key, what):
    r = dict(results)
    y, q, xs = (a.copy() for a in r[key])
    if what == "y":
        y[-1, -1] = y[-1, -1] * 1.01 + 1e-2 * float(np.sqrt(np.mean(y * y)))
    elif what == "code":
        q[0, 5] = q[0, 5] + 1 if q[0, 5] < 127 else q[0, 5] - 1
    else:
        xs.reshape(-1)[0] = np.nextafter(xs.reshape(-1)[0], np.float32(np.inf))
    r[key] = (y, q, xs)
    return r


@pytest.mark.parametrize("what", ["y", "code", "scale"])
def test_a_planted_mistake_fails(step, what):
    outs, results = step
    key = ("down", 1) if what == "y" else ("o", 0)
    msg = bench.compare_step(outs, _planted(results, key, what))
    assert msg.startswith("FAILED")
    assert ("down/target" if what == "y" else "o/draft") in msg
