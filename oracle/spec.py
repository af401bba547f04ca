"""Speculative decoding with the nested weights: the CPU oracle.

TEST INFRASTRUCTURE ONLY (see the package docstring): only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may use it.

BitNest-Llama-3-8B model card, opening paragraph: the W4A8 draft (hi plane)
proposes tokens, the W8A8 target (both planes) verifies every one of them, so
the output is exactly the target's greedy output; model table row "Default
draft length": gamma = 3.  The pages give no model to decode with; this
module's reading is a small synthetic one built from the nested linear layer
(the oracle's ``quantize`` and ``linear``):

  input at position p : x0 = fp16(E[t_p] + 0.5 E[t_{p-1}])   (t_{-1} := t_0)
  layer l             : x_{l+1} = fp16(tanh(W_l x_l)),  W_l nested [d, d]
  head                : logits = W_head x_L,             W_head nested [V, d]
  next token          : argmax(logits), the lowest index among equal maxima

and the speculative round on it:

  draft  : gamma tokens, one at a time, with the draft weights (M = 1);
  verify : the target on the gamma + 1 positions at once (M = gamma + 1);
  accept : the longest prefix of draft tokens the target agrees with, then
           the target's own token at the first disagreement (or after the
           last draft token): 1 .. gamma + 1 tokens per round.

Everything is evaluated in the oracle's precision: activations quantised in
fp32 (per token), the layer in fp64, tanh in fp64 rounded to fp16.
"""
from __future__ import annotations

import numpy as np

from . import DRAFT, TARGET, linear, quantize


class Model:
    """The synthetic model's tensors on the host.

    embed : fp16 [V, d];  layers : list of (hi, lo, scale) with planes uint8
    [d, d/2] and fp16 scales [d, d/128];  head : (hi, lo, scale) of [V, d]."""

    def __init__(self, embed, layers, head):
        self.embed = np.asarray(embed, np.float16)
        self.layers = list(layers)
        self.head = head
        self.vocab, self.dim = self.embed.shape


def embed_inputs(model: Model, cur, prev) -> np.ndarray:
    """fp16 [M, d]: E[cur] + 0.5 E[prev] (exact in fp64, then rounded)."""
    e = model.embed.astype(np.float64)
    cur = np.asarray(cur, np.int64)
    prev = np.asarray(prev, np.int64)
    return (e[cur] + 0.5 * e[prev]).astype(np.float16)


def forward_logits(model: Model, mode: int, cur, prev) -> np.ndarray:
    """fp64 logits [M, V] of the positions whose tokens are `cur` (and their
    predecessors `prev`), with the draft or the target weights."""
    d = model.dim
    x = embed_inputs(model, cur, prev)
    for hi, lo, s in model.layers:
        q, xs = quantize(x, 0)
        y = linear(mode, hi, lo if mode == TARGET else None, s, q, xs, d)
        x = np.tanh(y).astype(np.float16)
    hi, lo, s = model.head
    q, xs = quantize(x, 0)
    return linear(mode, hi, lo if mode == TARGET else None, s, q, xs, d)


def argmax_lowest(logits: np.ndarray) -> np.ndarray:
    """Row-wise argmax; np.argmax returns the first (lowest) maximal index."""
    return np.argmax(np.asarray(logits), axis=-1).astype(np.int64)


def _cur_prev(tokens, p):
    return tokens[p], tokens[max(p - 1, 0)]


def greedy(model: Model, seq, steps: int, mode: int = TARGET) -> list:
    """`steps` tokens appended one at a time by argmax of the model."""
    s = list(int(t) for t in seq)
    for _ in range(steps):
        c, p = _cur_prev(s, len(s) - 1)
        s.append(int(argmax_lowest(forward_logits(model, mode, [c], [p]))[0]))
    return s


def accept(draft, verify) -> tuple:
    """(k, emitted): k leading draft tokens the target agrees with, then the
    target's token at position k.  len(verify) == len(draft) + 1."""
    draft = [int(t) for t in draft]
    verify = [int(t) for t in verify]
    if len(verify) != len(draft) + 1:
        raise ValueError("verify needs one more token than draft")
    k = 0
    while k < len(draft) and draft[k] == verify[k]:
        k += 1
    return k, draft[:k] + [verify[k]]


def spec_round(model: Model, seq, gamma: int) -> tuple:
    """One round on `seq`: (new sequence, k accepted, draft, verify)."""
    s = list(int(t) for t in seq)
    n = len(s)
    ext = list(s)
    draft = []
    for _ in range(gamma):  # the draft, token by token
        c, p = _cur_prev(ext, len(ext) - 1)
        t = int(argmax_lowest(forward_logits(model, DRAFT, [c], [p]))[0])
        draft.append(t)
        ext.append(t)
    # the target on the gamma + 1 positions n - 1 .. n - 1 + gamma at once
    pos = [n - 1 + j for j in range(gamma + 1)]
    cur = [ext[q] for q in pos]
    prev = [ext[max(q - 1, 0)] for q in pos]
    verify = [int(t) for t in argmax_lowest(forward_logits(model, TARGET, cur, prev))]
    k, emitted = accept(draft, verify)
    return s + emitted, k, draft, verify


def spec_decode(model: Model, seq, gamma: int, rounds: int) -> tuple:
    """`rounds` speculative rounds: (sequence, accepted draft tokens)."""
    s = list(int(t) for t in seq)
    accepted = 0
    for _ in range(rounds):
        s, k, _, _ = spec_round(model, s, gamma)
        accepted += k
    return s, accepted
