"""Scalar online-softmax recurrence and block merge (test infrastructure only).

Restated from "Attenzione: softmax online, riscalamento e memoria":

* section 2 (the invariant): after t keys keep m_t (prefix maximum), l_t (sum
  of exp(s_i - m_t)) and u_t (the same sum weighted by the values).  A new key
  (s, v) gives m' = max(m_t, s); the old l and u are both multiplied by
  exp(m_t - m'), then exp(s - m') and exp(s - m') * v are added.  The state
  starts at the first key: m = s_1, l = 1, u = v_1.  The output is o = u / l.
* section 3 (the counter-example): rescaling l but not u gives a wrong o.
* section 4 (merge): two disjoint key sets, each summarised by (m, l, u), are
  combined by rescaling both to max(m_A, m_B) and adding.

Everything is plain Python floats (IEEE double) and lists, with no vectorised
library code, so each line can be checked against the text by eye.
"""
from __future__ import annotations

import math


def stream_row(scores, values, wrong_rescale=False, trace=None):
    """Run the per-key recurrence over one row.

    scores: sequence of N >= 1 finite floats; values: N vectors (lists) of one length.
    wrong_rescale=True reproduces the section-3 mistake (l rescaled, u not).
    trace: optional list that receives (m, l, o) after every key.
    Returns (m, l, u) for the whole row.
    """
    if len(scores) == 0:
        raise ValueError("the recurrence needs at least one key")
    m = float(scores[0])
    l = 1.0
    u = [float(x) for x in values[0]]
    if trace is not None:
        trace.append((m, l, [x / l for x in u]))
    for s, v in zip(scores[1:], values[1:]):
        m_new = max(m, float(s))
        old = math.exp(m - m_new)
        new = math.exp(float(s) - m_new)
        l = l * old + new
        if wrong_rescale:
            u = [ui + new * float(vi) for ui, vi in zip(u, v)]
        else:
            u = [ui * old + new * float(vi) for ui, vi in zip(u, v)]
        m = m_new
        if trace is not None:
            trace.append((m, l, [x / l for x in u]))
    return m, l, u


def output(state):
    m, l, u = state
    return [x / l for x in u]


def merge(a, b):
    """Combine the summaries of two disjoint key sets (section 4)."""
    m_a, l_a, u_a = a
    m_b, l_b, u_b = b
    m = max(m_a, m_b)
    fa = math.exp(m_a - m)
    fb = math.exp(m_b - m)
    return m, l_a * fa + l_b * fb, [x * fa + y * fb for x, y in zip(u_a, u_b)]


def blocked_row(scores, values, block):
    """Summarise each block of ``block`` consecutive keys with the recurrence,
    then fold the block summaries together left to right with ``merge``."""
    state = None
    for lo in range(0, len(scores), block):
        part = stream_row(scores[lo:lo + block], values[lo:lo + block])
        state = part if state is None else merge(state, part)
    return output(state)


def materialised_row(scores, values):
    """All weights at once, relative to the global maximum (the stable
    materialised computation the section-4 experiment compares against)."""
    mu = max(scores)
    w = [math.exp(s - mu) for s in scores]
    total = sum(w)
    dv = len(values[0])
    return [sum(w[j] * values[j][c] for j in range(len(w))) / total for c in range(dv)]
