"""Oracle of the draft-length policy -- TEST INFRASTRUCTURE ONLY.

Expected tokens per decode step by explicit enumeration: every pattern of
accept / reject outcomes of the k tested slots (each accepted independently
with probability alpha) is listed with its probability; for each the step's
accept length (leading accepts), its newly emitted tokens and the next step's
state (pre-accepted slot 1 or not) are read off the decode-step rules
("TiDAR: Think in Diffusion, Talk in Autoregression", awesome-system-papers
summary, "并行 self-speculative 生成 (§3.2)": drafts verified by rejection
sampling, a rejected slot replaced by a residual draw; the resampled token is
the next step's pre-accepted slot 1, already emitted).  The long-run share of
steps in each state of that two-state chain (its stationary distribution, from
the balance equations) weights the per-state expectations.
The choice of draft length is a brute-force argmax of tokens per microsecond
("局限与 Future Work", Future work 2: fit the draft block to the GPU).
"""
from __future__ import annotations

import itertools

import numpy as np


def step_outcomes(k: int, alpha: float, pre: int):
    """[(probability, new tokens, next pre)] over every accept pattern of one step in state `pre`."""
    out = []
    for pattern in itertools.product((True, False), repeat=k):
        if pre and not pattern[0]:
            continue  # slot 1 is pre-accepted: it is not tested
        prob = 1.0
        for i, acc in enumerate(pattern):
            if pre and i == 0:
                continue
            prob *= alpha if acc else (1.0 - alpha)
        j = 0
        while j < k and pattern[j]:
            j += 1
        new = (j - pre) + (1 if j < k else 0)  # accepted drafts not yet emitted, then the resampled token
        out.append((prob, new, 1 if j < k else 0))
    return out


def expected_tokens_per_step(k: int, alpha: float) -> float:
    trans = [[0.0, 0.0], [0.0, 0.0]]
    reward = [0.0, 0.0]
    for pre in (0, 1):
        for prob, new, nxt in step_outcomes(k, alpha, pre):
            trans[pre][nxt] += prob
            reward[pre] += prob * new
    # long-run share of steps in each state: the stationary distribution of the chain, pi = pi T with
    # pi_0 + pi_1 = 1 (unique: every state reaches the other unless alpha = 1, where state 1 is never entered)
    if trans[0][1] == 0.0:
        pi = [1.0, 0.0]
    else:
        a = np.array([[trans[0][0] - 1.0, trans[1][0]], [1.0, 1.0]])
        pi = np.linalg.solve(a, np.array([0.0, 1.0]))
    return float(pi[0] * reward[0] + pi[1] * reward[1])


def pick_draft_length(step_us, alpha: float):
    """(k, tokens per microsecond): the k = 1..len(step_us) with the most tokens per microsecond (shorter on
    ties), over the entries with a positive finite latency."""
    best_k, best = 0, -1.0
    for k, t in enumerate(step_us, start=1):
        if not (t > 0.0 and t != float("inf")):
            continue
        r = expected_tokens_per_step(k, alpha) / t
        if r > best:
            best_k, best = k, r
    return best_k, (best if best_k else 0.0)
