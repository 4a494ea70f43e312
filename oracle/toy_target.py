"""A toy 2-layer causal target model for the greedy-losslessness check.

TEST INFRASTRUCTURE ONLY (see dflash_oracle.py for who may import it).

The DFlash summary (key contributions; methodology step 3) states that the
speculative loop emits exactly what the target would emit by itself.  To
test that claim to the bit, this target computes in integers, so scoring a
whole block in one pass and scoring one token at a time give identical
logits whatever the evaluation order:

    h0_t = E[tok_t]
    for l in 1, 2:
        s_t  = sum_{u <= t} h_{l-1,u}              (causal prefix sum)
        c_t  = floor(s_t / (t + 1))                (causal mean, floored)
        h_l,t = h_{l-1,t} + clip(floor((A_l h_{l-1,t} + C_l c_t) / 8), -6, 6)
    z_t  = W_out h_2,t ;  next token = lowest id among the maxima of z_t

It exposes T = 3 hidden-state snapshots per position (embedding output,
after layer 1, after layer 2), which the draft fuses as its context.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

SNAPSHOT_SCALE = 0.25  # snapshots are handed to the draft as float(h) * 0.25


def forward(weights: dict, tokens: np.ndarray
            ) -> Tuple[np.ndarray, np.ndarray]:
    """Run the toy target over ``tokens`` [n].

    Returns (snapshots float32 [n][3][H], next-token argmax int32 [n]);
    next[t] is the target's greedy prediction for position t + 1."""
    tok = np.asarray(tokens, dtype=np.int64)
    n = tok.shape[0]
    h = weights["E"][tok].astype(np.int64)                   # [n][H]
    snaps = [h.copy()]
    counts = np.arange(1, n + 1, dtype=np.int64)[:, None]
    for A, C in ((weights["A1"], weights["C1"]), (weights["A2"], weights["C2"])):
        s = np.cumsum(h, axis=0)
        c = np.floor_divide(s, counts)
        pre = h @ A.T + c @ C.T
        h = h + np.clip(np.floor_divide(pre, 8), -6, 6)
        snaps.append(h.copy())
    z = h @ weights["W_out"].T                                # [n][V]
    nxt = np.argmax(z, axis=1).astype(np.int32)
    st = np.stack(snaps, axis=1).astype(np.float32) * np.float32(SNAPSHOT_SCALE)
    return st, nxt


def greedy(weights: dict, prompt: np.ndarray, n_new: int) -> np.ndarray:
    """Plain one-token-at-a-time greedy decoding: ``n_new`` tokens."""
    seq = [int(t) for t in prompt]
    for _ in range(n_new):
        _, nxt = forward(weights, np.asarray(seq))
        seq.append(int(nxt[-1]))
    return np.asarray(seq[len(prompt):], dtype=np.int32)
