"""CPU oracle for temperature-1 drafting and stochastic speculative acceptance.

TEST INFRASTRUCTURE ONLY (see dflash_oracle.py for who may import it).  The
product path never calls this module and it imports nothing from the product
package.

What it computes (plain NumPy float64, in the pages' order):

* DFlash summary, methodology step 3: the target checks the drafted block
  with the standard speculative acceptance test, a comparison of log
  probabilities; accepted tokens are emitted at once and the first rejected
  position is filled by the target's own generation.
* DFLARE summary, section 4: the same loop is also run with stochastic
  decoding at temperature 1.

Readings where the pages are silent:

* The draft at temperature 1 samples every block slot from its own softmax
  q_j independently (the block is one parallel pass), by the Gumbel-max
  rule: token = argmax_v (z_v + G_v), G_v = -log(-log U_v), U_v uniform.
* Slot j (1 <= j <= B-1) is accepted when log U_j < log p_j(d_j) -
  log q_j(d_j), i.e. U_j < p/q, with p_j the target's distribution for slot
  j (after reading slots 0..j-1) -- the standard test written as the
  log-probability comparison the page names.
* "The target's own generation" at the first rejected slot is read as the
  draw from the residual distribution norm(max(0, p_j - q_j)): that is the
  choice under which the emitted tokens follow the target's distribution
  exactly (the losslessness the pages claim); when every drafted slot is
  accepted, one more token is drawn from the target's distribution for the
  slot after the block.  Both draws use the Gumbel-max rule.
* Every uniform is a counter-based Philox4x32-10 draw (Salmon, Moraes, Dror
  and Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011), so the
  CUDA path and this oracle draw identical numbers from (seed, counter).
  Counter layout, words (c0, c1, c2, c3) and key (seed low, seed high):
    draft Gumbel of row m, vocabulary id v: (v >> 2, m, offset, DRAFT),
        word v & 3;
    acceptance uniform of block b, slot j:  (j, b, offset, ACCEPT), word 0;
    residual / bonus Gumbel of block b at emitted slot j, id v:
        (v >> 2, b * 64 + j, offset, RESID), word v & 3.
  A word x becomes U = (floor(x / 2^9) + 1/2) / 2^23, an odd multiple of
  2^-24 in (0, 1), exact in fp32.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

__all__ = ["philox4x32_10", "uniform_from_word", "gumbel", "draft_uniforms",
           "draft_sample", "accept_uniform", "resid_uniforms", "stochastic_accept",
           "PURPOSE_DRAFT", "PURPOSE_ACCEPT", "PURPOSE_RESID"]

# Purpose tags (the fourth counter word): ASCII "DRFT", "ACPT", "RESD".
PURPOSE_DRAFT = 0x44524654
PURPOSE_ACCEPT = 0x41435054
PURPOSE_RESID = 0x52455344

_M0, _M1 = np.uint64(0xD2511F53), np.uint64(0xCD9E8D57)
_W0, _W1 = np.uint64(0x9E3779B9), np.uint64(0xBB67AE85)
_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr: np.ndarray, key: np.ndarray) -> np.ndarray:
    """Philox4x32 with 10 rounds (Salmon et al., SC 2011, section 5).

    ctr: uint32 [..., 4]; key: uint32 [..., 2] (broadcast against ctr).
    One round multiplies c0 by M0 and c2 by M1 (64-bit products split into
    hi/lo 32-bit halves) and outputs (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0);
    the key is bumped by the Weyl constants (W0, W1) between rounds."""
    c = np.asarray(ctr, dtype=np.uint32).astype(np.uint64)
    k = np.broadcast_to(np.asarray(key, dtype=np.uint32).astype(np.uint64),
                        c.shape[:-1] + (2,)).copy()
    c0, c1, c2, c3 = c[..., 0], c[..., 1], c[..., 2], c[..., 3]
    k0, k1 = k[..., 0], k[..., 1]
    for r in range(10):
        if r:
            k0 = (k0 + _W0) & _MASK32
            k1 = (k1 + _W1) & _MASK32
        p0 = _M0 * c0
        p1 = _M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def _key(seed: int) -> np.ndarray:
    s = int(seed) & 0xFFFFFFFFFFFFFFFF
    return np.array([s & 0xFFFFFFFF, s >> 32], dtype=np.uint32)


def uniform_from_word(x: np.ndarray) -> np.ndarray:
    """32-bit word -> U = (floor(x / 2^9) + 1/2) / 2^23 in (0, 1)."""
    x = np.asarray(x, dtype=np.uint32)
    return ((x >> np.uint32(9)).astype(np.float64) + 0.5) * 2.0 ** -23


def gumbel(u: np.ndarray) -> np.ndarray:
    """Standard Gumbel variate from a uniform: -log(-log U)."""
    return -np.log(-np.log(np.asarray(u, dtype=np.float64)))


def _vocab_uniforms(seed: int, c1: int, offset: int, purpose: int, V: int) -> np.ndarray:
    v = np.arange(V, dtype=np.uint64)
    ctr = np.zeros((V, 4), dtype=np.uint32)
    ctr[:, 0] = (v >> np.uint64(2)).astype(np.uint32)
    ctr[:, 1] = np.uint32(c1 & 0xFFFFFFFF)
    ctr[:, 2] = np.uint32(offset & 0xFFFFFFFF)
    ctr[:, 3] = np.uint32(purpose)
    words = philox4x32_10(ctr, _key(seed))
    return uniform_from_word(words[np.arange(V), (v & np.uint64(3)).astype(np.int64)])


def draft_uniforms(seed: int, offset: int, row: int, V: int) -> np.ndarray:
    """U_v of the draft's Gumbel noise for token row ``row``, v < V."""
    return _vocab_uniforms(seed, row, offset, PURPOSE_DRAFT, V)


def resid_uniforms(seed: int, offset: int, block: int, slot: int, V: int) -> np.ndarray:
    """U_v of the residual / bonus draw of block ``block`` at slot ``slot``."""
    return _vocab_uniforms(seed, block * 64 + slot, offset, PURPOSE_RESID, V)


def accept_uniform(seed: int, offset: int, block: int, slot: int) -> float:
    """U_j of the acceptance test of block ``block`` at slot ``slot``."""
    ctr = np.array([[slot, block, offset & 0xFFFFFFFF, PURPOSE_ACCEPT]], dtype=np.uint32)
    return float(uniform_from_word(philox4x32_10(ctr, _key(seed))[0, 0]))


def _lse(z: np.ndarray) -> float:
    m = float(np.max(z))
    return m + float(np.log(np.sum(np.exp(z - m))))


def draft_sample(z: np.ndarray, seed: int, offset: int, rows: np.ndarray
                 ) -> Tuple[np.ndarray, np.ndarray]:
    """Temperature-1 draft tokens by the Gumbel-max rule.

    z [M][V] draft logits of token rows ``rows`` (their row ids in the
    batch, which select the noise).  tok[m] = argmax_v (z[m, v] + G[m, v])
    (lowest id on an exact tie); logq[m] = z[m, tok] - logsumexp(z[m]), the
    draft's log probability of its own token.  Returns (tok int32, logq)."""
    z = np.asarray(z, dtype=np.float64)
    M, V = z.shape
    tok = np.empty(M, dtype=np.int32)
    logq = np.empty(M, dtype=np.float64)
    for m in range(M):
        g = gumbel(draft_uniforms(seed, offset, int(rows[m]), V))
        t = int(np.argmax(z[m] + g))
        tok[m] = t
        logq[m] = z[m, t] - _lse(z[m])
    return tok, logq


def stochastic_accept(draft: np.ndarray, draft_logits: np.ndarray,
                      target_logp: np.ndarray, seed: int, offset: int
                      ) -> Tuple[np.ndarray, np.ndarray, dict]:
    """Speculative acceptance at temperature 1, one candidate per request.

    draft [R][B] (slot 0 = anchor, slots 1..B-1 drafted); draft_logits
    [R][B][V] (the draft's logits per slot, softmax = q_j); target_logp
    [R][B][V] with target_logp[r, j] = log p(. | slots 0..j), the target's
    distribution for slot j+1 (row B-1 is the slot after the block).
    For j = 1 .. B-1: accept d_j while log U_j < log p_j(d_j) - log q_j(d_j).
    At the first rejected slot j the emitted token is drawn from
    norm(max(0, p_j - q_j)); when all B-1 are accepted, from p_B.
    Returns (n_acc [R], out_tok [R][B]: d[1..n], drawn token, then -1, info)
    with info["margin"][r] the smallest |log U_j - (log p - log q)| among the
    tested slots and info["gap"][r] the top-2 gap of the final Gumbel draw
    (how close each integer decision came to flipping)."""
    draft = np.asarray(draft)
    dl = np.asarray(draft_logits, dtype=np.float64)
    tl = np.asarray(target_logp, dtype=np.float64)
    R, B, V = dl.shape
    n_acc = np.zeros(R, dtype=np.int32)
    out = np.full((R, B), -1, dtype=np.int32)
    margin = np.full(R, np.inf)
    gap = np.full(R, np.inf)
    for r in range(R):
        n = 0
        for j in range(1, B):
            d = int(draft[r, j])
            lq = dl[r, j, d] - _lse(dl[r, j])
            lp = tl[r, j - 1, d]
            lu = float(np.log(accept_uniform(seed, offset, r, j)))
            margin[r] = min(margin[r], abs(lu - (lp - lq)))
            if lu < lp - lq:
                n += 1
            else:
                break
        slot = n + 1
        g = gumbel(resid_uniforms(seed, offset, r, slot, V))
        if slot < B:
            p = np.exp(tl[r, n])
            q = np.exp(dl[r, slot] - _lse(dl[r, slot]))
            res = np.maximum(0.0, p - q)
            with np.errstate(divide="ignore"):
                key = np.where(res > 0.0, np.log(res) + g, -np.inf)
        else:
            key = tl[r, B - 1] + g
        t = int(np.argmax(key))
        srt = np.sort(key)
        gap[r] = srt[-1] - srt[-2] if V > 1 else np.inf
        n_acc[r] = n
        out[r, :n] = draft[r, 1:n + 1]
        out[r, n] = t
    return n_acc, out, {"margin": margin, "gap": gap}
