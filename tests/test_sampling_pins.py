"""Pins of the temperature-1 sampling oracle (oracle/sampling_oracle.py)
against things other than itself: the published Philox4x32-10 known-answer
values, closed forms of the uniform mapping, the Gumbel-max theorem (draws
follow softmax(z)), the special cases of the acceptance test, and the
losslessness of the speculative loop -- the emitted tokens follow the
target's own distribution (DFlash summary, key contributions and
methodology step 3; DFLARE summary, section 4, temperature 1) -- checked
against the exact target distribution by a chi-square test at fixed seeds.
A wrong residual, a flipped comparison or a mis-indexed target row biases
that distribution far beyond the test's threshold."""
import json
import os

import numpy as np
import scipy.special
import scipy.stats

from oracle import sampling_oracle as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_philox_known_answers():
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        ctr = np.array([[int(x, 16) for x in c["ctr"]]], dtype=np.uint32)
        key = np.array([int(x, 16) for x in c["key"]], dtype=np.uint32)
        got = S.philox4x32_10(ctr, key)[0]
        assert ["%08x" % w for w in got] == c["out"]


def test_uniform_mapping_closed_form():
    x = np.array([0, 1, 511, 512, 0xFFFFFFFF, 0x80000000], dtype=np.uint32)
    u = S.uniform_from_word(x)
    np.testing.assert_array_equal(u, [2.0 ** -24, 2.0 ** -24, 2.0 ** -24, 3 * 2.0 ** -24,
                                      1 - 2.0 ** -24, 0.5 + 2.0 ** -24])
    assert np.all(u.astype(np.float32).astype(np.float64) == u)   # exact in fp32
    assert np.all((u > 0) & (u < 1))


def test_vocab_uniforms_are_uniform_and_distinct_per_row():
    V = 1 << 15
    a = S.draft_uniforms(7, 0, 3, V)
    b = S.draft_uniforms(7, 0, 4, V)
    c = S.draft_uniforms(7, 1, 3, V)
    counts = np.histogram(a, bins=64, range=(0, 1))[0]
    assert scipy.stats.chisquare(counts).pvalue > 1e-3
    assert not np.array_equal(a, b) and not np.array_equal(a, c)
    assert abs(np.corrcoef(a, b)[0, 1]) < 0.05
    # the Gumbel transform has the Gumbel law's mean (Euler's constant)
    assert abs(S.gumbel(a).mean() - np.euler_gamma) < 0.03


def test_gumbel_max_draws_follow_softmax():
    rng = np.random.default_rng(41)
    V, n = 6, 30000
    z = rng.standard_normal(V) * 1.5
    tok, logq = S.draft_sample(np.tile(z, (n, 1)), seed=11, offset=2, rows=np.arange(n))
    p = scipy.special.softmax(z)
    counts = np.bincount(tok, minlength=V)
    assert scipy.stats.chisquare(counts, n * p).pvalue > 1e-3
    np.testing.assert_allclose(logq, np.log(p[tok]), rtol=1e-12, atol=1e-12)


def test_accept_special_cases():
    rng = np.random.default_rng(42)
    R, B, V = 40, 6, 9
    dl = rng.standard_normal((R, B, V))
    d = rng.integers(0, V, size=(R, B))
    # target == draft distribution: p/q = 1 > U, every drafted slot passes,
    # and the bonus comes from the target's row for the slot after the block
    tl = np.zeros_like(dl)
    tl[:, :B - 1] = scipy.special.log_softmax(dl[:, 1:], axis=-1)
    tl[:, B - 1] = scipy.special.log_softmax(rng.standard_normal((R, V)), axis=-1)
    n, out, _ = S.stochastic_accept(d, dl, tl, seed=3, offset=0)
    assert (n == B - 1).all()
    np.testing.assert_array_equal(out[:, :B - 1], d[:, 1:])
    # the target gives the drafted token of slot 1 probability 0: slot 1 is
    # always rejected and the drawn token is never that token
    tl2 = tl.copy()
    tl2[np.arange(R), 0, d[:, 1]] = -np.inf
    tl2[:, 0] = tl2[:, 0] - scipy.special.logsumexp(tl2[:, 0], axis=-1, keepdims=True)
    n2, out2, _ = S.stochastic_accept(d, dl, tl2, seed=3, offset=0)
    assert (n2 == 0).all()
    assert (out2[:, 0] != d[:, 1]).all()
    assert (out2[:, 1:] == -1).all()


def _markov(V, seed):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((V, V)) * 1.5            # p(next | last) = softmax(A[last])
    Zd = rng.standard_normal((8, V)) * 1.5           # the draft's per-slot logits
    return scipy.special.log_softmax(A, axis=1), Zd


def speculative_two_tokens(logP, Zd, B, anchor, trial):
    """First two tokens emitted by the temperature-1 speculative loop:
    draft every slot from its own q_j, score the drafted prefix with the
    Markov target, accept / resample, roll forward until two tokens exist."""
    V = logP.shape[0]
    emitted = []
    last = anchor
    step = 0
    while len(emitted) < 2:
        dl = np.zeros((B, V))
        dl[1:] = Zd[1:B]
        rows = np.arange(B) + trial * B
        d = np.zeros(B, dtype=np.int64)
        d[0] = last
        d[1:] = S.draft_sample(dl[1:], seed=trial, offset=step, rows=rows[1:])[0]
        tl = logP[d]                                   # tl[j] = log p(. | d[0..j])
        n, out, _ = S.stochastic_accept(d[None], dl[None], tl[None], seed=trial,
                                        offset=step)
        emitted += [int(t) for t in out[0, :n[0] + 1]]
        last = emitted[-1]
        step += 1
    return emitted[0], emitted[1]


def test_speculative_loop_emits_the_target_distribution():
    V, B, a0, trials = 4, 4, 1, 12000
    logP, Zd = _markov(V, 43)
    counts = np.zeros((V, V))
    for t in range(trials):
        t1, t2 = speculative_two_tokens(logP, Zd, B, a0, t)
        counts[t1, t2] += 1
    P = np.exp(logP)
    exact = P[a0][:, None] * P                         # p(t1 | a0) p(t2 | t1)
    res = scipy.stats.chisquare(counts.ravel(), trials * exact.ravel())
    assert res.pvalue > 1e-4, res
