"""Temperature-1 drafting and stochastic verification: CUDA path against the
sampling oracle (oracle/sampling_oracle.py) on identical inputs.

Integer decisions taken from floating point (a Gumbel-max draw, an
acceptance test) are compared bit-exactly except where the oracle's own
margin is within rounding of flipping: a top-2 gap of the Gumbel keys, or a
distance |log U - (log p - log q)|, below 1e-4 (fp32 on the device against
fp64 in the oracle).  Such rows are counted and must stay rare.
"""
import numpy as np
import pytest
import scipy.special
import torch

from oracle import sampling_oracle as S
from oracle import dflash_oracle as O
from block_diffusion_speculative_softmax_b200 import synth
from tests.gpu_common import TOL, need_gpu, oracle_for_workload, to_dev

pytestmark = pytest.mark.gpu
EPS_DECIDE = 1e-4


@pytest.fixture(scope="module")
def DF():
    need_gpu()
    from block_diffusion_speculative_softmax_b200 import dflash
    dflash.load()
    return dflash


def _cfg(V, B=16, dtype="bf16"):
    return synth.small_config("qwen3_4b", hidden=256, vocab=V, block=B, dtype=dtype)


def _oracle_gumbel(z, seed, offset, rows):
    """Tokens, logq and the top-2 gap of the Gumbel keys per row."""
    tok, logq = S.draft_sample(z, seed, offset, rows)
    gaps = []
    for m in range(z.shape[0]):
        k = np.sort(z[m] + S.gumbel(S.draft_uniforms(seed, offset, int(rows[m]), z.shape[1])))
        gaps.append(k[-1] - k[-2])
    return tok, logq, np.array(gaps)


@pytest.mark.parametrize("M,V,scale", [(64, 1000, 0.0), (40, 5000, 3.0), (16, 151936, 1.0),
                                       (9, 1001, 2.0)])
def test_sample_matches_oracle(DF, M, V, scale):
    # scale 0: all logits equal, the draw is the Gumbel noise alone (pins the
    # device's Philox counters, word choice and uniform mapping)
    rng = np.random.default_rng(M + V)
    z = (rng.standard_normal((M, V)) * scale).astype(np.float32)
    cc = DF.config_from(_cfg(V))
    zt = to_dev(z, torch.float32)
    tok = torch.empty(M, dtype=torch.int32, device="cuda")
    logq = torch.empty(M, dtype=torch.float32, device="cuda")
    lse = torch.empty(M, dtype=torch.float32, device="cuda")
    DF.dflash_sample(cc, zt, 12345678901, 3, tok, logq, lse)
    torch.cuda.synchronize()
    otok, ologq, gap = _oracle_gumbel(z.astype(np.float64), 12345678901, 3, np.arange(M))
    close = gap < EPS_DECIDE
    assert close.sum() <= 1
    got = tok.cpu().numpy()
    assert (got[~close] == otok[~close]).all(), np.nonzero(got != otok)
    np.testing.assert_allclose(lse.cpu().numpy(), scipy.special.logsumexp(z, axis=1),
                               rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(logq.cpu().numpy()[~close], ologq[~close], rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("R,B,V,sigma", [(64, 16, 3001, 0.7), (40, 32, 2048, 0.3),
                                         (50, 1, 777, 1.0), (8, 16, 151936, 0.5)])
def test_accept_stochastic_matches_oracle(DF, R, B, V, sigma):
    rng = np.random.default_rng(R * B + V)
    dl = (rng.standard_normal((R, B, V)) * 2.0).astype(np.float32)
    draft = np.zeros((R, B), dtype=np.int32)
    draft[:, 0] = rng.integers(0, V, R)
    for r in range(R):
        if B > 1:
            draft[r, 1:] = S.draft_sample(dl[r, 1:].astype(np.float64), 5, 0,
                                          np.arange(1, B) + r * B)[0]
    # target: the draft's next-slot logits plus noise; the last row unrelated
    zt = np.empty((R, B, V), dtype=np.float64)
    zt[:, :B - 1] = dl[:, 1:] + sigma * rng.standard_normal((R, B - 1, V))
    zt[:, B - 1] = 2.0 * rng.standard_normal((R, V))
    tl = scipy.special.log_softmax(zt, axis=-1).astype(np.float32)
    lse = scipy.special.logsumexp(dl.astype(np.float64), axis=-1).astype(np.float32)
    ws = DF.alloc_workspace(256 + 8 * R)
    n_acc = torch.empty(R, dtype=torch.int32, device="cuda")
    out = torch.empty(R, B, dtype=torch.int32, device="cuda")
    DF.dflash_accept_stochastic(to_dev(draft, torch.int32), to_dev(dl, torch.float32),
                                to_dev(lse, torch.float32), to_dev(tl, torch.float32), 99, 7,
                                n_acc, out, ws)
    torch.cuda.synchronize()
    # the oracle on the same inputs (its own logsumexp of the same fp32 logits)
    on, oout, info = S.stochastic_accept(draft, dl, tl, 99, 7)
    close = (info["margin"] < EPS_DECIDE) | (info["gap"] < EPS_DECIDE)
    assert close.sum() <= max(1, R // 20)
    gn, gout = n_acc.cpu().numpy(), out.cpu().numpy()
    np.testing.assert_array_equal(gn[~close], on[~close])
    np.testing.assert_array_equal(gout[~close], oout[~close])
    if B > 1:     # acceptance is exercised: neither all-pass nor all-fail
        assert 0 < on.mean() < B - 1


def _run_sampled_step(W, cfg, rng_seed=5):
    wl = W.Workload(cfg, seed=0, keep_host=True, sample=True, rng_seed=rng_seed)
    wl.draft()
    wl.check()
    return wl


@pytest.mark.parametrize("name", ["bf16", "fp32"])
def test_step_temperature_one_draft_and_verify(DF, name):
    from block_diffusion_speculative_softmax_b200 import workload as W
    if name == "bf16":
        cfg = synth.small_config("qwen3_4b", hidden=576, n_q_heads=8, n_kv_heads=2, head_dim=128,
                                 ffn=1000, n_draft_layers=2, n_target_layers=5, ctx_len=200,
                                 ctx_len_min=50, n_req=3, block=16, vocab=4099, dtype="bf16")
    else:
        cfg = synth.small_config("tiny", n_req=2, ctx_len=40, ctx_len_min=20)
    wl = _run_sampled_step(W, cfg)
    R, B = cfg.n_req, cfg.block
    reqs = list(range(R))
    blocks = [O.Block(r, [int(wl.anchors[r])] + [0] * (B - 1), 1) for r in reqs]
    _, _, keep = oracle_for_workload(wl, reqs, blocks)
    # draft logits against the oracle's
    z_or = np.stack([keep["logits"][i] for i in range(R)])            # [R][B][V]
    z_gpu = wl.buf.draft_logits.cpu().numpy().astype(np.float64)
    tol = TOL[cfg.dtype]
    scale = max(1.0, float(np.abs(z_or).max()))
    assert np.abs(z_gpu - z_or).max() / scale <= tol
    # drafted tokens: Gumbel draws over the oracle's logits; a slot whose
    # two best keys are within the logit tolerance may take either
    d_gpu = wl.buf.draft_tokens.cpu().numpy()
    for r in reqs:
        assert d_gpu[r, 0] == wl.anchors[r]
        rows = np.arange(1, B) + r * B
        otok, _, gap = _oracle_gumbel(z_or[r, 1:], wl.rng_seed, 0, rows)
        thr = 2 * tol * scale if cfg.dtype == "bf16" else EPS_DECIDE
        ok = (d_gpu[r, 1:] == otok) | (gap <= thr)
        assert ok.all(), (r, np.nonzero(~ok))
        if cfg.dtype == "fp32":
            assert (gap <= thr).sum() <= 1
    # the device's own logits feed the oracle's draw exactly
    for r in reqs:
        rows = np.arange(1, B) + r * B
        otok, _, gap = _oracle_gumbel(z_gpu[r, 1:], wl.rng_seed, 0, rows)
        close = gap < EPS_DECIDE
        assert (d_gpu[r, 1:][~close] == otok[~close]).all()
    # stochastic verification against a planted target, same inputs
    wl.plant_target_logp(sigma=0.5)
    wl.draft(verify=True)
    wl.check()
    dl = wl.buf.draft_logits.cpu().numpy()
    tl = wl.buf.target_logp.cpu().numpy()
    d = wl.buf.draft_tokens.cpu().numpy()
    on, oout, info = S.stochastic_accept(d, dl, tl, wl.rng_seed, 0)
    close = (info["margin"] < EPS_DECIDE) | (info["gap"] < EPS_DECIDE)
    gn, gout = wl.buf.n_acc.cpu().numpy(), wl.buf.out_tok.cpu().numpy()
    np.testing.assert_array_equal(gn[~close], on[~close])
    np.testing.assert_array_equal(gout[~close], oout[~close])
