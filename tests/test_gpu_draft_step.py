"""End-to-end parity of dflash_draft_step (+ verification) with the oracle.

Small shapes span several GEMM tiles, ragged tails (hidden, FFN, vocab and
context lengths that are not tile multiples), several requests and D2SD
candidates.  The five named workloads run at full size in the launch
configuration the benchmark times; the oracle checks every block it can
finish in seconds (for the 32-request serving batch, a sample of requests).
"""
import numpy as np
import pytest
import torch

from oracle import dflash_oracle as O
from block_diffusion_speculative_softmax_b200 import synth
from tests.gpu_common import TOL, check_draft, need_gpu, oracle_for_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def W():
    need_gpu()
    from block_diffusion_speculative_softmax_b200 import workload
    return workload


def _blocks_pass1(wl, reqs):
    B = wl.cfg.block
    return [O.Block(r, [int(wl.anchors[r])] + [0] * (B - 1), 1) for r in reqs]


def _run_pass1(W, cfg, reqs=None, mode="full", **kw):
    wl = W.Workload(cfg, seed=0, keep_host=True, mode=mode, **kw)
    if mode == "steady":
        # fill the caches with every row first, then recompute the last rows
        full = W.Workload(cfg, seed=0, host_weights=wl.host_weights, ctx_lens=wl.ctx_lens)
        full.draft()
        for i in range(cfg.n_draft_layers):
            wl.buf.k_cache[i].copy_(full.buf.k_cache[i])
            wl.buf.v_cache[i].copy_(full.buf.v_cache[i])
        # poison the rows that the steady step must recompute
        o = 0
        for L in wl.ctx_lens:
            for i in range(cfg.n_draft_layers):
                wl.buf.k_cache[i][o + L - wl.n_new_rows:o + L] = 7.0
                wl.buf.v_cache[i][o + L - wl.n_new_rows:o + L] = -7.0
            o += L
    wl.draft()
    wl.check()
    reqs = list(range(cfg.n_req)) if reqs is None else reqs
    blocks = _blocks_pass1(wl, reqs)
    ot, om, keep = oracle_for_workload(wl, reqs, blocks)
    gt = wl.buf.draft_tokens.cpu().numpy()[reqs]
    gm = wl.buf.max_logit.cpu().numpy()[reqs]
    rep = check_draft(wl, gt, gm, ot, om, keep, blocks, cfg.name)
    return wl, rep, ot


def _verify_planted(wl):
    """Plant targets against the GPU's own tokens, run the step again with
    verification and compare the accept outputs with the oracle's accept on
    identical inputs; the planted lengths must come back exactly."""
    n_pl = wl.plant_targets()
    wl.step(verify=True)
    wl.check()
    fb = wl.final_buf
    R, K, B = wl.R, wl.K, wl.cfg.block
    d = fb.draft_tokens.cpu().numpy().reshape(R, K, B)
    t = fb.target_tokens.cpu().numpy().reshape(R, K, B)
    on, obk, oout = O.accept(d, t)
    np.testing.assert_array_equal(fb.n_acc.cpu().numpy(), on)
    np.testing.assert_array_equal(fb.best_k.cpu().numpy(), obk)
    np.testing.assert_array_equal(fb.out_tok.cpu().numpy(), oout)
    if K == 1:      # the planted accept lengths come back exactly
        np.testing.assert_array_equal(on, n_pl)
    return n_pl, on


# ------------------------------------------------------------------ small shapes
SMALL = {
    "bf16_ragged": dict(hidden=576, n_q_heads=8, n_kv_heads=2, head_dim=128, ffn=1000,
                        n_draft_layers=3, n_target_layers=5, ctx_len=300, block=16,
                        vocab=5017, dtype="bf16"),
    "bf16_multi_req": dict(hidden=512, n_q_heads=16, n_kv_heads=2, head_dim=64, ffn=704,
                           n_draft_layers=2, n_target_layers=9, ctx_len=200, ctx_len_min=1,
                           n_req=5, block=16, vocab=3001, dtype="bf16"),
    "fp32_b1": dict(hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=512,
                    n_draft_layers=2, n_target_layers=3, ctx_len=40, block=1, vocab=700,
                    dtype="fp32"),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_shapes(W, name):
    cfg = synth.small_config("qwen3_4b", **SMALL[name])
    wl, rep, _ = _run_pass1(W, cfg)
    if cfg.block > 1:
        _verify_planted(wl)


@pytest.mark.parametrize("name", ["bf16_ragged", "bf16_multi_req", "fp32_b1"])
def test_small_dflash_fc_variant(W, name):
    # DFlash baseline: one FC-fused context for every layer, context and block
    # sharing the K/V projections (DFLARE summary, section 1 item 1, 2.2)
    cfg = synth.small_config("qwen3_4b", **SMALL[name])
    hw = synth.make_weights(cfg, 0, separate_kv=False)
    hw.update(synth.make_fc_weights(cfg, 0))
    wl, rep, _ = _run_pass1(W, cfg, host_weights=hw)
    if cfg.block > 1:
        _verify_planted(wl)


def test_small_steady_state_matches_full(W):
    cfg = synth.small_config("qwen3_4b", **SMALL["bf16_multi_req"])
    _run_pass1(W, cfg, mode="steady", steady_new_rows=7)


@pytest.mark.parametrize("conf_source", ["draft", "synthetic"])
def test_small_d2sd(W, conf_source):
    cfg = synth.small_config("d2sd_gptoss", hidden=640, n_q_heads=16, n_kv_heads=2, head_dim=64,
                             ffn=704, n_draft_layers=2, n_target_layers=5, ctx_len=150,
                             block=16, vocab=3001, n_req=3, n_cand=4)
    _d2sd(W, cfg, reqs=None, ctx_lens=[150, 77, 260], conf_source=conf_source)


def _d2sd(W, cfg, reqs=None, ctx_lens=None, conf_source="synthetic"):
    wl = W.Workload(cfg, seed=0, keep_host=True, ctx_lens=ctx_lens, conf_source=conf_source)
    reqs = list(range(cfg.n_req)) if reqs is None else reqs
    wl.draft()
    wl.check()
    blocks1 = _blocks_pass1(wl, reqs)
    ot1, om1, keep1 = oracle_for_workload(wl, reqs, blocks1)
    check_draft(wl, wl.buf.draft_tokens.cpu().numpy()[reqs],
                wl.buf.max_logit.cpu().numpy()[reqs], ot1, om1, keep1, blocks1, "d2sd pass 1")
    if conf_source == "draft":
        # the first pass's confidence against the oracle's softmax of its logits
        # (conf = exp(z_max - lse): logits within d of the oracle's move it
        # by a factor within exp(+-2d), d taken from the logit tolerance)
        z = np.stack([keep1["logits"][i] for i in range(len(blocks1))])
        oc = np.stack([O.draft_confidence(zi) for zi in z])[:, 1:]
        gc = wl.buf.confidence.cpu().numpy()[reqs][:, 1:].astype(np.float64)
        d = TOL[cfg.dtype] * max(1.0, float(np.abs(z).max()))
        assert np.all(np.abs(np.log(gc / oc)) <= 2 * d), np.abs(np.log(gc / oc)).max()
    # cuts on the GPU from the GPU's base tokens must equal the oracle's cuts
    # on the same base tokens
    wl.candidates()
    base = wl.buf.draft_tokens.cpu().numpy()
    conf = wl.conf.cpu().numpy()
    okl, ocand = O.d2sd_candidates(base, conf, cfg.n_cand, cfg.mask_token_id)
    np.testing.assert_array_equal(wl.buf2.known_len.cpu().numpy(), okl)
    np.testing.assert_array_equal(wl.buf2.block_tokens.cpu().numpy(), ocand)
    # pass 2 over the cached context
    wl.redraft()
    wl.check()
    K = cfg.n_cand
    blocks2 = [O.Block(r, ocand[r * K + k], int(okl[r * K + k])) for r in reqs for k in range(K)]
    ot2, om2, keep2 = oracle_for_workload(wl, reqs, blocks2)
    rows = [r * K + k for r in reqs for k in range(K)]
    check_draft(wl, wl.buf2.draft_tokens.cpu().numpy()[rows],
                wl.buf2.max_logit.cpu().numpy()[rows], ot2, om2, keep2, blocks2, "d2sd pass 2")
    _verify_planted(wl)


# ------------------------------------------------------------------ full-size workloads
def test_full_tiny_fp32(W):
    cfg = synth.get_config("tiny")
    wl, rep, _ = _run_pass1(W, cfg)
    assert rep["near_tie"] == 0
    _verify_planted(wl)


def test_full_qwen3_4b(W):
    wl, rep, _ = _run_pass1(W, synth.get_config("qwen3_4b"))
    _verify_planted(wl)


def test_full_qwen3_4b_steady(W):
    _run_pass1(W, synth.get_config("qwen3_4b"), mode="steady")


def test_full_qwen3_8b_dflare(W):
    wl, rep, _ = _run_pass1(W, synth.get_config("qwen3_8b_dflare"))
    _verify_planted(wl)


def test_full_serving32_sampled(W):
    cfg = synth.get_config("serving32")
    lens = synth.ctx_lengths(cfg, 0)
    order = np.argsort(lens)
    reqs = sorted({int(order[0]), int(order[len(order) // 2]), int(order[-1])})
    wl, rep, _ = _run_pass1(W, cfg, reqs=reqs)
    _verify_planted(wl)


def test_full_d2sd_gptoss_sampled(W):
    _d2sd(W, synth.get_config("d2sd_gptoss"), reqs=[0, 5])


# ------------------------------------------------------------------ graph capture
def test_draft_step_replays_in_cuda_graph(W):
    cfg = synth.small_config("qwen3_4b", **SMALL["bf16_ragged"])
    wl = W.Workload(cfg, seed=0)
    wl.plant_targets()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        wl.step(verify=True)      # warm-up outside capture
    torch.cuda.synchronize()
    ref = wl.buf.out_tok.clone(), wl.buf.draft_tokens.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        wl.step(verify=True)
    wl.buf.out_tok.zero_()
    wl.buf.draft_tokens.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(wl.buf.out_tok, ref[0])
    assert torch.equal(wl.buf.draft_tokens, ref[1])
    wl.check()

