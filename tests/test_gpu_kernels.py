"""Per-entry-point parity: each C-ABI call against the CPU oracle on the same
seeded inputs, at sizes that span several tiles and a ragged tail, plus the
edge cases (empty context, B=1, ties, ragged vocab, error paths)."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import dflash_oracle as O
from block_diffusion_speculative_softmax_b200 import synth
from tests.gpu_common import TOL, need_gpu, rel_err, to_dev, token_report

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def DF():
    need_gpu()
    from block_diffusion_speculative_softmax_b200 import dflash
    dflash.load()
    return dflash


def _cfg(dtype="bf16", **over):
    base = dict(hidden=576, n_q_heads=8, n_kv_heads=2, head_dim=128, ffn=1000,
                n_draft_layers=3, n_target_layers=5, ctx_len=300, block=16, vocab=5000,
                dtype=dtype)
    base.update(over)
    return synth.small_config("qwen3_4b", **base)


def _round(cfg, a):
    return synth.round_bf16(a.astype(np.float32)) if cfg.dtype == "bf16" else a.astype(np.float32)


def _tdt(cfg):
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


# ------------------------------------------------------------------ fusion
@pytest.mark.parametrize("dtype,H,T,D,N", [("fp32", 256, 3, 2, 37), ("bf16", 2560, 5, 5, 203),
                                           ("bf16", 4096, 9, 7, 65), ("bf16", 2880, 5, 5, 1)])
def test_fuse_ctx(DF, dtype, H, T, D, N):
    cfg = _cfg(dtype, hidden=H, n_target_layers=T, n_draft_layers=D)
    rng = np.random.default_rng(H + N)
    st = _round(cfg, rng.standard_normal((N, T, H)))
    wf = rng.standard_normal((D, T)).astype(np.float32)
    g = _round(cfg, 1 + 0.02 * rng.standard_normal((D, H)))
    ccfg = DF.config_from(cfg)
    dt = _tdt(cfg)
    gd = [to_dev(g[i], torch.float32) for i in range(D)]
    out = torch.empty(D, N, H, dtype=dt, device="cuda")
    DF.dflash_fuse_ctx(ccfg, to_dev(st, dt), to_dev(wf, torch.float32), gd, out)
    torch.cuda.synchronize()
    want = O.fuse_ctx(st, wf, g, cfg.rms_eps, bf16_storage=(dtype == "bf16"))
    assert rel_err(out.float().cpu().numpy(), want) <= TOL[dtype]


# The draft step's split fusion: unnormalised u * g plus per-warp partial sums
# of u^2; applying the row scale here (test arithmetic) must give the fused
# context of the oracle.  D up to 16 and T up to 9 (one and two CTAs per SM,
# ragged N over the persistent grid).
@pytest.mark.parametrize("H,T,D,N", [(576, 5, 3, 300), (2560, 5, 5, 2048), (4096, 9, 7, 301),
                                     (2880, 5, 5, 37), (1024, 3, 16, 500)])
def test_fuse_ctx_rss(DF, H, T, D, N):
    cfg = _cfg("bf16", hidden=H, n_target_layers=T, n_draft_layers=D)
    rng = np.random.default_rng(7 * H + N)
    st = _round(cfg, rng.standard_normal((N, T, H)))
    wf = rng.standard_normal((D, T)).astype(np.float32)
    g = _round(cfg, 1 + 0.02 * rng.standard_normal((D, H)))
    ccfg = DF.config_from(cfg)
    P = DF.dflash_fuse_rss_parts(H)
    assert P == -(-(H // 8) // 32)
    gd = [to_dev(g[i], torch.float32) for i in range(D)]
    v = torch.empty(D, N, H, dtype=torch.bfloat16, device="cuda")
    rss = torch.full((D, N, P), float("nan"), device="cuda")
    ws = DF.alloc_workspace(1 << 12)
    DF.dflash_fuse_ctx_rss(ccfg, to_dev(st, torch.bfloat16), to_dev(wf, torch.float32), gd, v,
                           rss, ws)
    DF.dflash_check(ws)
    ss = rss.double().sum(-1, keepdim=True).cpu().numpy()
    assert np.all(np.isfinite(ss))
    got = v.double().cpu().numpy() / np.sqrt(ss / H + cfg.rms_eps)
    want = O.fuse_ctx(st, wf, g, cfg.rms_eps, bf16_storage=True)
    assert rel_err(got, want) <= TOL["bf16"]
    # the sums of squares themselves, against the oracle's weighted sum
    a = np.exp(wf - wf.max(1, keepdims=True))
    a /= a.sum(1, keepdims=True)
    u = np.einsum("it,nth->inh", a.astype(np.float64), st.astype(np.float64))
    np.testing.assert_allclose(ss[..., 0], (u * u).sum(-1), rtol=1e-4)


# DFlash-style FC fusion: one Linear(T*H -> H) + RMSNorm shared by all layers
@pytest.mark.parametrize("dtype,H,T,N", [("fp32", 256, 3, 37), ("bf16", 576, 5, 300),
                                         ("bf16", 2560, 5, 2048), ("bf16", 4096, 9, 65),
                                         ("bf16", 2880, 5, 16)])
def test_fc_fuse_ctx(DF, dtype, H, T, N):
    # N = 2048 / 300 / 65: token-major tiles (2048: CTA pairs); 16: weight-major
    cfg = _cfg(dtype, hidden=H, n_target_layers=T)
    rng = np.random.default_rng(H + T + N)
    st = _round(cfg, rng.standard_normal((N, T, H)))
    w_fc = _round(cfg, 0.02 * rng.standard_normal((H, T * H)))
    g = _round(cfg, 1 + 0.02 * rng.standard_normal(H))
    ccfg = DF.config_from(cfg)
    dt = _tdt(cfg)
    out = torch.empty(N, H, dtype=dt, device="cuda")
    ws = DF.alloc_workspace(DF.dflash_workspace_size(ccfg, 1, 1, N, N))
    DF.dflash_fc_fuse_ctx(ccfg, to_dev(st, dt), to_dev(w_fc, dt), to_dev(g, torch.float32),
                          out, ws)
    DF.dflash_check(ws)
    want = O.fc_fuse_ctx(st, w_fc, g, cfg.rms_eps, bf16_storage=(dtype == "bf16"))
    assert rel_err(out.float().cpu().numpy(), want) <= TOL[dtype]


def test_fuse_ctx_zero_rows_is_noop(DF):
    cfg = _cfg()
    ccfg = DF.config_from(cfg)
    before = DF.dflash_launch_count()
    DF.dflash_fuse_ctx(ccfg, torch.empty(0, 5, 576, dtype=torch.bfloat16, device="cuda"),
                       torch.zeros(3, 5, device="cuda"), [torch.ones(576, device="cuda")] * 3,
                       torch.empty(16, dtype=torch.bfloat16, device="cuda"))
    assert DF.dflash_launch_count() == before


# ------------------------------------------------------------------ K/V projection
@pytest.mark.parametrize("dtype,M,scatter", [("fp32", 8, False), ("bf16", 16, False),
                                             ("bf16", 37, True), ("bf16", 700, False),
                                             ("bf16", 4700, True)])
def test_kv_project(DF, dtype, M, scatter):
    # M = 4700: 37 token tiles (odd) x 2 feature tiles runs on CTA pairs with
    # a padding tile; 700: token-major single CTAs with split K; <= 64: weight-major
    cfg = _cfg(dtype, hidden=576 if dtype == "bf16" else 256,
               n_kv_heads=2, head_dim=128 if dtype == "bf16" else 64)
    rng = np.random.default_rng(M)
    H, kvd = cfg.hidden, cfg.kv_dim
    x = _round(cfg, rng.standard_normal((M, H)))
    wk = _round(cfg, 0.02 * rng.standard_normal((kvd, H)))
    wv = _round(cfg, 0.02 * rng.standard_normal((kvd, H)))
    pos = rng.integers(0, 9000, M).astype(np.int32)
    rows = M + 11 if scatter else M
    dst = rng.permutation(rows)[:M].astype(np.int64) if scatter else None
    ccfg = DF.config_from(cfg)
    dt = _tdt(cfg)
    k_out = torch.zeros(rows, kvd, dtype=dt, device="cuda")
    v_out = torch.zeros(rows, kvd, dtype=dt, device="cuda")
    ws = DF.alloc_workspace(DF.dflash_workspace_size(ccfg, 1, 1, M, M))
    DF.dflash_kv_project(ccfg, to_dev(x, dt), to_dev(pos, torch.int32),
                         None if dst is None else to_dev(dst, torch.int64), to_dev(wk, dt),
                         to_dev(wv, dt), k_out, v_out, ws)
    DF.dflash_check(ws)
    k, v = O.kv_project(x, pos.astype(np.float64), wk, wv, cfg.n_kv_heads, cfg.head_dim,
                        cfg.rope_theta, bf16_storage=(dtype == "bf16"))
    idx = dst if scatter else np.arange(M)
    kg = k_out.float().cpu().numpy()[idx]
    vg = v_out.float().cpu().numpy()[idx]
    assert rel_err(kg, k.reshape(M, -1)) <= TOL[dtype]
    assert rel_err(vg, v.reshape(M, -1)) <= TOL[dtype]
    if scatter:   # rows not addressed by dst stay untouched
        rest = np.setdiff1d(np.arange(rows), dst)
        assert (k_out.float().cpu().numpy()[rest] == 0).all()


# ------------------------------------------------------------------ attention
@pytest.mark.parametrize("dtype,lens,B,Hq,Hkv,d,blk_req", [
    ("fp32", [64], 8, 4, 2, 64, [0]),
    ("bf16", [2048], 16, 32, 8, 128, [0]),
    ("bf16", [0, 5, 100, 777], 16, 8, 2, 128, [0, 1, 2, 3, 3]),
    ("bf16", [150, 77], 16, 16, 2, 64, [0, 0, 0, 1, 1]),
    ("bf16", [33], 1, 4, 4, 64, [0]),
    ("bf16", [400, 13], 16, 16, 4, 64, [1, 0]),
])
def test_block_attn(DF, dtype, lens, B, Hq, Hkv, d, blk_req):
    # bf16 cases cover split clusters of 16, 8, 2, 1 and 4 CTAs in that order
    cfg = _cfg(dtype, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, block=B)
    rng = np.random.default_rng(sum(lens) + B)
    nb = len(blk_req)
    SL = sum(lens)
    q = _round(cfg, rng.standard_normal((nb * B, Hq, d)))
    kb = _round(cfg, rng.standard_normal((nb * B, Hkv, d)))
    vb = _round(cfg, rng.standard_normal((nb * B, Hkv, d)))
    kc = _round(cfg, rng.standard_normal((max(1, SL), Hkv, d)))
    vc = _round(cfg, rng.standard_normal((max(1, SL), Hkv, d)))
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    ccfg = DF.config_from(cfg)
    dt = _tdt(cfg)
    out = torch.empty(nb * B, Hq, d, dtype=dt, device="cuda")
    ws = DF.alloc_workspace(DF.dflash_workspace_size(ccfg, len(lens), nb, 0, max(lens)))
    DF.dflash_block_attn(ccfg, nb, to_dev(q, dt), to_dev(kb, dt), to_dev(vb, dt),
                         to_dev(kc, dt), to_dev(vc, dt), to_dev(off, torch.int64),
                         to_dev(np.array(blk_req, dtype=np.int32), torch.int32), max(lens), out,
                         ws)
    DF.dflash_check(ws)
    got = out.float().cpu().numpy()
    for b, r in enumerate(blk_req):
        sl = slice(b * B, (b + 1) * B)
        want = O.block_attn(q[sl], kc[off[r]:off[r + 1]], vc[off[r]:off[r + 1]], kb[sl], vb[sl])
        assert rel_err(got[sl], want) <= TOL[dtype], (b, r)


# ------------------------------------------------------------------ MLP
@pytest.mark.parametrize("dtype,M,H,F", [("fp32", 8, 256, 512), ("bf16", 16, 2560, 9728),
                                         ("bf16", 48, 576, 1000), ("bf16", 512, 2880, 2880)])
def test_mlp(DF, dtype, M, H, F):
    cfg = _cfg(dtype, hidden=H, ffn=F)
    rng = np.random.default_rng(M + F)
    h = rng.standard_normal((M, H)).astype(np.float32)
    g = _round(cfg, 1 + 0.02 * rng.standard_normal(H))
    wg = _round(cfg, 0.02 * rng.standard_normal((F, H)))
    wu = _round(cfg, 0.02 * rng.standard_normal((F, H)))
    wd = _round(cfg, 0.02 * rng.standard_normal((H, F)))
    ccfg = DF.config_from(cfg)
    dt = _tdt(cfg)
    hd = to_dev(h, torch.float32)
    ws = DF.alloc_workspace(DF.dflash_workspace_size(ccfg, 1, (M + cfg.block - 1) // cfg.block,
                                                     0, 0))
    DF.dflash_mlp(ccfg, hd, to_dev(g, torch.float32), to_dev(wg, dt), to_dev(wu, dt),
                  to_dev(wd, dt), ws)
    DF.dflash_check(ws)
    want = O.swiglu_mlp(h, g, wg, wu, wd, cfg.rms_eps, bf16_storage=(dtype == "bf16"))
    assert rel_err(hd.cpu().numpy(), want) <= TOL[dtype]


# ------------------------------------------------------------------ LM head argmax
@pytest.mark.parametrize("dtype,M,H,V", [("fp32", 8, 256, 1024), ("bf16", 16, 2560, 151936),
                                         ("bf16", 37, 576, 5017), ("bf16", 512, 2880, 3001)])
def test_lmhead_argmax(DF, dtype, M, H, V):
    cfg = _cfg(dtype, hidden=H, vocab=V)
    rng = np.random.default_rng(V + M)
    x = _round(cfg, rng.standard_normal((M, H)))
    w = _round(cfg, 0.02 * rng.standard_normal((V, H)))
    # planted exact ties: three copies of the row that wins for x[0]
    z0 = x[0].astype(np.float64) @ w.astype(np.float64).T
    win = int(np.argmax(z0))
    dup = sorted({min(win, V - 1), V - 1, V // 2})
    for v in dup:
        w[v] = w[win]
    ccfg = DF.config_from(cfg)
    dt = _tdt(cfg)
    tok = torch.full((M,), -7, dtype=torch.int32, device="cuda")
    mx = torch.zeros(M, dtype=torch.float32, device="cuda")
    conf = torch.full((M,), -1.0, dtype=torch.float32, device="cuda")
    ws = DF.alloc_workspace(DF.dflash_workspace_size(ccfg, 1, (M + 15) // 16, 0, 0))
    DF.dflash_lmhead_argmax(ccfg, to_dev(x, dt), to_dev(w, dt), tok, mx, ws, conf=conf)
    DF.dflash_check(ws)
    otok, omax, z = O.lmhead_argmax(x, w)
    gt = tok.cpu().numpy()
    # stage-isolated check: both sides see the same bf16 inputs, only fp32
    # summation order differs, so rows whose top-2 gap exceeds 1e-3 are exact
    n_exact, n_near, bad = token_report(gt, z, dtype, tol=1e-3 if dtype == "bf16" else None)
    assert not bad, bad[:5]
    assert gt[0] == min(dup + [win])          # lowest index among exact ties
    assert rel_err(mx.cpu().numpy(), omax) <= (1e-5 if dtype == "fp32" else 1e-3)
    # confidence = softmax probability of the argmax (one log-sum-exp share
    # per vocabulary tile, merged in a second pass)
    oc = O.draft_confidence(z)
    gc = conf.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(gc - oc) <= (1e-4 if dtype == "fp32" else 1e-3) * oc + 1e-7)


def test_lmhead_nonfinite_reports_enumeric(DF):
    cfg = _cfg("bf16", hidden=576, vocab=300)
    ccfg = DF.config_from(cfg)
    x = torch.randn(16, 576, device="cuda").to(torch.bfloat16)
    x[3, 5] = float("inf")
    w = (0.02 * torch.randn(300, 576, device="cuda")).to(torch.bfloat16)
    tok = torch.empty(16, dtype=torch.int32, device="cuda")
    ws = DF.alloc_workspace(DF.dflash_workspace_size(ccfg, 1, 1, 0, 0))
    DF.dflash_lmhead_argmax(ccfg, x, w, tok, None, ws)
    with pytest.raises(DF.DFlashError) as e:
        DF.dflash_check(ws)
    assert e.value.status == DF.ENUMERIC
    DF.dflash_check(ws)    # cleared after being reported


# ------------------------------------------------------------------ accept
def test_accept_golden_and_random(DF):
    with open(os.path.join(GOLDEN, "accept_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        d = np.array(c["draft"], dtype=np.int32)
        t = np.array(c["target"], dtype=np.int32)
        R, K, B = d.shape
        n = torch.empty(R, dtype=torch.int32, device="cuda")
        bk = torch.empty(R, dtype=torch.int32, device="cuda")
        out = torch.empty(R, B, dtype=torch.int32, device="cuda")
        DF.dflash_accept(to_dev(d, torch.int32), to_dev(t, torch.int32), n, bk, out)
        assert n.cpu().tolist() == c["n_acc"], c["name"]
        assert bk.cpu().tolist() == c["best_k"], c["name"]
        assert out.cpu().tolist() == c["out"], c["name"]
    rng = np.random.default_rng(5)
    for (R, K, B) in [(1, 1, 1), (7, 1, 16), (33, 4, 16), (5, 32, 32), (100, 3, 8)]:
        d = rng.integers(0, 3, size=(R, K, B)).astype(np.int32)
        t = rng.integers(0, 3, size=(R, K, B)).astype(np.int32)
        n = torch.empty(R, dtype=torch.int32, device="cuda")
        bk = torch.empty(R, dtype=torch.int32, device="cuda")
        out = torch.empty(R, B, dtype=torch.int32, device="cuda")
        DF.dflash_accept(to_dev(d, torch.int32), to_dev(t, torch.int32), n, bk, out)
        on, obk, oout = O.accept(d, t)
        np.testing.assert_array_equal(n.cpu().numpy(), on)
        np.testing.assert_array_equal(bk.cpu().numpy(), obk)
        np.testing.assert_array_equal(out.cpu().numpy(), oout)


def test_accept_planted_lengths(DF):
    rng = np.random.default_rng(6)
    R, B, V = 4096, 16, 151936
    d = rng.integers(0, V, size=(R, B)).astype(np.int32)
    n_pl = synth.geometric_lengths(0.15552, R, B - 1, rng)
    t = synth.plant_targets(d, n_pl, V, rng)
    n = torch.empty(R, dtype=torch.int32, device="cuda")
    bk = torch.empty(R, dtype=torch.int32, device="cuda")
    out = torch.empty(R, B, dtype=torch.int32, device="cuda")
    DF.dflash_accept(to_dev(d[:, None], torch.int32), to_dev(t[:, None], torch.int32), n, bk, out)
    np.testing.assert_array_equal(n.cpu().numpy(), n_pl)


# ------------------------------------------------------------------ D2SD cuts
def test_d2sd_candidates_golden_and_random(DF):
    with open(os.path.join(GOLDEN, "d2sd_prefix_example.json")) as f:
        ex = json.load(f)
    base = np.array([ex["base"]], dtype=np.int32)
    conf = np.array([ex["confidence"]], dtype=np.float32)
    K, B = ex["K"], ex["block"]
    kl = torch.empty(K, dtype=torch.int32, device="cuda")
    cand = torch.empty(K, B, dtype=torch.int32, device="cuda")
    req = torch.empty(K, dtype=torch.int32, device="cuda")
    DF.dflash_d2sd_candidates(to_dev(base, torch.int32), to_dev(conf, torch.float32), K,
                              ex["mask_token_id"], kl, cand, req)
    assert kl.cpu().tolist() == ex["known_len"]
    assert cand.cpu().tolist() == ex["cand_tokens"]
    assert req.cpu().tolist() == [0] * K
    rng = np.random.default_rng(7)
    for (R, B, K) in [(8, 16, 4), (3, 32, 31), (50, 2, 1), (9, 9, 5)]:
        base = rng.integers(0, 1000, size=(R, B)).astype(np.int32)
        conf = (rng.integers(0, 5, size=(R, B)) / 4.0).astype(np.float32)   # many ties
        kl = torch.empty(R * K, dtype=torch.int32, device="cuda")
        cand = torch.empty(R * K, B, dtype=torch.int32, device="cuda")
        DF.dflash_d2sd_candidates(to_dev(base, torch.int32), to_dev(conf, torch.float32), K, 999,
                                  kl, cand)
        okl, ocand = O.d2sd_candidates(base, conf, K, 999)
        np.testing.assert_array_equal(kl.cpu().numpy(), okl)
        np.testing.assert_array_equal(cand.cpu().numpy(), ocand)


# ------------------------------------------------------------------ failure detection
def test_bounded_wait_reports_timeout_and_context_survives(DF):
    ws = DF.alloc_workspace(4096)
    DF.dflash_selftest_wait_timeout(ws, 20_000_000)       # 20 ms
    with pytest.raises(DF.DFlashError) as e:
        DF.dflash_check(ws)
    assert e.value.status == DF.ETIMEOUT
    # the context still works
    d = torch.tensor([[[1, 2, 3]]], dtype=torch.int32, device="cuda")
    n = torch.empty(1, dtype=torch.int32, device="cuda")
    DF.dflash_accept(d, torch.tensor([[[2, 3, 4]]], dtype=torch.int32, device="cuda"), n,
                     torch.empty(1, dtype=torch.int32, device="cuda"),
                     torch.empty(1, 3, dtype=torch.int32, device="cuda"))
    assert n.item() == 2
    DF.dflash_check(ws)
