"""Pins of the CPU oracle against things other than itself: library
routines (torch CPU fp64, scipy), closed forms, invariants, brute force on
tiny inputs and the worked example the D2SD summary prints.  A plausible
slip anywhere in the oracle (a dropped term, a wrong sign, an index off by
one, a transposed operand) fails at least one of these."""
import itertools
import json
import os

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

from oracle import dflash_oracle as O
from oracle import toy_target as TT
from block_diffusion_speculative_softmax_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _t(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64))


# ---------------------------------------------------------------- rounding

def test_bf16_matches_torch_rounding():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(10000) * 10.0 ** rng.integers(-8, 8, 10000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.0 + 2 ** -8 + 2 ** -9,
                         1.0 + 2 ** -9, 3.0e38, -1e-40]])
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.bf16(x), want)


# ---------------------------------------------------------------- softmax / rmsnorm

def test_softmax_matches_scipy():
    z = np.random.default_rng(2).standard_normal((7, 13)) * 30
    np.testing.assert_allclose(O.softmax(z, axis=1), scipy.special.softmax(z, axis=1),
                               rtol=1e-13, atol=1e-300)


def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5, 64)) * 3
    g = 1 + 0.1 * rng.standard_normal(64)
    want = F.rms_norm(_t(x), (64,), weight=_t(g), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rmsnorm(x, g, 1e-6), want, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- fusion

def _fusion_inputs(N=6, T=4, H=32, D=3, seed=4):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((N, T, H)), rng.standard_normal((D, T)),
            1 + 0.05 * rng.standard_normal((D, H)))


def test_fusion_equal_alpha_is_rmsnorm_of_mean():
    s, w, g = _fusion_inputs()
    w[:] = 0.7                                   # constant row -> alpha = 1/T
    out = O.fuse_ctx(s, w, g, 1e-6)
    for i in range(w.shape[0]):
        want = F.rms_norm(_t(s).mean(dim=1), (s.shape[2],), weight=_t(g[i]), eps=1e-6)
        np.testing.assert_allclose(out[i], want.numpy(), rtol=1e-12, atol=1e-12)


def test_fusion_one_hot_alpha_selects_a_layer():
    s, w, g = _fusion_inputs()
    w[:] = 0.0
    sel = [2, 0, 3]
    for i, j in enumerate(sel):
        w[i, j] = 60.0                           # softmax weight 1 - O(e^-60)
    out = O.fuse_ctx(s, w, g, 1e-6)
    for i, j in enumerate(sel):
        want = F.rms_norm(_t(s[:, j, :]), (s.shape[2],), weight=_t(g[i]), eps=1e-6)
        np.testing.assert_allclose(out[i], want.numpy(), rtol=1e-12, atol=1e-12)


def test_fusion_weights_follow_softmax_of_w_fuse():
    # two target layers that are constant rows a and b: the fused row before
    # the norm is alpha_0 a + alpha_1 b, a closed form checked via scipy
    N, H = 3, 16
    s = np.zeros((N, 2, H))
    s[:, 0, :] = 1.0
    s[:, 1, :] = -2.0
    w = np.array([[0.3, -1.1]])
    a = scipy.special.softmax(w[0])
    u = a[0] * 1.0 + a[1] * -2.0
    out = O.fuse_ctx(s, w, np.ones((1, H)), 0.0)
    np.testing.assert_allclose(out[0], np.sign(u) * np.ones((N, H)), rtol=1e-14)
    # and the sign flips when the weights swap
    out2 = O.fuse_ctx(s, w[:, ::-1].copy(), np.ones((1, H)), 0.0)
    u2 = a[1] * 1.0 + a[0] * -2.0
    np.testing.assert_allclose(out2[0], np.sign(u2) * np.ones((N, H)), rtol=1e-14)


def test_fusion_scale_invariant_and_row_independent():
    s, w, g = _fusion_inputs()
    a = O.fuse_ctx(s, w, g, 0.0)
    np.testing.assert_allclose(O.fuse_ctx(5.0 * s, w, g, 0.0), a, rtol=1e-12)
    # one draft layer alone gives the same rows as inside a D-layer call
    np.testing.assert_allclose(O.fuse_ctx(s, w[1:2], g[1:2], 0.0)[0], a[1], rtol=1e-14)
    np.testing.assert_allclose(O.fuse_ctx(s[2:3], w, g, 0.0)[:, 0], a[:, 2], rtol=1e-14)


# ---------------------------------------------------------------- rope

def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(5)
    M, nh, d, theta = 9, 3, 16, 1e4
    x = rng.standard_normal((M, nh, d))
    pos = rng.integers(0, 5000, M).astype(np.float64)
    got = O.rope(x, pos, theta)
    half = d // 2
    z = x[..., :half] + 1j * x[..., half:]
    freq = np.array([theta ** (-(2 * i) / d) for i in range(half)])
    rot = z * np.exp(1j * pos[:, None, None] * freq[None, None, :])
    np.testing.assert_allclose(got[..., :half], rot.real, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got[..., half:], rot.imag, rtol=1e-12, atol=1e-12)


def test_rope_position_zero_is_identity_and_scores_shift_invariant():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 1, 64))
    k = rng.standard_normal((1, 1, 64))
    np.testing.assert_array_equal(O.rope(q, np.zeros(1), 1e6), q)
    s1 = float((O.rope(q, np.array([10.0]), 1e6) * O.rope(k, np.array([3.0]), 1e6)).sum())
    s2 = float((O.rope(q, np.array([8010.0]), 1e6) * O.rope(k, np.array([8003.0]), 1e6)).sum())
    assert abs(s1 - s2) <= 1e-12 * max(1.0, abs(s1))


def test_kv_project_matches_linear_and_shared_projection():
    rng = np.random.default_rng(7)
    H, nkv, d = 32, 2, 8
    f = rng.standard_normal((5, H))     # fused context rows (W^t)
    x = rng.standard_normal((3, H))     # block rows (W^d)
    wk = rng.standard_normal((nkv * d, H))
    wv = rng.standard_normal((nkv * d, H))
    pos_f = np.arange(5.0)
    pos_x = 5.0 + np.arange(3.0)
    k0, v0 = O.kv_project(f, np.zeros(5), wk, wv, nkv, d, 1e6)
    np.testing.assert_allclose(k0.reshape(5, -1), F.linear(_t(f), _t(wk)).numpy(), rtol=1e-12)
    np.testing.assert_allclose(v0.reshape(5, -1), F.linear(_t(f), _t(wv)).numpy(), rtol=1e-12)
    # W^t == W^d: projecting the two row sets separately equals one shared
    # projection over [f ; x] (the DFlash case of heterogeneous projections)
    kf, vf = O.kv_project(f, pos_f, wk, wv, nkv, d, 1e6)
    kx, vx = O.kv_project(x, pos_x, wk, wv, nkv, d, 1e6)
    ka, va = O.kv_project(np.vstack([f, x]), np.concatenate([pos_f, pos_x]), wk, wv, nkv, d, 1e6)
    np.testing.assert_allclose(np.vstack([kf, kx]), ka, rtol=1e-13)
    np.testing.assert_allclose(np.vstack([vf, vx]), va, rtol=1e-13)


# ---------------------------------------------------------------- attention

def _sdpa(q, k, v):
    """torch SDPA reference: q [B][Hq][d], k/v [S][Hkv][d]."""
    Hq, Hkv = q.shape[1], k.shape[1]
    kk = _t(k).repeat_interleave(Hq // Hkv, dim=1).permute(1, 0, 2)
    vv = _t(v).repeat_interleave(Hq // Hkv, dim=1).permute(1, 0, 2)
    out = F.scaled_dot_product_attention(_t(q).permute(1, 0, 2), kk, vv)
    return out.permute(1, 0, 2).numpy()


def test_attention_single_query_no_context_is_plain_attention():
    rng = np.random.default_rng(8)
    q = rng.standard_normal((1, 4, 16))
    kb = rng.standard_normal((1, 2, 16))
    vb = rng.standard_normal((1, 2, 16))
    empty = np.zeros((0, 2, 16))
    got = O.block_attn(q, empty, empty, kb, vb)
    # one key: the output is that key's value for every head
    np.testing.assert_allclose(got, np.repeat(vb, 2, axis=1), rtol=1e-14)
    np.testing.assert_allclose(got, _sdpa(q, kb, vb), rtol=1e-12)


@pytest.mark.parametrize("L,B,Hq,Hkv,d", [(0, 6, 4, 4, 8), (7, 1, 4, 2, 16),
                                          (33, 5, 8, 2, 16), (12, 4, 6, 3, 8)])
def test_attention_matches_torch_sdpa(L, B, Hq, Hkv, d):
    rng = np.random.default_rng(L * 100 + B)
    q = rng.standard_normal((B, Hq, d)) * 2
    kc, vc = rng.standard_normal((L, Hkv, d)), rng.standard_normal((L, Hkv, d))
    kb, vb = rng.standard_normal((B, Hkv, d)), rng.standard_normal((B, Hkv, d))
    got = O.block_attn(q, kc, vc, kb, vb)
    want = _sdpa(q, np.concatenate([kc, kb]), np.concatenate([vc, vb]))
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12)


def test_attention_identical_keys_give_mean_value_and_gqa_equals_mha():
    rng = np.random.default_rng(9)
    L, B, Hq, Hkv, d = 10, 4, 6, 2, 8
    q = rng.standard_normal((B, Hq, d))
    kc = np.broadcast_to(rng.standard_normal((1, Hkv, d)), (L, Hkv, d)).copy()
    kb = np.broadcast_to(kc[:1], (B, Hkv, d)).copy()
    vc, vb = rng.standard_normal((L, Hkv, d)), rng.standard_normal((B, Hkv, d))
    got = O.block_attn(q, kc, vc, kb, vb)
    mean_v = np.concatenate([vc, vb]).mean(axis=0)          # [Hkv][d]
    np.testing.assert_allclose(got, np.broadcast_to(np.repeat(mean_v, 3, axis=0), got.shape),
                               rtol=1e-12)
    kc, kb = rng.standard_normal((L, Hkv, d)), rng.standard_normal((B, Hkv, d))
    g = O.block_attn(q, kc, vc, kb, vb)
    m = O.block_attn(q, np.repeat(kc, 3, 1), np.repeat(vc, 3, 1),
                     np.repeat(kb, 3, 1), np.repeat(vb, 3, 1))
    np.testing.assert_allclose(g, m, rtol=1e-14)


# ---------------------------------------------------------------- mlp / lm head

def test_swiglu_mlp_matches_torch():
    rng = np.random.default_rng(10)
    M, H, Fd = 5, 24, 40
    h = rng.standard_normal((M, H))
    g = 1 + 0.1 * rng.standard_normal(H)
    wg, wu, wd = (rng.standard_normal((Fd, H)) * 0.2, rng.standard_normal((Fd, H)) * 0.2,
                  rng.standard_normal((H, Fd)) * 0.2)
    x = F.rms_norm(_t(h), (H,), weight=_t(g), eps=1e-6)
    want = _t(h) + F.linear(F.silu(F.linear(x, _t(wg))) * F.linear(x, _t(wu)), _t(wd))
    np.testing.assert_allclose(O.swiglu_mlp(h, g, wg, wu, wd, 1e-6), want.numpy(),
                               rtol=1e-12, atol=1e-12)


def test_lmhead_argmax_brute_force_with_planted_ties():
    rng = np.random.default_rng(11)
    M, H, V = 6, 12, 50
    x = rng.standard_normal((M, H))
    w = rng.standard_normal((V, H))
    # plant exact ties: rows 31 and 44 duplicate the row that wins for x[0]
    z0 = x[0] @ w.T
    win = int(np.argmax(z0))
    w[31] = w[win]
    w[44] = w[win]
    w[3] = w[win]                          # a lower duplicate must win
    tok, zmax, _ = O.lmhead_argmax(x, w)
    for m in range(M):
        best_v, best_i = -np.inf, -1
        for v in range(V):
            s = float(sum(x[m, k] * w[v, k] for k in range(H)))
            if s > best_v + 1e-12:
                best_v, best_i = s, v
        assert tok[m] == best_i
        assert abs(zmax[m] - best_v) < 1e-12
    assert tok[0] == min(3, win)


# ---------------------------------------------------------------- accept

def _brute_accept(draft, target):
    R, K, B = draft.shape
    res = []
    for r in range(R):
        lens = []
        for k in range(K):
            ok = [m for m in range(B) if all(draft[r, k, j] == target[r, k, j - 1]
                                             for j in range(1, m + 1))]
            lens.append(max(ok))
        best = min(k for k in range(K) if lens[k] == max(lens))
        res.append((max(lens), best))
    return res


def test_accept_exhaustive_tiny_alphabet():
    V = 3
    for B in range(1, 5):
        for d in itertools.product(range(V), repeat=B):
            for t in itertools.product(range(V), repeat=B):
                dd = np.array(d).reshape(1, 1, B)
                tt = np.array(t).reshape(1, 1, B)
                n, bk, out = O.accept(dd, tt)
                (nb, _), = _brute_accept(dd, tt)
                assert n[0] == nb
                assert list(out[0, :nb]) == list(d[1:nb + 1])
                assert out[0, nb] == t[nb]
                assert (out[0, nb + 1:] == -1).all()


def test_accept_brute_force_over_candidates():
    rng = np.random.default_rng(12)
    for _ in range(400):
        R, K, B = 3, int(rng.integers(1, 5)), int(rng.integers(1, 7))
        d = rng.integers(0, 2, size=(R, K, B))
        t = rng.integers(0, 2, size=(R, K, B))
        n, bk, out = O.accept(d, t)
        for r, (nb, kb) in enumerate(_brute_accept(d, t)):
            assert n[r] == nb and bk[r] == kb
            assert out[r, nb] == t[r, kb, nb]


def test_accept_golden_cases():
    with open(os.path.join(GOLDEN, "accept_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        n, bk, out = O.accept(np.array(c["draft"]), np.array(c["target"]))
        assert n.tolist() == c["n_acc"], c["name"]
        assert bk.tolist() == c["best_k"], c["name"]
        assert out.tolist() == c["out"], c["name"]


def test_planted_targets_give_planted_accept_lengths():
    rng = np.random.default_rng(13)
    V, B, R = 1000, 16, 200
    d = rng.integers(0, V, size=(R, B)).astype(np.int32)
    n = synth.geometric_lengths(0.15552, R, B - 1, rng)
    t = synth.plant_targets(d, n, V, rng)
    got, _, out = O.accept(d[:, None, :], t[:, None, :])
    np.testing.assert_array_equal(got, n)


# ---------------------------------------------------------------- D2SD cuts

def test_d2sd_prefix_example_from_summary():
    with open(os.path.join(GOLDEN, "d2sd_prefix_example.json")) as f:
        ex = json.load(f)
    base = np.array([ex["base"]])
    conf = np.array([ex["confidence"]])
    known, cand = O.d2sd_candidates(base, conf, ex["K"], ex["mask_token_id"])
    assert known.tolist() == ex["known_len"]
    assert cand.tolist() == ex["cand_tokens"]
    spans = [[1, int(k) - 1] for k in known]
    assert spans == ex["prefix_spans"]


def test_d2sd_cuts_brute_force_sort():
    rng = np.random.default_rng(14)
    for _ in range(200):
        R, B = 3, int(rng.integers(2, 17))
        K = int(rng.integers(1, B))
        conf = rng.integers(0, 4, size=(R, B)).astype(np.float64)   # many ties
        base = rng.integers(0, 50, size=(R, B))
        known, cand = O.d2sd_candidates(base, conf, K, 99)
        for r in range(R):
            # brute force: the K-subset of slots 1..B-1 that is smallest in
            # lexicographic (confidence, slot) order
            best = min(itertools.combinations(range(1, B), K),
                       key=lambda S: sorted((conf[r, j], j) for j in S))
            assert known[r * K:(r + 1) * K].tolist() == sorted(best)
            for k, p in enumerate(sorted(best)):
                assert cand[r * K + k, :p].tolist() == base[r, :p].tolist()
                assert (cand[r * K + k, p:] == 99).all()


# ---------------------------------------------------------------- composed step

def _tiny_cfg(**over):
    kw = dict(hidden=32, n_q_heads=4, n_kv_heads=2, head_dim=8, ffn=48,
              n_draft_layers=2, n_target_layers=3, ctx_len=9, block=5, vocab=40)
    kw.update(over)
    return synth.small_config("tiny", **kw)


def test_draft_step_zero_query_reduces_to_mean_value_attention():
    cfg = _tiny_cfg(n_draft_layers=1)
    w = synth.make_weights(cfg, seed=3)
    lay = w["layers"][0]
    lay["w_q"][:] = 0.0          # every score 0 -> uniform attention
    lay["w_down"][:] = 0.0       # MLP contributes nothing
    st = synth.make_states(cfg, 3, 0, cfg.ctx_len)
    tok_in = np.array([7, 0, 0, 0, 0])
    toks, zmax = O.draft_step(cfg, w, [st], [O.Block(0, tok_in, 1)])
    # the same step written as plain torch ops
    B, H, L = cfg.block, cfg.hidden, cfg.ctx_len
    ids = torch.tensor([7] + [cfg.mask_token_id] * (B - 1))
    h = _t(w["embed"])[ids]
    a = torch.softmax(_t(w["w_fuse"][0]), 0)
    u = (a[None, :, None] * _t(st)).sum(1)
    f = F.rms_norm(u, (H,), weight=_t(lay["g_fuse"]), eps=cfg.rms_eps)
    x = F.rms_norm(h, (H,), weight=_t(lay["g_attn"]), eps=cfg.rms_eps)
    vals = torch.cat([F.linear(f, _t(lay["w_vt"])), F.linear(x, _t(lay["w_vd"]))])  # [L+B][kvd]
    mv = vals.mean(0).reshape(cfg.n_kv_heads, cfg.head_dim)
    o = mv.repeat_interleave(cfg.n_q_heads // cfg.n_kv_heads, 0).reshape(-1)
    h = h + F.linear(o, _t(lay["w_o"]))[None, :]
    z = F.linear(F.rms_norm(h, (H,), weight=_t(w["g_final"]), eps=cfg.rms_eps),
                 _t(w["lm_head"]))
    want = z.argmax(1).numpy()
    want[0] = 7
    np.testing.assert_array_equal(toks[0], want)
    np.testing.assert_allclose(zmax[0], z.max(1).values.numpy(), rtol=1e-12)


def test_draft_step_blocks_are_independent_and_share_context():
    cfg = _tiny_cfg()
    w = synth.make_weights(cfg, seed=4)
    st = [synth.make_states(cfg, 4, r, 6 + 3 * r) for r in range(2)]
    b = [O.Block(0, [3, 1, 2, 0, 0], 1), O.Block(1, [5, 0, 0, 0, 0], 1),
         O.Block(0, [3, 1, 2, 0, 0], 3)]
    tok, zm = O.draft_step(cfg, w, st, b)
    for i, blk in enumerate(b):
        t1, m1 = O.draft_step(cfg, w, st, [blk])
        np.testing.assert_array_equal(t1[0], tok[i])
        np.testing.assert_allclose(m1[0], zm[i], rtol=1e-14)
    assert tok[2][:3].tolist() == [3, 1, 2]


def test_shared_kv_weights_equal_heterogeneous_with_equal_matrices():
    cfg = _tiny_cfg()
    w = synth.make_weights(cfg, seed=5, separate_kv=False)
    st = [synth.make_states(cfg, 5, 0, 7)]
    blk = [O.Block(0, [4, 0, 0, 0, 0], 1)]
    t_a, m_a = O.draft_step(cfg, w, st, blk)
    for lay in w["layers"]:
        lay["w_kt"] = lay["w_kd"].copy()
        lay["w_vt"] = lay["w_vd"].copy()
    t_b, m_b = O.draft_step(cfg, w, st, blk)
    np.testing.assert_array_equal(t_a, t_b)
    np.testing.assert_array_equal(m_a, m_b)


# ------------------------------------------------ DFlash FC-fusion variant

def test_fc_fusion_single_layer_identity_is_rmsnorm():
    # T = 1 and W_fc = I: the shared context is RMSNorm of the one target layer
    rng = np.random.default_rng(21)
    H = 24
    st = rng.standard_normal((7, 1, H))
    g = 1 + 0.1 * rng.standard_normal(H)
    got = O.fc_fuse_ctx(st, np.eye(H), g, 1e-6)
    want = F.rms_norm(_t(st[:, 0]), (H,), weight=_t(g), eps=1e-6).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_fc_fusion_reproduces_softmax_fusion_with_stacked_identities():
    # W_fc = [a_1 I | ... | a_T I] with a = softmax(w) is the weighted sum of
    # the per-layer fusion; with the same gain both give the same context
    rng = np.random.default_rng(22)
    N, T, H = 6, 4, 16
    st = rng.standard_normal((N, T, H))
    w = rng.standard_normal(T)
    a = np.exp(w - w.max()) / np.exp(w - w.max()).sum()
    w_fc = np.concatenate([a[j] * np.eye(H) for j in range(T)], axis=1)   # [H][T*H]
    g = 1 + 0.1 * rng.standard_normal(H)
    got = O.fc_fuse_ctx(st, w_fc, g, 1e-6)
    want = O.fuse_ctx(st, w[None, :], g[None, :], 1e-6)[0]
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13)
    # a general W_fc is the concatenation times W_fc^T, then RMSNorm
    w_r = rng.standard_normal((H, T * H))
    u = st.reshape(N, T * H) @ w_r.T
    want_r = F.rms_norm(_t(u), (H,), weight=_t(g), eps=1e-6).numpy()
    np.testing.assert_allclose(O.fc_fuse_ctx(st, w_r, g, 1e-6), want_r, rtol=1e-12)


def test_dflash_variant_draft_step_equals_dflare_with_tied_fusion_and_kv():
    # The DFlash variant (one FC-fused context for all layers, context K/V
    # through the block's own W^d) must equal the DFLARE step when every
    # layer's alpha row and gain are the same, W^t = W^d, and W_fc stacks
    # alpha-scaled identities.
    cfg = _tiny_cfg()
    w = synth.make_weights(cfg, seed=6, separate_kv=False)
    T, H = cfg.n_target_layers, cfg.hidden
    row = w["w_fuse"][0].astype(np.float64)
    g = w["layers"][0]["g_fuse"].astype(np.float64)
    w_dflare = dict(w, w_fuse=np.tile(row, (cfg.n_draft_layers, 1)),
                    layers=[dict(l, g_fuse=g) for l in w["layers"]])
    a = np.exp(row - row.max()) / np.exp(row - row.max()).sum()
    w_dflash = dict(w, w_fc=np.concatenate([a[j] * np.eye(H) for j in range(T)], axis=1),
                    g_fc=g)
    st = [synth.make_states(cfg, 6, 0, 8)]
    blk = [O.Block(0, [9, 0, 0, 0, 0], 1), O.Block(0, [9, 2, 0, 0, 0], 2)]
    t_a, m_a = O.draft_step(cfg, w_dflare, st, blk)
    t_b, m_b = O.draft_step(cfg, w_dflash, st, blk)
    np.testing.assert_array_equal(t_a, t_b)
    np.testing.assert_allclose(m_a, m_b, rtol=1e-12)
    # and it genuinely differs once the layers' fusions differ
    t_c, m_c = O.draft_step(cfg, dict(w_dflare, w_fuse=w["w_fuse"]), st, blk)
    assert not np.allclose(m_a, m_c)


# ---------------------------------------------------------------- losslessness

def speculative_decode(tw, cfg, dw, prompt, n_new, draft_fn, accept_fn, rng,
                       force_p=0.3):
    """Speculative loop: draft a block from the target's context states,
    verify with the target, accept, roll forward (DFlash summary,
    methodology steps 1-4).  ``force_p``: with this per-slot continuation
    probability, leading draft slots are replaced by the target's greedy
    continuation so multi-token acceptance is exercised."""
    B = cfg.block
    seq = [int(t) for t in prompt]
    steps = 0
    while len(seq) - len(prompt) < n_new:
        ctx = np.asarray(seq[:-1])
        st, _ = TT.forward(tw, ctx)                       # [L][3][H]
        d = draft_fn(st, seq[-1])                         # [B], d[0] = anchor
        assert d[0] == seq[-1]
        m = min(int(rng.geometric(force_p)) - 1, B - 1)
        if m:
            cont = TT.greedy(tw, np.asarray(seq), m)
            d = d.copy()
            d[1:m + 1] = cont
        _, nxt = TT.forward(tw, np.asarray(seq + [int(v) for v in d[1:]]))
        t = nxt[len(seq) - 1: len(seq) - 1 + B]           # target[j] predicts slot j+1
        n, out = accept_fn(d, t)
        seq += [int(v) for v in out[:n + 1]]
        steps += 1
    return np.asarray(seq[len(prompt):len(prompt) + n_new]), steps


def test_speculative_loop_with_oracle_draft_is_lossless():
    cfg = synth.get_config("tiny")
    dw = synth.make_weights(cfg, seed=0)
    tw = synth.make_toy_target_weights(cfg.vocab, cfg.hidden, seed=0)
    prompt = synth.make_prompt(cfg.vocab, 24, seed=0)
    n_new = 30
    greedy = TT.greedy(tw, prompt, n_new)

    def draft_fn(states, anchor):
        toks, _ = O.draft_step(cfg, dw, [states],
                               [O.Block(0, [anchor] + [0] * (cfg.block - 1), 1)])
        return toks[0]

    def accept_fn(d, t):
        n, _, out = O.accept(d[None, None, :], np.asarray(t)[None, None, :])
        return int(n[0]), out[0]

    rng = np.random.default_rng(0)
    got, steps = speculative_decode(tw, cfg, dw, prompt, n_new, draft_fn, accept_fn, rng)
    np.testing.assert_array_equal(got, greedy)
    assert steps < n_new          # some steps accepted more than one token


# ---------------------------------------------------------------- draft confidence

def test_draft_confidence_is_top1_softmax_probability():
    rng = np.random.default_rng(15)
    z = rng.standard_normal((6, 40)) * 3
    want = scipy.special.softmax(z, axis=1).max(axis=1)
    np.testing.assert_allclose(O.draft_confidence(z), want, rtol=1e-13)
    # closed forms: a uniform row gives 1/V, a dominant logit gives ~1
    assert abs(O.draft_confidence(np.zeros((1, 40)))[0] - 1 / 40) < 1e-15
    big = np.zeros((1, 40))
    big[0, 7] = 800.0
    assert abs(O.draft_confidence(big)[0] - 1.0) < 1e-15
    # invariant to a constant shift of all logits
    np.testing.assert_allclose(O.draft_confidence(z + 123.0), O.draft_confidence(z), rtol=1e-12)


# ------------------------------------------- composed step, restated in torch

def _rope_complex(x, pos, theta):
    """Rotate-half RoPE written as a complex rotation: the pair
    (x_i, x_{i+d/2}) is the complex number x_i + i x_{i+d/2}, turned by the
    angle pos * theta^(-2i/d).  x [M][heads][d] (torch fp64), pos [M]."""
    d = x.shape[-1]
    half = d // 2
    freq = theta ** (-2.0 * torch.arange(half, dtype=torch.float64) / d)
    ang = pos.to(torch.float64)[:, None, None] * freq[None, None, :]
    z = torch.complex(x[..., :half], x[..., half:]) * torch.polar(torch.ones_like(ang), ang)
    return torch.cat([z.real, z.imag], dim=-1)


def _torch_draft_block(cfg, w, states, tokens, known_len, blk_pos0=None, swap_kv=False,
                       rope_q=True):
    """One draft block written with torch library routines, independently of
    the oracle (DFLARE summary sections 2.1-2.2; DFlash summary methodology
    step 2): per layer softmax fusion + RMSNorm of the T target states,
    context K/V through W^t at positions 0..L-1, block Q and K/V through W^d
    at positions L..L+B-1, unmasked GQA attention over [context ; block] by
    scaled_dot_product_attention, O projection and SwiGLU MLP with
    residuals, final RMSNorm and the LM head.  The keyword arguments plant
    plausible slips (block positions from 0, W^t and W^d swapped, no RoPE on
    Q) to show the comparison notices them.  Returns (x_final, logits)."""
    H, B, eps, theta = cfg.hidden, cfg.block, cfg.rms_eps, cfg.rope_theta
    Hq, Hkv, d = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    st = _t(states)
    L = st.shape[0]
    ids = torch.tensor([int(tokens[s]) if s < known_len else cfg.mask_token_id
                        for s in range(B)])
    h = _t(w["embed"])[ids]
    pos_c = torch.arange(L)
    pos_b = torch.arange(B) + (L if blk_pos0 is None else blk_pos0)
    for i, lay in enumerate(w["layers"]):
        wkt, wvt, wkd, wvd = (_t(lay[n]) for n in ("w_kt", "w_vt", "w_kd", "w_vd"))
        if swap_kv:
            wkt, wkd, wvt, wvd = wkd, wkt, wvd, wvt
        a = torch.softmax(_t(w["w_fuse"][i]), dim=0)
        f = F.rms_norm(torch.einsum("t,lth->lh", a, st), (H,), weight=_t(lay["g_fuse"]),
                       eps=eps)
        kc = _rope_complex(F.linear(f, wkt).reshape(L, Hkv, d), pos_c, theta)
        vc = F.linear(f, wvt).reshape(L, Hkv, d)
        x = F.rms_norm(h, (H,), weight=_t(lay["g_attn"]), eps=eps)
        q = F.linear(x, _t(lay["w_q"])).reshape(B, Hq, d)
        if rope_q:
            q = _rope_complex(q, pos_b, theta)
        kb = _rope_complex(F.linear(x, wkd).reshape(B, Hkv, d), pos_b, theta)
        vb = F.linear(x, wvd).reshape(B, Hkv, d)
        keys = torch.cat([kc, kb]).repeat_interleave(Hq // Hkv, dim=1).permute(1, 0, 2)
        vals = torch.cat([vc, vb]).repeat_interleave(Hq // Hkv, dim=1).permute(1, 0, 2)
        o = F.scaled_dot_product_attention(q.permute(1, 0, 2), keys, vals)   # [Hq][B][d]
        h = h + F.linear(o.permute(1, 0, 2).reshape(B, Hq * d), _t(lay["w_o"]))
        x = F.rms_norm(h, (H,), weight=_t(lay["g_mlp"]), eps=eps)
        act = F.silu(F.linear(x, _t(lay["w_gate"]))) * F.linear(x, _t(lay["w_up"]))
        h = h + F.linear(act, _t(lay["w_down"]))
    xf = F.rms_norm(h, (H,), weight=_t(w["g_final"]), eps=eps)
    return xf.numpy(), F.linear(xf, _t(w["lm_head"])).numpy()


def _strong_weights(cfg, seed):
    """Synthetic draft weights with matrices scaled to std 0.2, so attention
    scores are O(1) and every path (positions, W^t vs W^d, the MLP) moves
    the logits by far more than rounding."""
    w = synth.make_weights(cfg, seed)
    for lay in w["layers"]:
        for n in ("w_q", "w_kt", "w_vt", "w_kd", "w_vd", "w_o", "w_gate", "w_up", "w_down"):
            lay[n] = lay[n] * 10.0
    w["embed"] = w["embed"] * 50.0
    w["lm_head"] = w["lm_head"] * 10.0
    return w


@pytest.mark.parametrize("theta", [1.0e6, 100.0])
def test_whole_draft_step_matches_torch_restatement(theta):
    cfg = _tiny_cfg(rope_theta=theta)
    w = _strong_weights(cfg, seed=31)
    lens = [9, 4]
    st = [synth.make_states(cfg, 31, r, lens[r]) for r in range(2)]
    blocks = [O.Block(0, [5, 0, 0, 0, 0], 1), O.Block(1, [11, 0, 0, 0, 0], 1),
              O.Block(0, [5, 17, 3, 0, 0], 3)]
    keep = {}
    tok, zmax = O.draft_step(cfg, w, st, blocks, keep=keep)
    for i, blk in enumerate(blocks):
        xf, z = _torch_draft_block(cfg, w, st[blk.req], blk.tokens, blk.known_len)
        np.testing.assert_allclose(keep["x_final"][i], xf, rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(keep["logits"][i], z, rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(zmax[i], z.max(1), rtol=1e-10, atol=1e-11)
        want = z.argmax(1)
        want[:blk.known_len] = blk.tokens[:blk.known_len]
        np.testing.assert_array_equal(tok[i], want)


def test_torch_restatement_notices_position_and_projection_slips():
    # each planted slip moves the logits by far more than the 1e-10 the
    # comparison above allows, so the oracle cannot carry any of them
    cfg = _tiny_cfg(rope_theta=100.0)
    w = _strong_weights(cfg, seed=32)
    st = synth.make_states(cfg, 32, 0, 9)
    blk = O.Block(0, [5, 0, 0, 0, 0], 1)
    keep = {}
    O.draft_step(cfg, w, [st], [blk], keep=keep)
    ref = keep["logits"][0]
    scale = np.abs(ref).max()
    for slip in (dict(blk_pos0=0), dict(swap_kv=True), dict(rope_q=False)):
        _, z = _torch_draft_block(cfg, w, st, blk.tokens, blk.known_len, **slip)
        assert np.abs(z - ref).max() > 1e-3 * scale, slip
