"""CPU oracle for the block-diffusion draft step and its greedy verification.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its CPU-baseline and reference legs) may import this module.
The product path (the CUDA library and its binding) never calls it, and this
module imports nothing from the product package.

Plain, slow, obviously correct NumPy float64, step by step in the order the
pages give.  Sources (web summaries of three papers):

* "DFlash: Block Diffusion for Flash Speculative Decoding" -- methodology
  steps 1-4: target features -> one-pass block draft -> parallel
  verification (accepted tokens are emitted, the first rejected slot is
  replaced by the target's own token) -> roll the window forward.
* "D2SD: accelerating speculative decoding with dual diffusion drafters" --
  methodology 1-5: per-position confidence, a prefix tree keeping the top-K
  prefix spans cut at likely rejection points, a batched re-anchored second
  draft, and acceptance of the longest prefix that matches the target.
* "DFLARE: scaling draft capacity of block-diffusion speculative decoding"
  -- section 2.1 (per-layer softmax fusion alpha^(i) = softmax(W_fuse[i]),
  weighted sum of T target layers, then RMSNorm) and section 2.2 (separate
  K/V projections W^t for the target context and W^d for the draft block);
  section 1 item 1 and section 2.2 also describe the DFlash baseline (one
  FC-fused context shared by all draft layers, context and block sharing
  the K/V projections), available here as a variant (``fc_fuse_ctx``).

Readings where the pages are silent (kept identical in the CUDA path):
RMSNorm y = x / sqrt(mean(x^2) + eps) * g with a learned gain g; rotate-half
RoPE on Q and K with context positions 0..L-1 and block positions L..L+B-1;
attention scale 1/sqrt(d) with no mask; SwiGLU MLP; pre-norm residual
layers; argmax ties go to the lowest token id.

``bf16_storage=True`` rounds a tensor to bf16 (round to nearest even) at each
point where the GPU path stores it in bf16: the fused context, Q, K, V, the
normed activations that feed a matrix product, the attention output and the
SwiGLU product.  The residual stream h is never rounded (the GPU keeps it in
fp32).  No rounding inside a sum is emulated.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "bf16", "softmax", "rmsnorm", "fuse_ctx", "rope", "kv_project",
    "block_attn", "swiglu_mlp", "lmhead_logits", "lmhead_argmax", "accept",
    "d2sd_candidates", "draft_request", "draft_step", "Block", "draft_confidence",
]


# ---------------------------------------------------------------------------
# storage rounding
# ---------------------------------------------------------------------------

def bf16(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even), returned as float64.

    The value is first rounded to fp32 (the GPU holds fp32 before it stores
    bf16), then the low 16 bits of the fp32 pattern are rounded away."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    out = (u.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return out.astype(np.float64)


def _store(x: np.ndarray, bf16_storage: bool) -> np.ndarray:
    return bf16(x) if bf16_storage else np.asarray(x, dtype=np.float64)


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# building blocks
# ---------------------------------------------------------------------------

def softmax(z: np.ndarray, axis: int = -1) -> np.ndarray:
    """exp(z - max) / sum(exp(z - max)) along ``axis``."""
    z = _f64(z)
    e = np.exp(z - z.max(axis=axis, keepdims=True))
    return e / e.sum(axis=axis, keepdims=True)


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g."""
    x = _f64(x)
    ms = (x * x).mean(axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * _f64(g)


def fuse_ctx(states: np.ndarray, w_fuse: np.ndarray, g_fuse: np.ndarray,
             eps: float, bf16_storage: bool = False) -> np.ndarray:
    """Adaptive layer fusion (DFLARE summary, section 2.1).

    states [N][T][H] target hidden states, w_fuse [D][T], g_fuse [D][H].
    For every draft layer i: alpha^(i) = softmax(W_fuse[i, :]) over the T
    target layers, u = sum_j alpha^(i)_j h_j, f^(i) = RMSNorm_{g_fuse_i}(u).
    Returns [D][N][H]."""
    s = _f64(states)
    alpha = softmax(_f64(w_fuse), axis=1)                 # [D][T]
    D = alpha.shape[0]
    N, T, H = s.shape
    out = np.empty((D, N, H), dtype=np.float64)
    for i in range(D):
        u = np.zeros((N, H), dtype=np.float64)
        for j in range(T):
            u += alpha[i, j] * s[:, j, :]
        out[i] = _store(rmsnorm(u, g_fuse[i], eps), bf16_storage)
    return out


def fc_fuse_ctx(states: np.ndarray, w_fc: np.ndarray, g_fc: np.ndarray,
                eps: float, bf16_storage: bool = False) -> np.ndarray:
    """DFlash-style context fusion (DFLARE summary, section 1 item 1 and
    section 2.2, describing the DFlash baseline): one fully connected layer
    maps the T concatenated target hidden states of a row to a single shared
    representation that every draft layer receives.

    states [N][T][H], w_fc [H][T*H] (nn.Linear layout over the concatenation
    h_1 | h_2 | ... | h_T), g_fc [H].  The pages do not say whether the FC
    output is normalised; it is read here as RMSNorm_{g_fc}(concat(h) W_fc^T),
    the same normalisation the per-layer fusion applies, so both variants
    hand the K/V projections vectors of the same scale.  Returns [N][H]."""
    s = _f64(states)
    N, T, H = s.shape
    u = s.reshape(N, T * H) @ _f64(w_fc).T
    return _store(rmsnorm(u, g_fc, eps), bf16_storage)


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding of x [M][n_heads][d] at positions pos[M].

    With inv_freq_i = theta^(-2i/d) for i < d/2 and angle a = pos * inv_freq:
    out[:i] = x1 cos a - x2 sin a, out[d/2+i] = x2 cos a + x1 sin a."""
    x = _f64(x)
    d = x.shape[-1]
    half = d // 2
    inv = theta ** (-2.0 * np.arange(half, dtype=np.float64) / d)
    ang = _f64(pos)[:, None] * inv[None, :]               # [M][d/2]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def kv_project(x: np.ndarray, pos: np.ndarray, w_k: np.ndarray,
               w_v: np.ndarray, n_kv_heads: int, head_dim: int,
               theta: float, bf16_storage: bool = False
               ) -> Tuple[np.ndarray, np.ndarray]:
    """K = RoPE(x W_K^T) and V = x W_V^T as [M][Hkv][d] (DFLARE summary,
    section 2.2: the same routine serves W^t for context rows and W^d for
    block rows)."""
    x = _f64(x)
    M = x.shape[0]
    k = (x @ _f64(w_k).T).reshape(M, n_kv_heads, head_dim)
    v = (x @ _f64(w_v).T).reshape(M, n_kv_heads, head_dim)
    k = rope(k, pos, theta)
    return _store(k, bf16_storage), _store(v, bf16_storage)


def block_attn(q: np.ndarray, k_ctx: np.ndarray, v_ctx: np.ndarray,
               k_blk: np.ndarray, v_blk: np.ndarray) -> np.ndarray:
    """Block attention over [context KV ; block KV] with GQA and no mask.

    q [B][Hq][d]; k_ctx/v_ctx [L][Hkv][d]; k_blk/v_blk [B][Hkv][d].
    q head h reads kv head h // (Hq / Hkv).  Returns [B][Hq][d]."""
    q = _f64(q)
    keys = np.concatenate([_f64(k_ctx), _f64(k_blk)], axis=0)   # [L+B][Hkv][d]
    vals = np.concatenate([_f64(v_ctx), _f64(v_blk)], axis=0)
    B, Hq, d = q.shape
    Hkv = keys.shape[1]
    group = Hq // Hkv
    out = np.empty_like(q)
    scale = 1.0 / np.sqrt(d)
    for h in range(Hq):
        g = h // group
        s = (q[:, h, :] @ keys[:, g, :].T) * scale             # [B][L+B]
        p = softmax(s, axis=1)
        out[:, h, :] = p @ vals[:, g, :]
    return out


def swiglu_mlp(h: np.ndarray, g_mlp: np.ndarray, w_gate: np.ndarray,
               w_up: np.ndarray, w_down: np.ndarray, eps: float,
               bf16_storage: bool = False) -> np.ndarray:
    """Pre-norm SwiGLU MLP with residual: h + (silu(x Wg^T) * (x Wu^T)) Wd^T
    with x = RMSNorm_{g_mlp}(h) and silu(z) = z / (1 + exp(-z))."""
    h = _f64(h)
    x = _store(rmsnorm(h, g_mlp, eps), bf16_storage)
    gate = x @ _f64(w_gate).T
    up = x @ _f64(w_up).T
    act = _store(gate / (1.0 + np.exp(-gate)) * up, bf16_storage)
    return h + act @ _f64(w_down).T


def lmhead_logits(x: np.ndarray, w_lm: np.ndarray,
                  chunk: int = 16384) -> np.ndarray:
    """z = x W_lm^T, computed over vocabulary rows in chunks (each logit is
    still one full dot product; chunking only bounds host memory)."""
    x = _f64(x)
    V = w_lm.shape[0]
    z = np.empty((x.shape[0], V), dtype=np.float64)
    for v0 in range(0, V, chunk):
        z[:, v0:v0 + chunk] = x @ _f64(w_lm[v0:v0 + chunk]).T
    return z


def lmhead_argmax(x: np.ndarray, w_lm: np.ndarray
                  ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Greedy draft tokens: tok[m] = smallest v with z[m, v] = max_v z[m, v].
    Returns (tokens int32 [M], max logit [M], logits [M][V])."""
    z = lmhead_logits(x, w_lm)
    tok = np.argmax(z, axis=1).astype(np.int32)   # first occurrence = lowest id
    return tok, z.max(axis=1), z


def draft_confidence(z: np.ndarray) -> np.ndarray:
    """Per-slot confidence of the draft's own prediction: the softmax
    probability of its argmax token, 1 / sum_v exp(z_v - max z).

    D2SD summary, methodology step 1: the first drafter reports, for every
    position, a confidence that its token will be accepted.  The pages do not
    say how it is computed; the draft's top-1 probability is the plainest
    reading (it needs no extra head)."""
    z = _f64(z)
    m = z.max(axis=-1, keepdims=True)
    return 1.0 / np.exp(z - m).sum(axis=-1)


# ---------------------------------------------------------------------------
# verification
# ---------------------------------------------------------------------------

def accept(draft: np.ndarray, target: np.ndarray
           ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Greedy acceptance over K candidate blocks per request.

    draft, target: int [R][K][B].  Slot 0 of a block is the anchor (the last
    accepted token); draft[j] for j >= 1 is a drafted token; target[j] is the
    target model's argmax after reading slots 0..j, i.e. its prediction for
    slot j+1 (DFlash summary, methodology step 3).  For candidate k,
    n_k = the largest m <= B-1 with draft[j] == target[j-1] for all 1<=j<=m.
    The longest candidate wins, lowest k on ties (D2SD summary, methodology
    step 4).  Output: draft[k*][1..n] followed by the target's own token
    target[k*][n]; remaining slots -1.
    Returns (n_acc [R], best_k [R], out_tok [R][B])."""
    draft = np.asarray(draft)
    target = np.asarray(target)
    R, K, B = draft.shape
    n_acc = np.zeros(R, dtype=np.int32)
    best_k = np.zeros(R, dtype=np.int32)
    out = np.full((R, B), -1, dtype=np.int32)
    for r in range(R):
        best_n, best = -1, 0
        for k in range(K):
            n = 0
            while n < B - 1 and draft[r, k, n + 1] == target[r, k, n]:
                n += 1
            if n > best_n:
                best_n, best = n, k
        n_acc[r] = best_n
        best_k[r] = best
        out[r, :best_n] = draft[r, best, 1:best_n + 1]
        out[r, best_n] = target[r, best, best_n]
    return n_acc, best_k, out


def d2sd_candidates(base: np.ndarray, conf: np.ndarray, K: int,
                    mask_token_id: int) -> Tuple[np.ndarray, np.ndarray]:
    """D2SD prefix selection and re-anchoring (D2SD summary, methodology
    steps 2-3).

    base [R][B] first-pass block (slot 0 = anchor), conf [R][B] per-position
    confidence (slot 0 unused).  The K slots in 1..B-1 with the lowest
    confidence (ties: lower slot first) are the cut points p_1 < ... < p_K.
    Candidate k keeps slots 0..p_k-1 of the base block (known_len = p_k) and
    masks slots p_k..B-1 for the second drafter.
    Returns (known_len int32 [R*K], cand_tokens int32 [R*K][B])."""
    base = np.asarray(base)
    conf = np.asarray(conf)
    R, B = base.shape
    known = np.zeros(R * K, dtype=np.int32)
    cand = np.zeros((R * K, B), dtype=np.int32)
    for r in range(R):
        order = sorted(range(1, B), key=lambda j: (float(conf[r, j]), j))
        cuts = sorted(order[:K])
        for k, p in enumerate(cuts):
            known[r * K + k] = p
            cand[r * K + k, :p] = base[r, :p]
            cand[r * K + k, p:] = mask_token_id
    return known, cand


# ---------------------------------------------------------------------------
# the draft step
# ---------------------------------------------------------------------------

class Block:
    """One draft block: the request it belongs to, its B slot tokens and how
    many leading slots are known (1 = anchor only, the DFlash case)."""

    def __init__(self, req: int, tokens: Sequence[int], known_len: int = 1):
        self.req = int(req)
        self.tokens = np.asarray(tokens, dtype=np.int64)
        self.known_len = int(known_len)


def _ctx_kv(cfg, weights, states, bf16_storage):
    """Per draft layer context K/V of one request.

    DFLARE (default): fuse all T target layers with that layer's own alpha,
    RMSNorm, then that layer's W^t projections.  DFlash variant (weights
    carry "w_fc"): one FC-fused context shared by every layer, projected by
    each layer's W^t -- which the DFlash baseline shares with the block's
    W^d (pass weights with w_kt = w_kd and w_vt = w_vd for that)."""
    eps, theta = cfg.rms_eps, cfg.rope_theta
    lays = weights["layers"]
    L = states.shape[0]
    if "w_fc" in weights:
        c = fc_fuse_ctx(states, weights["w_fc"], weights["g_fc"], eps, bf16_storage)
        fused = [c] * len(lays)
    else:
        g_fuse = np.stack([_f64(l["g_fuse"]) for l in lays])
        fused = fuse_ctx(states, weights["w_fuse"], g_fuse, eps, bf16_storage)
    pos = np.arange(L, dtype=np.float64)
    kv = []
    for i, lay in enumerate(lays):
        kv.append(kv_project(fused[i], pos, lay["w_kt"], lay["w_vt"],
                             cfg.n_kv_heads, cfg.head_dim, theta, bf16_storage))
    return kv


def draft_request(cfg, weights: dict, states: np.ndarray,
                  blocks: List[Block], bf16_storage: bool = False,
                  keep: Optional[Dict] = None):
    """Draft every block of one request in one forward pass each.

    states [L][T][H] are the request's target hidden states.  For each draft
    layer: context K/V through W^t from that layer's fused context; the
    block's pre-normed hidden states give Q and block K/V through W^d; the B
    block queries attend to [context ; block] without a mask; O projection,
    then the SwiGLU MLP, each with a residual.  After the final RMSNorm the
    LM head's argmax gives one token per slot; slots inside the known prefix
    keep their input token.  Returns (tokens [nb][B], max_logit [nb][B])."""
    eps, theta = cfg.rms_eps, cfg.rope_theta
    L = states.shape[0]
    B = cfg.block
    kv = _ctx_kv(cfg, weights, states, bf16_storage)
    toks, maxz = [], []
    for blk in blocks:
        slot_tok = np.where(np.arange(B) < blk.known_len, blk.tokens,
                            cfg.mask_token_id)
        h = _f64(weights["embed"][slot_tok])                 # [B][H]
        pos = L + np.arange(B, dtype=np.float64)
        for i, lay in enumerate(weights["layers"]):
            x = _store(rmsnorm(h, lay["g_attn"], eps), bf16_storage)
            q = (x @ _f64(lay["w_q"]).T).reshape(B, cfg.n_q_heads, cfg.head_dim)
            q = _store(rope(q, pos, theta), bf16_storage)
            kb, vb = kv_project(x, pos, lay["w_kd"], lay["w_vd"],
                                cfg.n_kv_heads, cfg.head_dim, theta,
                                bf16_storage)
            o = block_attn(q, kv[i][0], kv[i][1], kb, vb)
            o = _store(o.reshape(B, -1), bf16_storage)
            h = h + o @ _f64(lay["w_o"]).T
            h = swiglu_mlp(h, lay["g_mlp"], lay["w_gate"], lay["w_up"],
                           lay["w_down"], eps, bf16_storage)
        x = _store(rmsnorm(h, weights["g_final"], eps), bf16_storage)
        tok, zmax, z = lmhead_argmax(x, weights["lm_head"])
        tok = np.where(np.arange(B) < blk.known_len, blk.tokens, tok)
        toks.append(tok.astype(np.int32))
        maxz.append(zmax)
        if keep is not None:
            keep.setdefault("x_final", []).append(x)
            keep.setdefault("logits", []).append(z)
    return np.stack(toks), np.stack(maxz)


def draft_step(cfg, weights: dict, states: Sequence[np.ndarray],
               blocks: List[Block], bf16_storage: bool = False,
               keep: Optional[Dict] = None):
    """All blocks of all requests; blocks keep their input order."""
    out_tok = [None] * len(blocks)
    out_max = [None] * len(blocks)
    for r in sorted({b.req for b in blocks}):
        idx = [i for i, b in enumerate(blocks) if b.req == r]
        sub_keep = {} if keep is not None else None
        t, m = draft_request(cfg, weights, states[r], [blocks[i] for i in idx],
                             bf16_storage, sub_keep)
        for j, i in enumerate(idx):
            out_tok[i] = t[j]
            out_max[i] = m[j]
            if keep is not None:
                for key, vals in sub_keep.items():
                    keep.setdefault(key, {})[i] = vals[j]
    return np.stack(out_tok), np.stack(out_max)
