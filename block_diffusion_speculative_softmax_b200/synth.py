"""Seeded synthetic inputs for the block-diffusion draft step.

This module only draws random numbers and lays them out.  It holds none of
the draft step's arithmetic (no fusion, norm, projection, attention, MLP,
argmax or acceptance), so both the CUDA path and the CPU oracle can take
their inputs from here without sharing any of the method.

Recipe (DFlash summary, "Methodology"; DFLARE summary, sections 2.1-2.2):

* target hidden states ~ N(0, 1), shape [L][T][H] per request;
* every weight matrix ~ N(0, 0.02), stored [out][in];
* W_fuse ~ N(0, 1), shape [D][T];
* every RMSNorm gain = 1 + N(0, 0.02) (a pure N(0, 0.02) gain would shrink
  the logits to ~0.02 and turn every argmax into a near-tie);
* anchors (last accepted token) uniform over [0, V-2]; the mask id is V-1;
* target argmax tokens are planted so that the draft's accepted prefix has a
  truncated geometric length (see ``plant_targets``);
* D2SD per-position confidences ~ U(0, 1).

bf16 configurations draw in fp32 and round to bf16 (round to nearest even)
so that the host copy holds exactly the bits that are uploaded.  Every array
comes from ``numpy.random.default_rng([seed, config_index, stream])`` so a
single request can be regenerated without drawing the others.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np

__all__ = [
    "DraftConfig", "CONFIGS", "CONFIG_ORDER", "get_config", "to_bf16_bits",
    "round_bf16", "make_weights", "make_fc_weights", "make_states", "ctx_lengths", "make_anchors",
    "make_confidence", "geometric_lengths", "plant_targets",
    "plant_targets_d2sd", "small_config",
]


@dataclasses.dataclass(frozen=True)
class DraftConfig:
    name: str
    index: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    n_draft_layers: int
    n_target_layers: int
    ctx_len: int            # context length L (max for ragged configs)
    block: int              # block length B
    vocab: int
    dtype: str              # "fp32" or "bf16"
    n_req: int = 1
    n_cand: int = 1         # D2SD candidates per request (K)
    ctx_len_min: int = 0    # > 0: ragged L ~ U[ctx_len_min, ctx_len]
    accept_p: float = 0.15552  # per-position stop probability of the planted prefix
    rope_theta: float = 1.0e6
    rms_eps: float = 1.0e-6

    @property
    def mask_token_id(self) -> int:
        return self.vocab - 1

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def n_blocks(self) -> int:
        return self.n_req * self.n_cand


# The five workloads: a tiny fp32 model, a Qwen3-4B-shaped draft, a Qwen3-8B
# shaped DFLARE draft (per-layer alpha over 9 target layers, separate W^t/W^d),
# 32 ragged serving requests on the 8B shapes, and D2SD multi-candidate
# drafting on GPT-OSS-20B-like shapes.
CONFIGS: Dict[str, DraftConfig] = {
    "tiny": DraftConfig("tiny", 0, 256, 4, 2, 64, 512, 2, 3, 64, 8, 1024,
                        "fp32", accept_p=0.25),
    "qwen3_4b": DraftConfig("qwen3_4b", 1, 2560, 32, 8, 128, 9728, 5, 5,
                            2048, 16, 151936, "bf16"),
    "qwen3_8b_dflare": DraftConfig("qwen3_8b_dflare", 2, 4096, 32, 8, 128,
                                   12288, 7, 9, 4096, 16, 151936, "bf16"),
    "serving32": DraftConfig("serving32", 3, 4096, 32, 8, 128, 12288, 7, 9,
                             8192, 16, 151936, "bf16", n_req=32,
                             ctx_len_min=512),
    "d2sd_gptoss": DraftConfig("d2sd_gptoss", 4, 2880, 64, 8, 64, 2880, 5, 5,
                               2048, 16, 201088, "bf16", n_req=8, n_cand=4),
}
CONFIG_ORDER: List[str] = ["tiny", "qwen3_4b", "qwen3_8b_dflare", "serving32",
                           "d2sd_gptoss"]


def get_config(name: str) -> DraftConfig:
    return CONFIGS[name]


def small_config(base: str = "qwen3_4b", **over) -> DraftConfig:
    """A shrunken copy of a named config (for parity tests that must finish
    on the CPU oracle in seconds).  ``index`` is kept so seeds differ from
    the full-size draw only through the shapes."""
    return dataclasses.replace(CONFIGS[base], name=base + "_small", **over)


# --------------------------------------------------------------------------
# bf16 storage of inputs
# --------------------------------------------------------------------------

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even.
    Inputs are finite (they are Gaussian draws)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 array whose values are exactly representable in bf16."""
    bits = to_bf16_bits(x).astype(np.uint32) << 16
    return bits.view(np.float32)


def _rng(cfg: DraftConfig, seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([seed, cfg.index, stream])


def _draw(rng: np.random.Generator, shape, scale: float, cfg: DraftConfig,
          shift: float = 0.0) -> np.ndarray:
    a = rng.standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        a *= np.float32(scale)
    if shift != 0.0:
        a += np.float32(shift)
    if cfg.dtype == "bf16":
        a = round_bf16(a)
    return a


# Stream ids: weights of layer i use 100 + i, global weights 10..13,
# request r uses 1000 + r (states) and 5000 + r (tokens/acceptance).
def make_weights(cfg: DraftConfig, seed: int = 0,
                 separate_kv: bool = True) -> dict:
    """All draft weights as fp32 numpy arrays (bf16-exact for bf16 configs).

    ``separate_kv=False`` returns W^t_K = W^d_K and W^t_V = W^d_V (the shared
    projection of the DFlash baseline)."""
    H, F, qd, kvd = cfg.hidden, cfg.ffn, cfg.q_dim, cfg.kv_dim
    D, T, V = cfg.n_draft_layers, cfg.n_target_layers, cfg.vocab
    g = _rng(cfg, seed, 10)
    w = {
        "w_fuse": g.standard_normal((D, T), dtype=np.float32),
        "embed": _draw(_rng(cfg, seed, 11), (V, H), 0.02, cfg),
        "lm_head": _draw(_rng(cfg, seed, 12), (V, H), 0.02, cfg),
        "g_final": _draw(_rng(cfg, seed, 13), (H,), 0.02, cfg, 1.0),
        "layers": [],
    }
    for i in range(D):
        r = _rng(cfg, seed, 100 + i)
        lay = {
            "w_q": _draw(r, (qd, H), 0.02, cfg),
            "w_kt": _draw(r, (kvd, H), 0.02, cfg),
            "w_vt": _draw(r, (kvd, H), 0.02, cfg),
            "w_kd": _draw(r, (kvd, H), 0.02, cfg),
            "w_vd": _draw(r, (kvd, H), 0.02, cfg),
            "w_o": _draw(r, (H, qd), 0.02, cfg),
            "w_gate": _draw(r, (F, H), 0.02, cfg),
            "w_up": _draw(r, (F, H), 0.02, cfg),
            "w_down": _draw(r, (H, F), 0.02, cfg),
            "g_fuse": _draw(r, (H,), 0.02, cfg, 1.0),
            "g_attn": _draw(r, (H,), 0.02, cfg, 1.0),
            "g_mlp": _draw(r, (H,), 0.02, cfg, 1.0),
        }
        if not separate_kv:
            lay["w_kt"] = lay["w_kd"]
            lay["w_vt"] = lay["w_vd"]
        w["layers"].append(lay)
    return w


def make_fc_weights(cfg: DraftConfig, seed: int = 0) -> dict:
    """Weights of the DFlash-style FC context fusion: w_fc [H][T*H] ~
    N(0, 0.02) and its RMSNorm gain g_fc = 1 + N(0, 0.02) (streams 14, 15).
    Add them to a ``make_weights`` dict to select that variant."""
    H, T = cfg.hidden, cfg.n_target_layers
    return {"w_fc": _draw(_rng(cfg, seed, 14), (H, T * H), 0.02, cfg),
            "g_fc": _draw(_rng(cfg, seed, 15), (H,), 0.02, cfg, 1.0)}


def ctx_lengths(cfg: DraftConfig, seed: int = 0) -> List[int]:
    """Context length per request: fixed L, or seeded ragged U[min, L]."""
    if cfg.ctx_len_min <= 0:
        return [cfg.ctx_len] * cfg.n_req
    g = _rng(cfg, seed, 20)
    return [int(v) for v in g.integers(cfg.ctx_len_min, cfg.ctx_len + 1,
                                       size=cfg.n_req)]


def make_states(cfg: DraftConfig, seed: int, req: int, length: int,
                start: int = 0) -> np.ndarray:
    """Target hidden states [length][T][H] of request ``req`` for context
    positions [start, start + length).  Rows are drawn position by position
    from one stream, so any window of a request is reproducible."""
    T, H = cfg.n_target_layers, cfg.hidden
    g = _rng(cfg, seed, 1000 + req)
    if start:
        g.standard_normal((start, T, H), dtype=np.float32)  # skip
    return _draw(g, (length, T, H), 1.0, cfg)


def make_anchors(cfg: DraftConfig, seed: int = 0) -> np.ndarray:
    """Last accepted token per request, uniform over [0, V-2]."""
    g = _rng(cfg, seed, 30)
    return g.integers(0, cfg.vocab - 1, size=cfg.n_req).astype(np.int32)


def make_confidence(cfg: DraftConfig, seed: int = 0) -> np.ndarray:
    """D2SD per-position confidence [R][B] ~ U(0, 1) (float32)."""
    g = _rng(cfg, seed, 40)
    return g.random((cfg.n_req, cfg.block), dtype=np.float32)


def geometric_lengths(p: float, n: int, cap: int,
                      rng: np.random.Generator) -> np.ndarray:
    """min(G, cap) with G = failures before the first success, P(success)=p."""
    g = rng.geometric(p, size=n) - 1
    return np.minimum(g, cap).astype(np.int32)


def _other_token(rng: np.random.Generator, avoid: int, vocab: int) -> int:
    t = int(rng.integers(0, vocab - 1))
    return t + 1 if t >= avoid else t


def plant_targets(draft: np.ndarray, n_plant: np.ndarray, vocab: int,
                  rng: np.random.Generator) -> np.ndarray:
    """Target argmax tokens for draft blocks ``draft[R][B]`` such that
    exactly ``n_plant[r]`` draft tokens are accepted.

    t[j-1] = d[j] for 1 <= j <= n; t[n] differs from d[n+1] (when slot n+1
    exists); every other target token is uniform over the vocabulary."""
    R, B = draft.shape
    t = rng.integers(0, vocab, size=(R, B)).astype(np.int32)
    for r in range(R):
        n = int(n_plant[r])
        for j in range(1, n + 1):
            t[r, j - 1] = draft[r, j]
        if n + 1 < B:
            t[r, n] = _other_token(rng, int(draft[r, n + 1]), vocab)
    return t


def plant_targets_d2sd(cand: np.ndarray, n_plant: np.ndarray, vocab: int,
                       rng: np.random.Generator,
                       known_len: Optional[np.ndarray] = None) -> np.ndarray:
    """Target tokens for K candidate blocks per request ``cand[R][K][B]``.

    One planted candidate k_p per request defines a true continuation y:
    y[0..m] = cand[k_p][0..m] with m = n_plant[r], y[m+1] differs from
    cand[k_p][m+1], later y uniform.  The target's prediction after a prefix
    is a function of that prefix only: for every candidate, t_k[j] = y[j+1]
    while cand_k[0..j] equals y[0..j]; while the prefix still lies inside
    the base block shared by all candidates (slot j+1 < known_len[k]) a
    per-request random token is used; otherwise a fresh uniform token."""
    R, K, B = cand.shape
    t = np.zeros((R, K, B), dtype=np.int32)
    for r in range(R):
        kp = int(rng.integers(0, K))
        m = int(n_plant[r])
        y = rng.integers(0, vocab, size=B + 1).astype(np.int64)
        y[: m + 1] = cand[r, kp, : m + 1]
        if m + 1 < B:
            y[m + 1] = _other_token(rng, int(cand[r, kp, m + 1]), vocab)
        shared = rng.integers(0, vocab, size=B).astype(np.int64)
        for k in range(K):
            kl = B if known_len is None else int(known_len[r * K + k])
            match = True
            for j in range(B):
                match = match and int(cand[r, k, j]) == int(y[j])
                if match:
                    t[r, k, j] = y[j + 1]
                elif j + 1 < kl:
                    t[r, k, j] = shared[j]
                else:
                    t[r, k, j] = int(rng.integers(0, vocab))
    return t


def accept_p_for_mean(mean_n: float, cap: int) -> float:
    """Per-position stop probability p whose truncated geometric length
    min(G, cap) has expectation ``mean_n`` (bisection)."""
    def mean(p):
        q = 1.0 - p
        return q * (1.0 - q ** cap) / p
    lo, hi = 1e-6, 1.0 - 1e-9
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if mean(mid) > mean_n:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def truncated_geometric_mean(p: float, cap: int) -> float:
    q = 1.0 - p
    return q * (1.0 - q ** cap) / p if p > 0 else float(cap)


def human_bytes(n: float) -> str:
    for unit in ("B", "KB", "MB", "GB", "TB"):
        if abs(n) < 1000:
            return f"{n:.1f} {unit}"
        n /= 1000.0
    return f"{n:.1f} PB"



def make_toy_target_weights(vocab: int, hidden: int, seed: int = 0) -> dict:
    """Integer weights of the toy 2-layer target used by the losslessness
    check: embedding E in [-4, 4], mixing matrices A_l, C_l in {-1, 0, 1}
    (about 30% non-zero) and an output matrix W_out in [-2, 2]."""
    g = np.random.default_rng([seed, 99, 7])

    def tern(shape):
        a = g.integers(-1, 2, size=shape)
        return (a * (g.random(shape) < 0.3)).astype(np.int64)

    return {
        "E": g.integers(-4, 5, size=(vocab, hidden)).astype(np.int64),
        "A1": tern((hidden, hidden)), "C1": tern((hidden, hidden)),
        "A2": tern((hidden, hidden)), "C2": tern((hidden, hidden)),
        "W_out": g.integers(-2, 3, size=(vocab, hidden)).astype(np.int64),
    }


def make_prompt(vocab: int, length: int, seed: int = 0) -> np.ndarray:
    g = np.random.default_rng([seed, 99, 8])
    return g.integers(0, vocab - 1, size=length).astype(np.int32)
