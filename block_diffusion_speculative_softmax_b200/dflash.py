"""Python binding of libdflash.so (ctypes).

Argument marshalling only: every step of the draft pass runs in the CUDA
kernels behind the C ABI declared in include/dflash.h.  PyTorch provides
device memory and streams.  There is no fallback: if the library cannot be
loaded, every call raises.

Typical use (one draft step + verification per decoding step)::

    from block_diffusion_speculative_softmax_b200 import build, dflash as DF
    build.build()                                   # compiles libdflash.so once
    cfg = DF.make_config(hidden=2560, n_q_heads=32, n_kv_heads=8, head_dim=128,
                         ffn=9728, n_draft_layers=5, n_target_layers=5, block=16,
                         vocab=151936)              # bf16, mask id V-1, theta 1e6
    w = DF.DeviceWeights(cfg, host_weights)         # dict of numpy arrays, see synth.make_weights
    buf = DF.StepBuffers(cfg, ctx_lens, n_blocks)   # KV caches, block and output buffers
    ws = DF.alloc_workspace(DF.dflash_workspace_size(cfg, len(ctx_lens), n_blocks,
                                                     n_ctx_new, max(ctx_lens)))
    # fill buf.block_tokens (anchor in slot 0), buf.block_req, buf.known_len,
    # and buf.target_tokens with the target's argmax tokens; new_states holds
    # the target states [n_ctx_new][T][H] of the context rows to (re)fuse:
    DF.dflash_draft_step(cfg, w, buf, new_states, ws, verify=True)
    DF.dflash_check(ws)                              # device-side errors, if any
    # buf.draft_tokens, buf.n_acc, buf.best_k and buf.out_tok hold the result

``block_diffusion_speculative_softmax_b200.workload.Workload`` builds all of
this from the seeded synthetic inputs of a named configuration.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# DFLASH_LIB selects another build of the same ABI (e.g. the debug-bounds
# libdflash_debug.so that `build --debug-bounds` writes beside this one).
LIB_PATH = os.environ.get("DFLASH_LIB") or os.path.join(_HERE, "libdflash.so")

OK, EINVAL, EUNSUPPORTED, ECUDA, ETIMEOUT, ENUMERIC, EBOUNDS = range(7)
STATUS_NAMES = {0: "OK", 1: "EINVAL", 2: "EUNSUPPORTED", 3: "ECUDA", 4: "ETIMEOUT",
                5: "ENUMERIC", 6: "EBOUNDS"}
FP32, BF16 = 0, 1


class DFlashError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Config(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("n_q_heads", C.c_int32), ("n_kv_heads", C.c_int32),
                ("head_dim", C.c_int32), ("ffn", C.c_int32), ("n_draft_layers", C.c_int32),
                ("n_target_layers", C.c_int32), ("block", C.c_int32), ("vocab", C.c_int32),
                ("mask_token_id", C.c_int32), ("rope_theta", C.c_float),
                ("rms_eps", C.c_float), ("dtype", C.c_int32)]


class LayerWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("w_q", "w_kt", "w_vt", "w_kd", "w_vd", "w_o",
                                          "w_gate", "w_up", "w_down", "g_fuse", "g_attn",
                                          "g_mlp")]


class Weights(C.Structure):
    _fields_ = [("w_fuse", C.c_void_p), ("layers", C.POINTER(LayerWeights)),
                ("embed", C.c_void_p), ("g_final", C.c_void_p), ("lm_head", C.c_void_p),
                ("w_fc", C.c_void_p), ("g_fc", C.c_void_p)]


class StepArgs(C.Structure):
    _fields_ = [("n_req", C.c_int32), ("n_blocks", C.c_int32), ("n_ctx_new", C.c_int64),
                ("max_ctx_len", C.c_int64), ("block_req", C.c_void_p),
                ("block_tokens", C.c_void_p), ("known_len", C.c_void_p),
                ("new_states", C.c_void_p), ("ctx_off", C.c_void_p), ("new_off", C.c_void_p),
                ("ctx_cached", C.c_void_p), ("k_cache", C.POINTER(C.c_void_p)),
                ("v_cache", C.POINTER(C.c_void_p)), ("draft_tokens", C.c_void_p),
                ("max_logit", C.c_void_p), ("confidence", C.c_void_p),
                ("target_tokens", C.c_void_p),
                ("n_cand", C.c_int32), ("n_acc", C.c_void_p), ("best_k", C.c_void_p),
                ("out_tok", C.c_void_p), ("sample", C.c_int32), ("rng_offset", C.c_uint32),
                ("seed", C.c_uint64), ("draft_logits", C.c_void_p), ("draft_logq", C.c_void_p),
                ("target_logp", C.c_void_p), ("ctx_len", C.c_void_p),
                ("new_count", C.c_void_p)]


_VP, _I32, _I64, _SZ = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
_CFG = C.POINTER(Config)

# name -> (restype, argtypes); mirrors include/dflash.h
SIGNATURES = {
    "dflash_workspace_size": (_SZ, [_CFG, _I32, _I32, _I64, _I64]),
    "dflash_workspace_init": (C.c_int, [_VP, _SZ, _VP]),
    "dflash_check": (C.c_int, [_VP, _VP]),
    "dflash_last_error": (C.c_char_p, []),
    "dflash_launch_count": (C.c_uint64, []),
    "dflash_version": (C.c_char_p, []),
    "dflash_fuse_ctx": (C.c_int, [_CFG, _VP, _I64, _VP, C.POINTER(_VP), _VP, _VP]),
    "dflash_fc_fuse_ctx": (C.c_int, [_CFG, _VP, _I64, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "dflash_fuse_rss_parts": (C.c_int32, [C.c_int32]),
    "dflash_fuse_ctx_rss": (C.c_int, [_CFG, _VP, _I64, _VP, C.POINTER(_VP), _VP, _VP, _VP, _SZ,
                                      _VP]),
    "dflash_kv_project": (C.c_int, [_CFG, _VP, _I64, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ,
                                    _VP]),
    "dflash_block_attn": (C.c_int, [_CFG, _I32, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I64, _VP,
                                    _VP, _SZ, _VP]),
    "dflash_mlp": (C.c_int, [_CFG, _I64, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "dflash_lmhead_argmax": (C.c_int, [_CFG, _I64, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "dflash_lmhead_logits": (C.c_int, [_CFG, _I64, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "dflash_sample": (C.c_int, [_CFG, _I64, _VP, C.c_uint64, C.c_uint32, _VP, _VP, _VP, _VP]),
    "dflash_accept_stochastic": (C.c_int, [_I32, _I32, _I32, _VP, _VP, _VP, _VP, C.c_uint64,
                                           C.c_uint32, _VP, _VP, _VP, _SZ, _VP]),
    "dflash_accept": (C.c_int, [_I32, _I32, _I32, _VP, _VP, _VP, _VP, _VP, _VP]),
    "dflash_d2sd_candidates": (C.c_int, [_I32, _I32, _I32, _I32, _VP, _VP, _VP, _VP, _VP,
                                         _VP]),
    "dflash_draft_step": (C.c_int, [_CFG, C.POINTER(Weights), C.POINTER(StepArgs), _VP, _SZ,
                                    _VP]),
    "dflash_selftest_wait_timeout": (C.c_int, [_VP, _SZ, _I64, _VP]),
    "dflash_advance": (C.c_int, [_CFG, _I32, _I32, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                 _VP, _VP, _SZ, _VP]),
    "dflash_lmhead_argmax_noalloc": (C.c_int, [_CFG, _I64, _VP, _VP, _VP, _VP, _VP]),
}

_lib = None


def load(path: str = LIB_PATH) -> C.CDLL:
    """Load libdflash.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with "
            "`python -m block_diffusion_speculative_softmax_b200.build`")
    lib = C.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int):
    if status != OK:
        msg = load().dflash_last_error()
        raise DFlashError(status, msg.decode() if msg else "")


def _p(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def make_config(hidden, n_q_heads, n_kv_heads, head_dim, ffn, n_draft_layers, n_target_layers,
                block, vocab, mask_token_id=None, rope_theta=1e6, rms_eps=1e-6,
                dtype="bf16") -> Config:
    return Config(hidden, n_q_heads, n_kv_heads, head_dim, ffn, n_draft_layers,
                  n_target_layers, block, vocab,
                  vocab - 1 if mask_token_id is None else mask_token_id, rope_theta, rms_eps,
                  BF16 if dtype in ("bf16", BF16, torch.bfloat16) else FP32)


def config_from(cfg) -> Config:
    """Config from an object with the synthetic-config field names."""
    return make_config(cfg.hidden, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.ffn,
                       cfg.n_draft_layers, cfg.n_target_layers, cfg.block, cfg.vocab,
                       cfg.mask_token_id, cfg.rope_theta, cfg.rms_eps, cfg.dtype)


def torch_dtype(cfg: Config):
    return torch.bfloat16 if cfg.dtype == BF16 else torch.float32


# ---------------------------------------------------------------- workspace

def dflash_workspace_size(cfg: Config, n_req: int, n_blocks: int, n_ctx_new: int,
                          max_ctx_len: int) -> int:
    n = load().dflash_workspace_size(C.byref(cfg), n_req, n_blocks, n_ctx_new, max_ctx_len)
    if n == 0:
        raise DFlashError(EINVAL, "invalid config for workspace sizing")
    return int(n)


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    ws = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + nbytes]
    dflash_workspace_init(ws)
    return ws


def dflash_workspace_init(ws: torch.Tensor, stream=None):
    _check(load().dflash_workspace_init(_p(ws), ws.numel(), _stream(stream)))


def dflash_check(ws: torch.Tensor, stream=None):
    _check(load().dflash_check(_p(ws), _stream(stream)))


def dflash_launch_count() -> int:
    return int(load().dflash_launch_count())


def dflash_version() -> str:
    return load().dflash_version().decode()


# ---------------------------------------------------------------- single ops

def dflash_fuse_ctx(cfg: Config, states: torch.Tensor, w_fuse: torch.Tensor,
                    g_fuse: Sequence[torch.Tensor], fused: torch.Tensor, stream=None):
    arr = (C.c_void_p * len(g_fuse))(*[g.data_ptr() for g in g_fuse])
    _check(load().dflash_fuse_ctx(C.byref(cfg), _p(states), states.shape[0], _p(w_fuse), arr,
                                  _p(fused), _stream(stream)))


def dflash_fuse_rss_parts(hidden: int) -> int:
    return int(load().dflash_fuse_rss_parts(hidden))


def dflash_fuse_ctx_rss(cfg: Config, states: torch.Tensor, w_fuse: torch.Tensor,
                        g_fuse: Sequence[torch.Tensor], fused: torch.Tensor, rss: torch.Tensor,
                        ws, stream=None):
    arr = (C.c_void_p * len(g_fuse))(*[g.data_ptr() for g in g_fuse])
    _check(load().dflash_fuse_ctx_rss(C.byref(cfg), _p(states), states.shape[0], _p(w_fuse), arr,
                                      _p(fused), _p(rss), _p(ws), ws.numel(), _stream(stream)))


def dflash_fc_fuse_ctx(cfg: Config, states: torch.Tensor, w_fc: torch.Tensor,
                       g_fc: torch.Tensor, fused: torch.Tensor, ws, stream=None):
    _check(load().dflash_fc_fuse_ctx(C.byref(cfg), _p(states), states.shape[0], _p(w_fc),
                                     _p(g_fc), _p(fused), _p(ws), ws.numel(), _stream(stream)))


def dflash_kv_project(cfg: Config, x, pos, dst_row, w_k, w_v, k_out, v_out, ws, stream=None):
    _check(load().dflash_kv_project(C.byref(cfg), _p(x), x.shape[0], _p(pos), _p(dst_row),
                                    _p(w_k), _p(w_v), _p(k_out), _p(v_out), _p(ws), ws.numel(),
                                    _stream(stream)))


def dflash_block_attn(cfg: Config, n_blocks, q, k_blk, v_blk, k_ctx, v_ctx, ctx_off, block_req,
                      max_ctx_len, out, ws, stream=None):
    _check(load().dflash_block_attn(C.byref(cfg), n_blocks, _p(q), _p(k_blk), _p(v_blk),
                                    _p(k_ctx), _p(v_ctx), _p(ctx_off), _p(block_req),
                                    max_ctx_len, _p(out), _p(ws), ws.numel(), _stream(stream)))


def dflash_mlp(cfg: Config, h, g_mlp, w_gate, w_up, w_down, ws, stream=None):
    _check(load().dflash_mlp(C.byref(cfg), h.shape[0], _p(h), _p(g_mlp), _p(w_gate), _p(w_up),
                             _p(w_down), _p(ws), ws.numel(), _stream(stream)))


def dflash_lmhead_argmax(cfg: Config, x, w_lm, tok, max_logit, ws, stream=None, conf=None):
    _check(load().dflash_lmhead_argmax(C.byref(cfg), x.shape[0], _p(x), _p(w_lm), _p(tok),
                                       _p(max_logit), _p(conf), _p(ws), ws.numel(),
                                       _stream(stream)))


def dflash_lmhead_argmax_noalloc(cfg: Config, x, w_lm, tok, max_logit=None, stream=None):
    """LM-head argmax without a workspace, for callers that cannot allocate
    device memory (scratch lives in the library's device globals; at most
    4096 tokens per call; concurrent calls on one device race)."""
    _check(load().dflash_lmhead_argmax_noalloc(C.byref(cfg), x.shape[0], _p(x), _p(w_lm),
                                               _p(tok), _p(max_logit), _stream(stream)))


def dflash_lmhead_logits(cfg: Config, x, w_lm, logits, ws, stream=None):
    _check(load().dflash_lmhead_logits(C.byref(cfg), x.shape[0], _p(x), _p(w_lm), _p(logits),
                                       _p(ws), ws.numel(), _stream(stream)))


def dflash_sample(cfg: Config, logits, seed: int, offset: int, tok, logq=None, lse=None,
                  stream=None):
    _check(load().dflash_sample(C.byref(cfg), logits.shape[0], _p(logits), seed, offset,
                                _p(tok), _p(logq), _p(lse), _stream(stream)))


def dflash_accept_stochastic(draft, draft_logits, draft_lse, target_logp, seed: int,
                             offset: int, n_acc, out_tok, ws, stream=None):
    R, B, V = draft_logits.shape
    _check(load().dflash_accept_stochastic(R, B, V, _p(draft), _p(draft_logits), _p(draft_lse),
                                           _p(target_logp), seed, offset, _p(n_acc),
                                           _p(out_tok), _p(ws), ws.numel(), _stream(stream)))


def dflash_accept(draft: torch.Tensor, target: torch.Tensor, n_acc, best_k, out_tok,
                  stream=None):
    R, K, B = draft.shape
    _check(load().dflash_accept(R, K, B, _p(draft), _p(target), _p(n_acc), _p(best_k),
                                _p(out_tok), _stream(stream)))


def dflash_d2sd_candidates(base_tokens, conf, K, mask_token_id, known_len, cand_tokens,
                           block_req=None, stream=None):
    R, B = base_tokens.shape
    _check(load().dflash_d2sd_candidates(R, B, K, mask_token_id, _p(base_tokens), _p(conf),
                                         _p(known_len), _p(cand_tokens), _p(block_req),
                                         _stream(stream)))


def dflash_advance(cfg: Config, n_acc, best_k, out_tok, verify_states, ctx_len, ctx_off,
                   new_states, new_count, block_tokens, known_len, ws, stream=None):
    """Roll every request's window forward on the device (see dflash.h).
    verify_states [R][K][B][T][H]; new_states [R][B][T][H]."""
    R, K = verify_states.shape[0], verify_states.shape[1]
    _check(load().dflash_advance(C.byref(cfg), R, K, _p(n_acc), _p(best_k), _p(out_tok),
                                 _p(verify_states), _p(ctx_len), _p(ctx_off), _p(new_states),
                                 _p(new_count), _p(block_tokens), _p(known_len), _p(ws),
                                 ws.numel(), _stream(stream)))


def dflash_selftest_wait_timeout(ws, limit_ns: int, stream=None):
    _check(load().dflash_selftest_wait_timeout(_p(ws), ws.numel(), limit_ns, _stream(stream)))


# ---------------------------------------------------------------- draft step

class DeviceWeights:
    """Draft weights resident on the device plus the C structs that point at
    them (kept alive together)."""

    def __init__(self, cfg: Config, host: dict, device="cuda"):
        dt = torch_dtype(cfg)
        f32 = torch.float32

        def dev(a, dtype):
            return torch.as_tensor(a).to(device=device, dtype=dtype).contiguous()

        self.w_fuse = dev(host["w_fuse"], f32)
        # DFlash FC fusion (optional): one shared context for every layer
        self.w_fc = dev(host["w_fc"], dt) if "w_fc" in host else None
        self.g_fc = dev(host["g_fc"], f32) if "w_fc" in host else None
        self.embed = dev(host["embed"], dt)
        self.lm_head = dev(host["lm_head"], dt)
        self.g_final = dev(host["g_final"], f32)
        self.layers = []
        for lay in host["layers"]:
            d = {}
            for k in ("w_q", "w_kt", "w_vt", "w_kd", "w_vd", "w_o", "w_gate", "w_up", "w_down"):
                d[k] = dev(lay[k], dt)
            for k in ("g_fuse", "g_attn", "g_mlp"):
                d[k] = dev(lay[k], f32)
            self.layers.append(d)
        n = len(self.layers)
        self._lw = (LayerWeights * n)(*[
            LayerWeights(*[d[k].data_ptr() for k in (
                "w_q", "w_kt", "w_vt", "w_kd", "w_vd", "w_o", "w_gate", "w_up", "w_down",
                "g_fuse", "g_attn", "g_mlp")]) for d in self.layers])
        self.struct = Weights(self.w_fuse.data_ptr(), self._lw, self.embed.data_ptr(),
                              self.g_final.data_ptr(), self.lm_head.data_ptr(),
                              None if self.w_fc is None else self.w_fc.data_ptr(),
                              None if self.g_fc is None else self.g_fc.data_ptr())

    def nbytes(self) -> int:
        tot = sum(t.numel() * t.element_size() for t in (self.w_fuse, self.embed, self.lm_head,
                                                        self.g_final, self.w_fc, self.g_fc)
                  if t is not None)
        for d in self.layers:
            tot += sum(t.numel() * t.element_size() for t in d.values())
        return tot


class StepBuffers:
    """Device buffers of one draft step (inputs, caches, outputs)."""

    def __init__(self, cfg: Config, ctx_lens: List[int], n_blocks: int, n_cand: int = 1,
                 device="cuda", share_caches: Optional["StepBuffers"] = None):
        D = cfg.n_draft_layers
        kvd = cfg.n_kv_heads * cfg.head_dim
        dt = torch_dtype(cfg)
        self.cfg = cfg
        self.R = len(ctx_lens)
        self.nb = n_blocks
        self.n_cand = n_cand
        self.ctx_lens = list(ctx_lens)
        off = [0]
        for L in ctx_lens:
            off.append(off[-1] + L)
        self.sum_L = off[-1]
        self.max_L = max(ctx_lens) if ctx_lens else 0
        self.ctx_off = torch.tensor(off, dtype=torch.int64, device=device)
        rows = max(1, self.sum_L)
        if share_caches is not None:
            self.k_cache, self.v_cache = share_caches.k_cache, share_caches.v_cache
        else:
            self.k_cache = [torch.zeros(rows, kvd, dtype=dt, device=device) for _ in range(D)]
            self.v_cache = [torch.zeros(rows, kvd, dtype=dt, device=device) for _ in range(D)]
        self._kc = (C.c_void_p * D)(*[t.data_ptr() for t in self.k_cache])
        self._vc = (C.c_void_p * D)(*[t.data_ptr() for t in self.v_cache])
        B = cfg.block
        self.block_req = torch.zeros(n_blocks, dtype=torch.int32, device=device)
        self.block_tokens = torch.zeros(n_blocks, B, dtype=torch.int32, device=device)
        self.known_len = torch.ones(n_blocks, dtype=torch.int32, device=device)
        self.draft_tokens = torch.zeros(n_blocks, B, dtype=torch.int32, device=device)
        self.max_logit = torch.zeros(n_blocks, B, dtype=torch.float32, device=device)
        self.confidence = torch.zeros(n_blocks, B, dtype=torch.float32, device=device)
        self.target_tokens = torch.zeros(n_blocks, B, dtype=torch.int32, device=device)
        self.n_acc = torch.zeros(self.R, dtype=torch.int32, device=device)
        self.best_k = torch.zeros(self.R, dtype=torch.int32, device=device)
        self.out_tok = torch.zeros(self.R, B, dtype=torch.int32, device=device)
        self.draft_logits = None      # temperature-1 mode buffers (alloc_sampling)
        self.draft_logq = None
        self.target_logp = None

    def alloc_sampling(self, device="cuda"):
        """Buffers of the temperature-1 mode: the draft's logits and log
        probabilities per slot and the target's log probabilities."""
        B, V = self.cfg.block, self.cfg.vocab
        self.draft_logits = torch.zeros(self.nb, B, V, dtype=torch.float32, device=device)
        self.draft_logq = torch.zeros(self.nb, B, dtype=torch.float32, device=device)
        self.target_logp = torch.zeros(self.nb, B, V, dtype=torch.float32, device=device)


def dflash_draft_step(cfg: Config, w: DeviceWeights, buf: StepBuffers,
                      new_states: Optional[torch.Tensor], ws: torch.Tensor,
                      new_off: Optional[torch.Tensor] = None,
                      ctx_cached: Optional[torch.Tensor] = None, verify: bool = False,
                      stream=None, confidence: bool = False, sample: bool = False,
                      seed: int = 0, rng_offset: int = 0,
                      ctx_len: Optional[torch.Tensor] = None,
                      new_count: Optional[torch.Tensor] = None,
                      max_ctx_len: Optional[int] = None):
    """One draft step over ``buf``'s blocks.  ``new_states`` [n_new][T][H]
    holds the target states of the context rows to (re)compute: all rows
    (``ctx_cached`` None) or rows [cached_r, L_r) of every request."""
    n_new = 0 if new_states is None else int(new_states.shape[0])
    a = StepArgs()
    a.n_req = buf.R
    a.n_blocks = buf.nb
    a.n_ctx_new = n_new
    a.max_ctx_len = buf.max_L if max_ctx_len is None else max_ctx_len
    a.block_req = buf.block_req.data_ptr()
    a.block_tokens = buf.block_tokens.data_ptr()
    a.known_len = buf.known_len.data_ptr()
    a.new_states = None if new_states is None else new_states.data_ptr()
    a.ctx_off = buf.ctx_off.data_ptr()
    a.new_off = None if new_off is None else new_off.data_ptr()
    a.ctx_cached = None if ctx_cached is None else ctx_cached.data_ptr()
    a.k_cache = buf._kc
    a.v_cache = buf._vc
    a.draft_tokens = buf.draft_tokens.data_ptr()
    a.max_logit = buf.max_logit.data_ptr()
    a.confidence = buf.confidence.data_ptr() if confidence else None
    a.target_tokens = buf.target_tokens.data_ptr() if verify else None
    a.n_cand = buf.n_cand
    a.n_acc = buf.n_acc.data_ptr()
    a.best_k = buf.best_k.data_ptr()
    a.out_tok = buf.out_tok.data_ptr()
    a.ctx_len = None if ctx_len is None else ctx_len.data_ptr()
    a.new_count = None if new_count is None else new_count.data_ptr()
    if sample:
        a.sample = 1
        a.seed = seed
        a.rng_offset = rng_offset
        a.draft_logits = buf.draft_logits.data_ptr()
        a.draft_logq = buf.draft_logq.data_ptr()
        a.target_logp = buf.target_logp.data_ptr() if verify else None
        a.target_tokens = None
    _check(load().dflash_draft_step(C.byref(cfg), C.byref(w.struct), C.byref(a), _p(ws),
                                    ws.numel(), _stream(stream)))
