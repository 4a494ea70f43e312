"""Synthetic draft-step workloads on the device.

Builds the device-resident inputs of one configuration from the seeded
generator (``synth``) and drives the C ABI through the binding: one
DFlash/DFLARE draft step over every request, optionally followed by greedy
verification, or the two-pass D2SD step (first draft -> lowest-confidence
cuts -> batched re-anchored second draft over K candidates -> acceptance of
the longest candidate).
"""
from __future__ import annotations

from typing import List, Optional

import numpy as np
import torch

from . import dflash as DF
from . import synth


def _bf16_or_f32(a: np.ndarray, dt) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(dt)


class Workload:
    """All device inputs of ``cfg`` (seeded), the workspace and the output
    buffers.  ``mode``: "full" re-fuses and re-projects every context row in
    every step; "steady" appends ``n_new`` rows per request per step to a
    context whose earlier rows are already in the KV caches."""

    def __init__(self, cfg: synth.DraftConfig, seed: int = 0, device: str = "cuda",
                 mode: str = "full", steady_new_rows: int = 6, host_weights: Optional[dict] = None,
                 keep_host: bool = False, ctx_lens: Optional[List[int]] = None,
                 conf_source: str = "synthetic", sample: bool = False, rng_seed: int = 1):
        self.cfg = cfg
        self.seed = seed
        self.device = device
        self.mode = mode
        self.ccfg = DF.config_from(cfg)
        self.dt = DF.torch_dtype(self.ccfg)
        hw = host_weights if host_weights is not None else synth.make_weights(cfg, seed)
        self.host_weights = hw if keep_host else None
        self.w = DF.DeviceWeights(self.ccfg, hw, device)
        self.ctx_lens = list(ctx_lens) if ctx_lens is not None else synth.ctx_lengths(cfg, seed)
        R, K, B = cfg.n_req, cfg.n_cand, cfg.block
        T, H = cfg.n_target_layers, cfg.hidden
        self.R, self.K = R, K
        # target hidden states of every context row, packed [sum L][T][H]
        self.sum_L = int(sum(self.ctx_lens))
        self.states = torch.empty(max(1, self.sum_L), T, H, dtype=self.dt, device=device)
        o = 0
        for r, L in enumerate(self.ctx_lens):
            if L:
                self.states[o:o + L] = _bf16_or_f32(synth.make_states(cfg, seed, r, L),
                                                    self.dt).to(device)
            o += L
        self.anchors = synth.make_anchors(cfg, seed)
        # pass-1 buffers: one block per request (anchor + masks)
        self.buf = DF.StepBuffers(self.ccfg, self.ctx_lens, R, 1, device)
        tok = np.zeros((R, B), dtype=np.int32)
        tok[:, 0] = self.anchors
        self.buf.block_tokens.copy_(torch.from_numpy(tok))
        self.buf.block_req.copy_(torch.arange(R, dtype=torch.int32))
        # steady-state: only the last n_new rows of every request are new
        self.n_new_rows = min(steady_new_rows, min(self.ctx_lens) if self.ctx_lens else 0)
        if mode == "steady":
            cached = [L - self.n_new_rows for L in self.ctx_lens]
            self.ctx_cached = torch.tensor(cached, dtype=torch.int32, device=device)
            noff = [0]
            idx = []
            o = 0
            for L in self.ctx_lens:
                idx.extend(range(o + L - self.n_new_rows, o + L))
                noff.append(noff[-1] + self.n_new_rows)
                o += L
            self.new_off = torch.tensor(noff, dtype=torch.int64, device=device)
            self.new_states = self.states[torch.tensor(idx, dtype=torch.int64, device=device)]
        else:
            self.ctx_cached = None
            self.new_off = None
            self.new_states = self.states if self.sum_L else None
        n_new = 0 if self.new_states is None else int(self.new_states.shape[0])
        # pass-2 (D2SD) buffers share the KV caches of pass 1
        self.buf2 = None
        if K > 1:
            self.buf2 = DF.StepBuffers(self.ccfg, self.ctx_lens, R * K, K, device,
                                       share_caches=self.buf)
            # per-slot confidence for the D2SD cuts: a seeded U(0,1) field
            # ("synthetic", the workload's stated input), or the first pass's
            # own softmax probability of each drafted token ("draft")
            if conf_source == "draft":
                self.conf = self.buf.confidence
            else:
                self.conf = torch.from_numpy(synth.make_confidence(cfg, seed)).to(device)
            self.cached_all = torch.tensor(self.ctx_lens, dtype=torch.int32, device=device)
        self.conf_source = conf_source if K > 1 else None
        # temperature-1 mode: sampled drafts, stochastic verification
        self.sample = sample
        self.rng_seed = rng_seed
        self.rng_offset = 0
        if sample:
            assert K == 1, "stochastic verification takes one candidate per request"
            self.buf.alloc_sampling(device)
        nb_max = R * K
        self.ws_bytes = DF.dflash_workspace_size(self.ccfg, R, nb_max, n_new, max(self.ctx_lens))
        self.ws = DF.alloc_workspace(self.ws_bytes, device)
        self.n_new = n_new

    # ------------------------------------------------------------ steps
    def draft(self, verify: bool = False, stream=None):
        """Pass 1: one block per request (the DFlash / DFLARE step)."""
        DF.dflash_draft_step(self.ccfg, self.w, self.buf, self.new_states, self.ws,
                             new_off=self.new_off, ctx_cached=self.ctx_cached,
                             verify=verify, stream=stream,
                             confidence=self.conf_source == "draft", sample=self.sample,
                             seed=self.rng_seed, rng_offset=self.rng_offset)

    def candidates(self, stream=None):
        """D2SD cuts from pass-1 tokens into the pass-2 block buffers."""
        b2 = self.buf2
        DF.dflash_d2sd_candidates(self.buf.draft_tokens, self.conf, self.K,
                                  self.cfg.mask_token_id, b2.known_len, b2.block_tokens,
                                  b2.block_req, stream=stream)

    def redraft(self, verify: bool = False, stream=None):
        """Pass 2: all R*K re-anchored candidates in one batched pass over the
        cached context (no new context rows)."""
        DF.dflash_draft_step(self.ccfg, self.w, self.buf2, None, self.ws,
                             ctx_cached=self.cached_all, verify=verify, stream=stream)

    def step(self, verify: bool = True, stream=None):
        """One whole step of the hot path for this configuration."""
        if self.K > 1:
            self.draft(False, stream)
            self.candidates(stream)
            self.redraft(verify, stream)
        else:
            self.draft(verify, stream)

    # ------------------------------------------------------------ planting
    def plant_targets(self, seed_offset: int = 0) -> np.ndarray:
        """Plant target argmax tokens against the current draft tokens so
        that the accepted lengths are truncated-geometric (synthetic stand-in
        for a real target model).  Returns the planted accept lengths."""
        cfg = self.cfg
        rng = np.random.default_rng([self.seed, cfg.index, 7000 + seed_offset])
        n = synth.geometric_lengths(cfg.accept_p, self.R, cfg.block - 1, rng)
        if self.K > 1:
            d = self.buf2.draft_tokens.cpu().numpy().reshape(self.R, self.K, cfg.block)
            kl = self.buf2.known_len.cpu().numpy()
            t = synth.plant_targets_d2sd(d, n, cfg.vocab, rng, kl)
            self.buf2.target_tokens.copy_(torch.from_numpy(t.reshape(self.R * self.K, -1)))
        else:
            d = self.buf.draft_tokens.cpu().numpy()
            t = synth.plant_targets(d, n, cfg.vocab, rng)
            self.buf.target_tokens.copy_(torch.from_numpy(t))
        return n

    def plant_target_logp(self, sigma: float = 0.5, seed_offset: int = 0):
        """Temperature-1 stand-in for the target model: its distribution for
        slot j+1 is the draft's slot j+1 logits perturbed by N(0, sigma^2)
        noise (so drafts are often, not always, accepted), and for the slot
        after the block an unrelated random distribution; stored as log
        probabilities.  Needs the draft logits of a previous step."""
        b = self.buf
        g = torch.Generator(device=b.draft_logits.device)
        g.manual_seed(int(self.seed) * 1000003 + 7919 + seed_offset)
        z = torch.empty_like(b.target_logp)
        z[:, :-1] = b.draft_logits[:, 1:] + sigma * torch.randn(
            b.draft_logits[:, 1:].shape, device=z.device, generator=g)
        z[:, -1] = 2.0 * torch.randn(z[:, -1].shape, device=z.device, generator=g)
        b.target_logp.copy_(torch.log_softmax(z, dim=-1))

    @property
    def final_buf(self):
        return self.buf2 if self.K > 1 else self.buf

    def check(self):
        DF.dflash_check(self.ws)
