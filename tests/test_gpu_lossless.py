"""Greedy losslessness on the GPU (DFlash summary, key contributions and
methodology steps 3-4): a speculative loop whose draft blocks come from
dflash_draft_step (context KV cached across steps, only the newly accepted
rows fused and projected) and whose verification runs through dflash_accept
emits exactly the tokens of plain greedy decoding from the toy target."""
import numpy as np
import pytest
import torch

from oracle import toy_target as TT
from block_diffusion_speculative_softmax_b200 import synth
from tests.gpu_common import need_gpu

pytestmark = pytest.mark.gpu


def test_gpu_speculative_loop_is_lossless():
    need_gpu()
    from block_diffusion_speculative_softmax_b200 import dflash as DF
    cfg = synth.get_config("tiny")
    ccfg = DF.config_from(cfg)
    B, D = cfg.block, cfg.n_draft_layers
    tw = synth.make_toy_target_weights(cfg.vocab, cfg.hidden, seed=1)
    prompt = synth.make_prompt(cfg.vocab, 20, seed=1)
    n_new = 40
    greedy = TT.greedy(tw, prompt, n_new)

    Lmax = len(prompt) + n_new + B + 1
    w = DF.DeviceWeights(ccfg, synth.make_weights(cfg, seed=1))
    buf = DF.StepBuffers(ccfg, [Lmax], 1)
    ws = DF.alloc_workspace(DF.dflash_workspace_size(ccfg, 1, 1, Lmax, Lmax))
    rng = np.random.default_rng(3)
    seq = [int(t) for t in prompt]
    cached = 0
    steps = 0
    while len(seq) - len(prompt) < n_new:
        L = len(seq) - 1                                   # context rows before the anchor
        st, _ = TT.forward(tw, np.asarray(seq[:-1]))
        buf.ctx_off.copy_(torch.tensor([0, L], dtype=torch.int64))
        buf.max_L = L
        new = torch.from_numpy(np.ascontiguousarray(st[cached:L])).cuda()
        buf.block_tokens.zero_()
        buf.block_tokens[0, 0] = seq[-1]
        DF.dflash_draft_step(ccfg, w, buf, new, ws,
                             new_off=torch.tensor([0, L - cached], dtype=torch.int64,
                                                  device="cuda"),
                             ctx_cached=torch.tensor([cached], dtype=torch.int32, device="cuda"))
        DF.dflash_check(ws)
        cached = L
        d = buf.draft_tokens[0].cpu().numpy().copy()
        assert d[0] == seq[-1]
        m = min(int(rng.geometric(0.3)) - 1, B - 1)        # exercise multi-token acceptance
        if m:
            d[1:m + 1] = TT.greedy(tw, np.asarray(seq), m)
        _, nxt = TT.forward(tw, np.asarray(seq + [int(v) for v in d[1:]]))
        t = nxt[len(seq) - 1:len(seq) - 1 + B].astype(np.int32)
        n = torch.empty(1, dtype=torch.int32, device="cuda")
        out = torch.empty(1, B, dtype=torch.int32, device="cuda")
        DF.dflash_accept(torch.from_numpy(d[None, None]).cuda(),
                         torch.from_numpy(t[None, None]).cuda(), n,
                         torch.empty(1, dtype=torch.int32, device="cuda"), out)
        k = int(n.item())
        seq += [int(v) for v in out[0, :k + 1].cpu().numpy()]
        steps += 1
    got = np.asarray(seq[len(prompt):len(prompt) + n_new])
    np.testing.assert_array_equal(got, greedy)
    assert steps < n_new
