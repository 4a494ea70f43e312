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


def test_gpu_device_loop_is_lossless():
    """The same loop with the window rolled forward on the device: each
    decode step is ONE replay of a CUDA graph holding accept -> advance ->
    draft step (context lengths, new-row counts and the next anchor stay in
    device memory; only the newly accepted rows are fused and projected).
    The host only stands in for the target model: it reads the drafted block,
    runs the toy target over it and uploads the target's hidden states and
    argmax tokens for the block's slots."""
    need_gpu()
    from block_diffusion_speculative_softmax_b200 import dflash as DF
    cfg = synth.get_config("tiny")
    ccfg = DF.config_from(cfg)
    B, T, H = cfg.block, cfg.n_target_layers, cfg.hidden
    tw = synth.make_toy_target_weights(cfg.vocab, cfg.hidden, seed=2)
    prompt = synth.make_prompt(cfg.vocab, 20, seed=2)
    n_new = 40
    greedy = TT.greedy(tw, prompt, n_new)

    cap = len(prompt) + n_new + 2 * B
    w = DF.DeviceWeights(ccfg, synth.make_weights(cfg, seed=2))
    buf = DF.StepBuffers(ccfg, [cap], 1)              # ctx_off = [0, cap]: capacity
    L0 = len(prompt) - 1
    ws = DF.alloc_workspace(DF.dflash_workspace_size(ccfg, 1, 1, max(B, L0), cap))
    dev = dict(device="cuda")
    ctx_len = torch.tensor([L0], dtype=torch.int32, **dev)
    # first step: the prompt's context rows through the ordinary new-row path
    st0, _ = TT.forward(tw, np.asarray(prompt[:-1]))
    buf.block_tokens.zero_()
    buf.block_tokens[0, 0] = int(prompt[-1])
    DF.dflash_draft_step(ccfg, w, buf, torch.from_numpy(st0).cuda(), ws,
                         new_off=torch.tensor([0, L0], dtype=torch.int64, **dev),
                         ctx_cached=torch.zeros(1, dtype=torch.int32, **dev),
                         ctx_len=ctx_len, max_ctx_len=cap)
    DF.dflash_check(ws)
    # fixed-shape buffers of the device loop
    verify = torch.zeros(1, 1, B, T, H, dtype=torch.float32, **dev)
    target = torch.zeros(1, 1, B, dtype=torch.int32, **dev)
    new_states = torch.zeros(1, B, T, H, dtype=torch.float32, **dev)
    new_count = torch.zeros(1, dtype=torch.int32, **dev)
    n_acc = torch.zeros(1, dtype=torch.int32, **dev)
    best_k = torch.zeros(1, dtype=torch.int32, **dev)
    out_tok = torch.zeros(1, B, dtype=torch.int32, **dev)

    def device_step():
        DF.dflash_accept(buf.draft_tokens.view(1, 1, B), target, n_acc, best_k, out_tok)
        DF.dflash_advance(ccfg, n_acc, best_k, out_tok, verify, ctx_len, buf.ctx_off,
                          new_states, new_count, buf.block_tokens, buf.known_len, ws)
        DF.dflash_draft_step(ccfg, w, buf, new_states.view(B, T, H), ws, ctx_len=ctx_len,
                             new_count=new_count, max_ctx_len=cap)

    rng = np.random.default_rng(5)
    seq = [int(t) for t in prompt]
    graph = None
    steps = 0
    while len(seq) - len(prompt) < n_new:
        # --- the target model's part (host stand-in)
        d = buf.draft_tokens[0].cpu().numpy().copy()
        assert d[0] == seq[-1]
        m = min(int(rng.geometric(0.3)) - 1, B - 1)        # exercise multi-token acceptance
        if m:
            d[1:m + 1] = TT.greedy(tw, np.asarray(seq), m)
            buf.draft_tokens[0].copy_(torch.from_numpy(d))
        st, nxt = TT.forward(tw, np.asarray(seq + [int(v) for v in d[1:]]))
        L = len(seq) - 1
        verify[0, 0].copy_(torch.from_numpy(np.ascontiguousarray(st[L:L + B])))
        target[0, 0].copy_(torch.from_numpy(nxt[L:L + B].astype(np.int32)))
        # --- one decode step on the device: one graph replay
        if graph is None:
            device_step()                                   # first call outside capture
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                device_step()
        else:
            graph.replay()
        torch.cuda.synchronize()
        DF.dflash_check(ws)
        k = int(n_acc.item())
        seq += [int(v) for v in out_tok[0, :k + 1].cpu().numpy()]
        assert int(ctx_len.item()) == len(seq) - 1          # the device kept count
        assert int(buf.block_tokens[0, 0].item()) == seq[-1]
        steps += 1
    got = np.asarray(seq[len(prompt):len(prompt) + n_new])
    np.testing.assert_array_equal(got, greedy)
    assert steps < n_new
