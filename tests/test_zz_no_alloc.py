"""The allocation-free LM-head argmax entry point.

Some callers cannot allocate device memory or hand the library a workspace
(for example a plugin inside a serving process whose GPU memory belongs to
that process's caching allocator).  dflash_lmhead_argmax_noalloc keeps its
scratch in a fixed device array inside the library instead.  This test calls
it through the C ABI and checks it against dflash_lmhead_argmax (which uses a
caller workspace) on two calls in a row with different inputs, so leftovers
of the first call in the shared array would show up in the second.

This file sorts last so that a run stopping at the first failure has run
every other test already; it also passes when run alone in a fresh process.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from block_diffusion_speculative_softmax_b200 import synth

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2   # the bf16 tolerance of the other parity tests


@pytest.fixture(scope="module")
def DF():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from block_diffusion_speculative_softmax_b200 import build
    build.build()
    from block_diffusion_speculative_softmax_b200 import dflash
    dflash.load()
    return dflash


def _case(cfg, M, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn(M, cfg.hidden, device="cuda", generator=g).to(torch.bfloat16)
    w = (0.02 * torch.randn(cfg.vocab, cfg.hidden, device="cuda", generator=g)).to(torch.bfloat16)
    return x, w


def test_noalloc_lmhead_matches_workspace_variant_twice(DF):
    cfg = synth.small_config("qwen3_4b", hidden=2560, vocab=151936)
    cc = DF.config_from(cfg)
    lib = DF.load()
    for call, (M, seed) in enumerate([(48, 1), (16, 2)]):
        x, w = _case(cfg, M, seed)
        # reference: the workspace entry point
        tok_ref = torch.empty(M, dtype=torch.int32, device="cuda")
        max_ref = torch.empty(M, dtype=torch.float32, device="cuda")
        ws = DF.alloc_workspace(DF.dflash_workspace_size(cc, 1, (M + 15) // 16, 0, 0))
        DF.dflash_lmhead_argmax(cc, x, w, tok_ref, max_ref, ws)
        # the allocation-free entry point, called through the C ABI
        tok = torch.full((M,), -1, dtype=torch.int32, device="cuda")
        mx = torch.zeros(M, dtype=torch.float32, device="cuda")
        st = lib.dflash_lmhead_argmax_noalloc(
            C.byref(cc), M, C.c_void_p(x.data_ptr()), C.c_void_p(w.data_ptr()),
            C.c_void_p(tok.data_ptr()), C.c_void_p(mx.data_ptr()),
            C.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == DF.OK, lib.dflash_last_error()
        torch.cuda.synchronize()
        DF.dflash_check(ws)
        assert torch.equal(tok, tok_ref), f"call {call}: tokens differ"
        ref = max_ref.cpu().numpy().astype(np.float64)
        err = np.max(np.abs(mx.cpu().numpy() - ref)) / max(1.0, np.max(np.abs(ref)))
        assert err <= TOL_BF16, f"call {call}: max-logit error {err}"


def test_noalloc_rejects_more_tokens_than_its_scratch(DF):
    cfg = synth.small_config("qwen3_4b", hidden=256, vocab=512)
    cc = DF.config_from(cfg)
    lib = DF.load()
    st = lib.dflash_lmhead_argmax_noalloc(C.byref(cc), 4097, C.c_void_p(256), C.c_void_p(256),
                                          C.c_void_p(256), None, None)
    assert st == DF.EINVAL
    assert b"4096" in lib.dflash_last_error()
