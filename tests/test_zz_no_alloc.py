"""The allocation-free LM-head argmax entry point.

Some callers cannot allocate device memory or hand the library a workspace
(for example a plugin inside a serving process whose GPU memory belongs to
that process's caching allocator).  dflash_lmhead_argmax_noalloc keeps its
scratch in a fixed device array inside the library instead.  This test calls
it through the C ABI and checks it against dflash_lmhead_argmax (which uses a
caller workspace) on calls in a row with different inputs, so leftovers of
one call in the shared array would show up in the next: the small-batch
weight-streaming path (16 and 48 tokens), the token-major path (80 tokens),
the 4096-token limit and the fp32 path.  Where the CPU oracle finishes in
seconds, its argmax is checked as well.

This file sorts last so that a run stopping at the first failure has run
every other test already; it also passes when run alone in a fresh process.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from block_diffusion_speculative_softmax_b200 import synth

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "fp32": 1e-4}   # the tolerances of the other parity tests


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
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn(M, cfg.hidden, device="cuda", generator=g).to(dt)
    w = (0.02 * torch.randn(cfg.vocab, cfg.hidden, device="cuda", generator=g)).to(dt)
    return x, w


def _noalloc(DF, cc, x, w, M):
    lib = DF.load()
    tok = torch.full((M,), -1, dtype=torch.int32, device="cuda")
    mx = torch.zeros(M, dtype=torch.float32, device="cuda")
    st = lib.dflash_lmhead_argmax_noalloc(
        C.byref(cc), M, C.c_void_p(x.data_ptr()), C.c_void_p(w.data_ptr()),
        C.c_void_p(tok.data_ptr()), C.c_void_p(mx.data_ptr()),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == DF.OK, lib.dflash_last_error()
    torch.cuda.synchronize()
    return tok, mx


def _check_oracle(cfg, x, w, tok, mx):
    from oracle import dflash_oracle as O
    from tests.gpu_common import token_report
    xo = x.float().cpu().numpy().astype(np.float64)
    wo = w.float().cpu().numpy().astype(np.float64)
    otok, omax, z = O.lmhead_argmax(xo, wo)
    # same inputs on both sides: only the fp32 summation order differs
    _, _, bad = token_report(tok.cpu().numpy(), z, cfg.dtype,
                             tol=1e-3 if cfg.dtype == "bf16" else None)
    assert not bad, bad[:3]
    err = np.max(np.abs(mx.cpu().numpy() - omax)) / max(1.0, np.max(np.abs(omax)))
    assert err <= TOL[cfg.dtype], err


# (tokens, seed, hidden, vocab, dtype, also against the oracle)
CALLS = [(48, 1, 2560, 151936, "bf16", False), (16, 2, 2560, 151936, "bf16", True),
         (80, 3, 2560, 151936, "bf16", False), (4096, 4, 1024, 32000, "bf16", False),
         (80, 5, 576, 5000, "bf16", True), (24, 6, 256, 1000, "fp32", True),
         (16, 7, 2560, 151936, "bf16", False)]


def test_noalloc_lmhead_matches_workspace_variant_calls_in_a_row(DF):
    for call, (M, seed, H, V, dtype, with_oracle) in enumerate(CALLS):
        cfg = synth.small_config("qwen3_4b", hidden=H, vocab=V, dtype=dtype)
        cc = DF.config_from(cfg)
        x, w = _case(cfg, M, seed)
        # reference: the workspace entry point
        tok_ref = torch.empty(M, dtype=torch.int32, device="cuda")
        max_ref = torch.empty(M, dtype=torch.float32, device="cuda")
        ws = DF.alloc_workspace(DF.dflash_workspace_size(cc, 1, (M + 15) // 16, 0, 0))
        DF.dflash_lmhead_argmax(cc, x, w, tok_ref, max_ref, ws)
        DF.dflash_check(ws)
        # the allocation-free entry point, called through the C ABI
        tok, mx = _noalloc(DF, cc, x, w, M)
        assert torch.equal(tok, tok_ref), f"call {call} (M={M}): tokens differ"
        ref = max_ref.cpu().numpy().astype(np.float64)
        err = np.max(np.abs(mx.cpu().numpy() - ref)) / max(1.0, np.max(np.abs(ref)))
        assert err <= TOL[dtype], f"call {call}: max-logit error {err}"
        if with_oracle:
            _check_oracle(cfg, x, w, tok, mx)


def test_noalloc_rejects_more_tokens_than_its_scratch(DF):
    cfg = synth.small_config("qwen3_4b", hidden=256, vocab=512)
    cc = DF.config_from(cfg)
    lib = DF.load()
    st = lib.dflash_lmhead_argmax_noalloc(C.byref(cc), 4097, C.c_void_p(256), C.c_void_p(256),
                                          C.c_void_p(256), None, None)
    assert st == DF.EINVAL
    assert b"4096" in lib.dflash_last_error()
