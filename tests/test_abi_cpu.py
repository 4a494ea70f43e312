"""The C ABI without a GPU: libdflash.so loads, exports every function that
include/dflash.h declares, and rejects bad arguments on the host before any
CUDA call (these tests run on machines with no CUDA driver)."""
import ctypes as C
import os
import re

import pytest

from block_diffusion_speculative_softmax_b200 import build as B
from block_diffusion_speculative_softmax_b200 import dflash as DF
from block_diffusion_speculative_softmax_b200 import synth

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "dflash.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return DF.load()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dflash_\w+)\s*\(", text)))


def test_header_functions_are_exported(lib):
    names = header_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), f"{n} declared in dflash.h but not exported"


def test_binding_covers_exactly_the_header(lib):
    assert sorted(DF.SIGNATURES) == header_functions()


def test_version_and_counter(lib):
    assert "sm_100a" in DF.dflash_version()
    assert DF.dflash_launch_count() == 0


def _cfg(**over):
    c = DF.config_from(synth.get_config("qwen3_4b"))
    for k, v in over.items():
        setattr(c, k, v)
    return c


def test_workspace_size_valid_and_invalid(lib):
    n = DF.dflash_workspace_size(_cfg(), 1, 1, 2048, 2048)
    assert n > 0
    assert n % 256 == 0
    # more rows need more workspace
    assert DF.dflash_workspace_size(_cfg(), 1, 1, 4096, 4096) > n
    assert lib.dflash_workspace_size(C.byref(_cfg(head_dim=96)), 1, 1, 16, 16) == 0
    assert lib.dflash_workspace_size(None, 1, 1, 16, 16) == 0


@pytest.mark.parametrize("field,value,status", [
    ("dtype", 7, DF.EINVAL), ("head_dim", 96, DF.EUNSUPPORTED), ("block", 33, DF.EINVAL),
    ("block", 0, DF.EINVAL), ("n_q_heads", 12, DF.EINVAL), ("hidden", 2561, DF.EINVAL),
    ("mask_token_id", 151936, DF.EINVAL), ("n_draft_layers", 17, DF.EINVAL),
    ("rope_theta", 0.0, DF.EINVAL), ("hidden", 16384, DF.EUNSUPPORTED)])
def test_bad_config_rejected_before_any_launch(lib, field, value, status):
    cfg = _cfg(**{field: value})
    g = (C.c_void_p * 16)(*([16] * 16))
    st = lib.dflash_fuse_ctx(C.byref(cfg), C.c_void_p(16), 4, C.c_void_p(16), g,
                             C.c_void_p(16), None)
    assert st == status
    assert lib.dflash_last_error()
    assert DF.dflash_launch_count() == 0


def test_bad_pointers_and_sizes_rejected(lib):
    cfg = _cfg()
    # null / misaligned pointers
    st = lib.dflash_lmhead_argmax(C.byref(cfg), 4, None, C.c_void_p(16), C.c_void_p(16), None,
                                  None, C.c_void_p(256), 1 << 20, None)
    assert st == DF.EINVAL and b"x is NULL" in lib.dflash_last_error()
    st = lib.dflash_lmhead_argmax(C.byref(cfg), 4, C.c_void_p(24), C.c_void_p(16),
                                  C.c_void_p(16), None, None, C.c_void_p(256), 1 << 20, None)
    assert st == DF.EINVAL and b"aligned" in lib.dflash_last_error()
    # workspace too small
    st = lib.dflash_lmhead_argmax(C.byref(cfg), 4, C.c_void_p(16), C.c_void_p(16),
                                  C.c_void_p(16), None, None, C.c_void_p(256), 64, None)
    assert st == DF.EINVAL and b"workspace too small" in lib.dflash_last_error()
    # accept: K and B out of range
    assert lib.dflash_accept(1, 0, 8, *([C.c_void_p(16)] * 5), None) == DF.EINVAL
    assert lib.dflash_accept(1, 1, 33, *([C.c_void_p(16)] * 5), None) == DF.EINVAL
    assert lib.dflash_accept(1, 1, 8, None, *([C.c_void_p(16)] * 4), None) == DF.EINVAL
    # D2SD: K must be in [1, B-1]
    assert lib.dflash_d2sd_candidates(1, 16, 16, 5, *([C.c_void_p(16)] * 5), None) == DF.EINVAL
    assert lib.dflash_d2sd_candidates(1, 1, 1, 5, *([C.c_void_p(16)] * 5), None) == DF.EINVAL
    # self test: limit must be bounded
    assert lib.dflash_selftest_wait_timeout(C.c_void_p(256), 4096, 10 ** 10, None) == DF.EINVAL
    # empty work is a no-op, not an error
    assert lib.dflash_accept(0, 1, 8, None, None, None, None, None, None) == DF.OK
    assert DF.dflash_launch_count() == 0


def test_draft_step_argument_checks(lib):
    cfg = _cfg()
    w = DF.Weights()
    a = DF.StepArgs()
    st = lib.dflash_draft_step(C.byref(cfg), C.byref(w), C.byref(a), C.c_void_p(256), 1 << 30,
                               None)
    assert st == DF.EINVAL and b"n_req" in lib.dflash_last_error()
    a.n_req, a.n_blocks = 2, 3
    a.target_tokens = 16
    a.n_cand = 1
    st = lib.dflash_draft_step(C.byref(cfg), C.byref(w), C.byref(a), C.c_void_p(256), 1 << 30,
                               None)
    assert st == DF.EINVAL
    assert DF.dflash_launch_count() == 0


def test_misaligned_index_and_output_pointers_rejected(lib):
    """int32 / fp32 / int64 arrays must be naturally aligned; a misaligned
    one is refused on the host (it would fault a kernel)."""
    cfg = _cfg()
    odd = C.c_void_p(258)     # 2 mod 4
    ok = C.c_void_p(256)
    st = lib.dflash_lmhead_argmax(C.byref(cfg), 4, ok, ok, odd, None, None, ok, 1 << 30, None)
    assert st == DF.EINVAL and b"tok is not 4-byte aligned" in lib.dflash_last_error()
    st = lib.dflash_lmhead_argmax(C.byref(cfg), 4, ok, ok, ok, None, odd, ok, 1 << 30, None)
    assert st == DF.EINVAL and b"conf is not 4-byte aligned" in lib.dflash_last_error()
    assert lib.dflash_accept(1, 1, 8, ok, ok, ok, ok, odd, None) == DF.EINVAL
    assert b"out_tok" in lib.dflash_last_error()
    assert lib.dflash_d2sd_candidates(1, 16, 4, 5, ok, odd, ok, ok, None, None) == DF.EINVAL
    st = lib.dflash_kv_project(C.byref(cfg), ok, 4, ok, C.c_void_p(260), ok, ok, ok, ok, ok,
                               1 << 30, None)
    assert st == DF.EINVAL and b"dst_row is not 8-byte aligned" in lib.dflash_last_error()
    w = DF.Weights()
    a = DF.StepArgs()
    a.n_req, a.n_blocks = 1, 1
    a.block_req, a.block_tokens, a.ctx_off, a.draft_tokens = 256, 256, 260, 256
    kc = (C.c_void_p * 16)(*([256] * 16))
    a.k_cache = kc
    a.v_cache = kc
    st = lib.dflash_draft_step(C.byref(cfg), C.byref(w), C.byref(a), ok, 1 << 30, None)
    assert st == DF.EINVAL and b"ctx_off is not 8-byte aligned" in lib.dflash_last_error()
    assert DF.dflash_launch_count() == 0


def test_workspace_size_is_monotone_in_blocks_and_rows():
    """A workspace sized for (n_blocks, n_ctx_new) must serve every call with
    fewer blocks or rows (a D2SD first pass drafts fewer blocks than its
    second pass; a steady step fuses fewer rows than a full one)."""
    from block_diffusion_speculative_softmax_b200 import dflash as DF
    DF.load()
    for kw in (dict(hidden=640, n_q_heads=16, n_kv_heads=2, head_dim=64, ffn=704,
                    n_draft_layers=2, n_target_layers=5, block=16, vocab=3001),
               dict(hidden=2560, n_q_heads=32, n_kv_heads=8, head_dim=128, ffn=9728,
                    n_draft_layers=5, n_target_layers=5, block=16, vocab=151936)):
        cc = DF.make_config(**kw)
        sizes = {}
        for nb in (1, 2, 3, 4, 5, 8, 12, 32):
            for n_new in (0, 7, 100, 2048):
                sizes[nb, n_new] = DF.dflash_workspace_size(cc, nb, nb, n_new, 4096)
        for (nb, n_new), v in sizes.items():
            for (nb2, n2), v2 in sizes.items():
                if nb2 <= nb and n2 <= n_new:
                    assert v2 <= v, ((nb, n_new, v), (nb2, n2, v2))


def test_fuse_rss_parts_is_one_per_warp_of_columns(lib):
    # one partial sum of squares per 32 threads x 8 bf16 columns
    for H, parts in [(4096, 16), (2880, 12), (2560, 10), (576, 3), (64, 1)]:
        assert DF.dflash_fuse_rss_parts(H) == parts
    assert DF.dflash_fuse_rss_parts(0) == 0


def test_split_fusion_rejects_fp32_and_bad_arguments(lib):
    cfg = DF.config_from(synth.get_config("tiny"))          # fp32 model
    assert lib.dflash_fuse_ctx_rss(C.byref(cfg), None, 0, None, None, None, None, None, 0,
                                   None) == DF.EUNSUPPORTED
    cfg = DF.config_from(synth.small_config("qwen3_4b", hidden=576, n_q_heads=8, n_kv_heads=2,
                                            head_dim=128, ffn=1000, n_draft_layers=2,
                                            n_target_layers=3, ctx_len=64, block=16,
                                            vocab=1000, dtype="bf16"))
    # no workspace for the status word
    assert lib.dflash_fuse_ctx_rss(C.byref(cfg), None, 0, None, None, None, None, None, 0,
                                   None) == DF.EINVAL


def test_split_fusion_pointer_checks_before_any_launch(lib):
    # fake device addresses: every check here runs on the host and fails
    # before the library touches CUDA
    cfg = DF.config_from(synth.small_config("qwen3_4b", hidden=576, n_q_heads=8, n_kv_heads=2,
                                            head_dim=128, ffn=1000, n_draft_layers=2,
                                            n_target_layers=3, ctx_len=64, block=16,
                                            vocab=1000, dtype="bf16"))
    ws, big = C.c_void_p(1 << 20), 1 << 20
    g = (C.c_void_p * 2)(1 << 21, 1 << 22)
    good = dict(states=C.c_void_p(1 << 23), w=C.c_void_p(1 << 24), fused=C.c_void_p(1 << 25),
                rss=C.c_void_p(1 << 26))

    def call(**over):
        a = dict(good, **over)
        return lib.dflash_fuse_ctx_rss(C.byref(cfg), a["states"], 10, a["w"], g, a["fused"],
                                       a["rss"], ws, big, None)

    assert call(rss=C.c_void_p((1 << 26) + 2)) == DF.EINVAL      # rss not 4-byte aligned
    assert call(rss=None) == DF.EINVAL
    assert call(fused=C.c_void_p((1 << 25) + 8)) == DF.EINVAL   # bulk tensor not 16-byte aligned
    assert call(states=None) == DF.EINVAL
    assert lib.dflash_fuse_ctx_rss(C.byref(cfg), good["states"], 10, good["w"], g, good["fused"],
                                   good["rss"], C.c_void_p((1 << 20) + 64), big,
                                   None) == DF.EINVAL                # workspace not 256-aligned
