"""The debug-bounds build (libdflash_debug.so, compiled with
-DDFLASH_DEBUG_BOUNDS).  Its device-side index checks turn an index read from
device memory that falls outside its buffer (a context length beyond the
request's cache capacity, a token id beyond the vocabulary) into
DFLASH_EBOUNDS in the workspace status word, and the access is skipped or
clamped instead of made.  On valid inputs it drafts exactly the tokens of the
release library.

Each case runs in a child process that loads one library through DFLASH_LIB.
The out-of-range inputs go to the debug library only: its checks guard every
access they would steer (the new-row bookkeeping, the attention's context
range, the slot embedding)."""
import json
import os
import subprocess
import sys

import pytest

from tests.gpu_common import need_gpu

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# One draft step of a tiny bf16 model in the device-loop form (capacity
# layout, context length and new-row count in device memory).  CASE selects
# the input: "ok", "ctx_len" (one past capacity + 4) or "token" (an anchor id
# beyond the vocabulary).  Prints {"status": ..., "tag": ..., "tokens": ...}.
CHILD = r"""
import json, os, sys
import numpy as np
import torch
sys.path.insert(0, os.environ["REPO_ROOT"])
from block_diffusion_speculative_softmax_b200 import dflash as DF, synth
case = os.environ["CASE"]
cfg = synth.small_config("qwen3_4b", hidden=576, n_q_heads=8, n_kv_heads=2, head_dim=128,
                         ffn=1000, n_draft_layers=2, n_target_layers=3, ctx_len=200,
                         block=16, vocab=4096, dtype="bf16")
cc = DF.config_from(cfg)
B, T, H = cfg.block, cfg.n_target_layers, cfg.hidden
cap = 256
w = DF.DeviceWeights(cc, synth.make_weights(cfg, seed=3))
buf = DF.StepBuffers(cc, [cap], 1)
ws = DF.alloc_workspace(DF.dflash_workspace_size(cc, 1, 1, max(B, 150), cap))
dev = dict(device="cuda")
L0 = 150
st0 = torch.from_numpy(synth.make_states(cfg, 3, 0, L0)).to(**dev, dtype=torch.bfloat16)
ctx_len = torch.tensor([L0], dtype=torch.int32, **dev)
buf.block_tokens.zero_()
buf.block_tokens[0, 0] = 17
DF.dflash_draft_step(cc, w, buf, st0, ws,
                     new_off=torch.tensor([0, L0], dtype=torch.int64, **dev),
                     ctx_cached=torch.zeros(1, dtype=torch.int32, **dev),
                     ctx_len=ctx_len, max_ctx_len=cap)
DF.dflash_check(ws)
if case == "ctx_len":
    ctx_len.fill_(cap + 4)
elif case == "token":
    buf.block_tokens[0, 0] = cfg.vocab + 3
new_states = torch.zeros(B, T, H, dtype=torch.bfloat16, **dev)
new_count = torch.zeros(1, dtype=torch.int32, **dev)
DF.dflash_draft_step(cc, w, buf, new_states, ws, ctx_len=ctx_len, new_count=new_count,
                     max_ctx_len=cap)
out = {"status": "OK", "tag": None}
try:
    DF.dflash_check(ws)
except DF.DFlashError as e:
    out["status"] = DF.STATUS_NAMES.get(e.status, str(e.status))
    out["tag"] = str(e)
out["tokens"] = buf.draft_tokens[0].cpu().tolist()
print("RESULT " + json.dumps(out))
"""


def _run(lib, case):
    env = dict(os.environ, DFLASH_LIB=lib, CASE=case, REPO_ROOT=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("RESULT ")][-1]
    return json.loads(line[len("RESULT "):])


@pytest.fixture(scope="module")
def libs():
    need_gpu()
    from block_diffusion_speculative_softmax_b200 import build
    return build.build(), build.build(debug_bounds=True)


def test_debug_build_matches_release_on_valid_input(libs):
    rel, dbg = libs
    a = _run(rel, "ok")
    b = _run(dbg, "ok")
    assert a["status"] == "OK" and b["status"] == "OK"
    assert a["tokens"] == b["tokens"]


def test_context_length_past_capacity_is_reported(libs):
    _, dbg = libs
    r = _run(dbg, "ctx_len")
    assert r["status"] == "EBOUNDS", r
    assert "tag 82" in r["tag"], r      # the new-row bookkeeping sees it first


def test_token_beyond_vocabulary_is_reported(libs):
    _, dbg = libs
    r = _run(dbg, "token")
    assert r["status"] == "EBOUNDS", r
    assert "tag 87" in r["tag"], r      # the slot embedding
