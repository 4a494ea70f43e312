"""Helpers shared by the GPU parity tests (CUDA path vs CPU oracle)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import dflash_oracle as O
from block_diffusion_speculative_softmax_b200 import synth

# Tolerances: max|gpu - oracle| / max(1, max|oracle|).
TOL = {"fp32": 1e-4, "bf16": 2e-2}


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from block_diffusion_speculative_softmax_b200 import build
    build.build()


def rel_err(gpu, ref) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(gpu - ref)) / max(1.0, float(np.max(np.abs(ref)))))


def to_dev(a, dtype, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dtype)


def token_report(gpu_tok, logits, dtype: str, tol: float = None):
    """Compare GPU argmax tokens with the oracle's logits row by row.

    A row is exact when the GPU token is the oracle's argmax.  When the
    oracle's top-2 gap is at most 2*tol*max(1, max|z|) (a near-tie at the
    stated fp tolerance) the GPU token may be any id whose oracle logit is
    within that margin of the maximum.  Returns (n_exact, n_near, bad_rows)."""
    tol = TOL[dtype] if tol is None else tol
    gpu_tok = np.asarray(gpu_tok).reshape(-1)
    if gpu_tok.shape[0] == 0:
        return 0, 0, []
    logits = np.asarray(logits, dtype=np.float64).reshape(gpu_tok.shape[0], -1)
    n_exact = n_near = 0
    bad = []
    for m in range(gpu_tok.shape[0]):
        z = logits[m]
        top = int(np.argmax(z))
        if int(gpu_tok[m]) == top:
            n_exact += 1
            continue
        thr = 2.0 * tol * max(1.0, float(np.max(np.abs(z))))
        srt = np.sort(z)
        gap = srt[-1] - srt[-2]
        g = int(gpu_tok[m])
        if dtype != "fp32" and gap <= thr and 0 <= g < z.shape[0] and z[g] >= z[top] - thr:
            n_near += 1
        else:
            bad.append((m, g, top, float(gap)))
    return n_exact, n_near, bad


def oracle_for_workload(wl, reqs, blocks):
    """Run the oracle draft step for the listed requests.  ``blocks``: list of
    O.Block (their ``req`` must be in ``reqs``).  Returns (tokens, maxz, keep)."""
    cfg = wl.cfg
    states = {}
    for r in reqs:
        states[r] = synth.make_states(cfg, wl.seed, r, wl.ctx_lens[r])
    keep = {}
    toks, maxz = O.draft_step(cfg, wl.host_weights, states, blocks,
                              bf16_storage=(cfg.dtype == "bf16"), keep=keep)
    return toks, maxz, keep


def check_draft(wl, gpu_tok, gpu_max, orc_tok, orc_max, keep, blocks, label=""):
    """Tokens bit-exact outside near-ties (none allowed for fp32); max logit
    within the fp tolerance; known-prefix slots copy their input."""
    cfg = wl.cfg
    tol = TOL[cfg.dtype]
    B = cfg.block
    n_exact = n_near = 0
    bad = []
    for i, blk in enumerate(blocks):
        kl = blk.known_len
        assert gpu_tok[i][:kl].tolist() == [int(t) for t in blk.tokens[:kl]], label
        e, n, b = token_report(gpu_tok[i][kl:], keep["logits"][i][kl:], cfg.dtype)
        n_exact += e
        n_near += n
        bad += [(i, kl + m, g, t, gap) for (m, g, t, gap) in b]
    assert not bad, f"{label}: token mismatches outside near-ties: {bad[:5]}"
    err = rel_err(gpu_max, orc_max)
    assert err <= tol, f"{label}: max-logit error {err:.3e} > {tol}"
    return {"exact": n_exact, "near_tie": n_near, "rows": len(blocks) * B, "max_logit_err": err}
