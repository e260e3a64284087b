"""Shared helpers of the GPU parity tests (marshalling and error metrics only)."""
from __future__ import annotations

import numpy as np
import torch

import synth
from segmented_fine_tuning_b200 import Dims


def dims_of(w: synth.Workload, nblk: int | None = None) -> Dims:
    return Dims(w.B, w.Hq, w.Hkv, w.d, w.blk, w.S, w.nblk if nblk is None else nblk, w.topk, w.dtype, w.qblk)


def to_dev(t: synth.Tensor, device="cuda") -> torch.Tensor:
    if t.dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(t.store).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(t.store)).to(device)


def to_host(x: torch.Tensor) -> np.ndarray:
    return x.detach().float().cpu().numpy().astype(np.float64)


def errors(got: np.ndarray, want: np.ndarray):
    """(max abs error, relative L2 error) over entries where want is finite."""
    m = np.isfinite(want)
    g, w = got[m], want[m]
    diff = g - w
    return float(np.abs(diff).max()), float(np.linalg.norm(diff) / max(np.linalg.norm(w), 1e-30))


def assert_close(name, got, want, max_abs, rel_l2=None):
    ma, rl = errors(got, want)
    assert np.all(np.isfinite(got[np.isfinite(want)])), f"{name}: non-finite values"
    assert ma <= max_abs, f"{name}: max abs err {ma:.3e} > {max_abs:.1e} (rel L2 {rl:.3e})"
    if rel_l2 is not None:
        assert rl <= rel_l2, f"{name}: rel L2 err {rl:.3e} > {rel_l2:.1e} (max abs {ma:.3e})"
    return ma, rl


# Tolerances: fp32 workloads max abs 1e-4 on O, LSE, dQ, dK, dV; bf16
# workloads max abs 2e-2 and relative L2 1e-2 against the fp64 oracle.
F32_ABS = 1e-4
BF16_ABS = 2e-2
BF16_REL = 1e-2


def check_selection(D, idx_gpu: np.ndarray, idx_ref: np.ndarray, score_ref: np.ndarray, near_tie) -> int:
    """Bit-exact selection except at oracle near-ties, where the GPU's set
    must still be a valid choice: same size, distinct, ascending, and every
    block it picks scores at least the oracle's K-th best minus the tie
    margin.  Returns the number of accepted near-tie differences."""
    diff = np.any(idx_gpu != idx_ref, axis=-1)
    bad = diff & ~near_tie
    assert not bad.any(), f"selection differs at {np.argwhere(bad)[:5].tolist()}"
    n_acc = 0
    keff = min(D.topk, D.n_hist_blocks)
    for pos in np.argwhere(diff):
        b, h, i = pos
        sel = idx_gpu[b, h, i]
        v = sel[sel >= 0]
        assert len(v) == keff and len(set(v.tolist())) == keff and np.all(np.diff(v) > 0)
        s = score_ref[b, h, i]
        kth = np.sort(s)[::-1][keff - 1]
        assert np.all(s[v] >= kth - 1e-3 * max(abs(kth), 1e-6)), "near-tie alternative is not a valid top-K"
        n_acc += 1
    return n_acc
