"""The hot path at its documented maximum sizes, against the fp64 oracle.

- Selection over 4,096 history blocks (the largest the selection kernels
  take) with K = 64 (the largest K), then attention through the CUDA-core
  path (32-token blocks) over those 64 selected blocks.
- The tensor-core path with K = 64: forward and backward, every output.
- The tensor-core path with a 128-block segment (16,384 tokens, the longest
  its tile lists hold: 2 history tiles + 128 segment tiles for the last query
  block): forward on two rows of every query block, and the sparse backward
  with two chosen query blocks (the first and the last), so that the oracle's
  backward stays small while the dQ and dK/dV kernels run their longest lists.

Tolerances as the other parity tests: bf16 max abs 2e-2 and relative L2 1e-2.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from hga_testutil import BF16_ABS, BF16_REL, assert_close, check_selection, dims_of, to_dev, to_host
from segmented_fine_tuning_b200 import hga_attn_bwd_sparse, hga_attn_bwd_workspace_size, hga_device_status
from segmented_fine_tuning_b200.step import AttentionStep

pytestmark = pytest.mark.gpu


def _odims(w):
    return oracle.Dims(w.B, w.Hq, w.Hkv, w.d, w.blk, w.S, w.nblk, w.topk, w.qblk)


def _run(w, x, backward=True):
    D = dims_of(w)
    dev = {n: to_dev(getattr(x, n)) for n in ("q", "k_seg", "v_seg", "k_hist", "v_hist", "d_o")}
    st = AttentionStep(D)
    st.select(dev["q"], dev["k_hist"])
    st.forward(dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"])
    if backward:
        st.backward(dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], dev["d_o"])
    torch.cuda.synchronize()
    hga_device_status()
    return st, dev


def _check_full(w, x, st):
    od = _odims(w)
    idx_ref, score_ref = oracle.select(od, x.q.f64, x.k_hist.f64)
    idx = st.idx.cpu().numpy()
    check_selection(dims_of(w), idx, idx_ref, score_ref, oracle.near_tie_positions(od, score_ref))
    args = (x.q.f64, x.k_seg.f64, x.v_seg.f64, x.k_hist.f64, x.v_hist.f64, idx)
    o_ref, lse_ref = oracle.attn_fwd(od, *args)
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd(od, *args, x.d_o.f64)
    for name, got, want in (("O", st.o, o_ref), ("LSE", st.lse, lse_ref), ("dQ", st.dq, dq_ref),
                            ("dK", st.dk, dk_ref), ("dV", st.dv, dv_ref)):
        assert_close(f"{w.name} {name}", to_host(got), want, BF16_ABS, BF16_REL)


def test_max_history_and_k():
    """4,096 history blocks of 32 tokens, K = 64; the selection uses the radix
    path, the attention the CUDA-core kernels (32-token blocks)."""
    w = synth.Workload("max-hist4096-K64: Hq4/Hkv2 blk32 S128", 1, 4, 2, 128, 32, 128, 4096, 64, "bf16", 201)
    x = synth.draw(w)
    st, _ = _run(w, x)
    assert int((st.idx >= 0).sum().item()) == w.B * w.Hkv * w.nqb * 64
    _check_full(w, x, st)


def test_max_k_tensor_core_path():
    """K = 64 of 72 history blocks on the tensor-core kernels: every tile list
    holds 64 history tiles before the causal segment tiles."""
    w = synth.Workload("tc-K64: Hq4/Hkv2 S256 hist72 K64", 1, 4, 2, 128, 128, 256, 72, 64, "bf16", 202,
                       structured_keys=True)
    x = synth.draw(w)
    st, _ = _run(w, x)
    _check_full(w, x, st)


def test_max_segment_tensor_core_path():
    """A 16,384-token segment (128 query blocks): forward on two rows of every
    query block; sparse backward with query blocks 0 and 127 chosen."""
    w = synth.Workload("tc-S16384: Hq2/Hkv1 hist4 K2", 1, 2, 1, 128, 128, 16384, 4, 2, "bf16", 203)
    x = synth.draw(w)
    st, dev = _run(w, x, backward=False)
    od = _odims(w)
    idx_ref, score_ref = oracle.select(od, x.q.f64, x.k_hist.f64)
    idx = st.idx.cpu().numpy()
    check_selection(dims_of(w), idx, idx_ref, score_ref, oracle.near_tie_positions(od, score_ref))
    args = (x.q.f64, x.k_seg.f64, x.v_seg.f64, x.k_hist.f64, x.v_hist.f64, idx)
    rows = sorted({i * w.blk + r for i in range(w.nqb) for r in (0, 127 - (i % 5) * 11)})
    o_ref, lse_ref = oracle.attn_fwd(od, *args, rows=rows)
    assert_close("O rows", to_host(st.o)[:, rows], o_ref[:, rows], BF16_ABS, BF16_REL)
    assert_close("LSE rows", to_host(st.lse)[:, :, rows], lse_ref[:, :, rows], BF16_ABS, BF16_REL)

    mask = torch.zeros((w.B, w.nqb), dtype=torch.uint8)
    mask[:, 0] = 1
    mask[:, w.nqb - 1] = 1
    D = dims_of(w)
    dq = torch.empty((w.B, w.S, w.Hq, w.d), dtype=torch.float32, device="cuda")
    dk = torch.empty((w.B, w.S, w.Hkv, w.d), dtype=torch.float32, device="cuda")
    dv = torch.empty_like(dk)
    ws = torch.empty((hga_attn_bwd_workspace_size(D),), dtype=torch.uint8, device="cuda")
    hga_attn_bwd_sparse(D, dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], w.nblk, st.idx,
                        st.o, st.lse, dev["d_o"], mask.cuda(), 1.0, dq, dk, dv, ws)
    torch.cuda.synchronize()
    hga_device_status()
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd_sparse(od, *args, x.d_o.f64, mask.numpy().astype(np.int8), 1.0)
    assert_close("sparse dQ", to_host(dq), dq_ref, BF16_ABS, BF16_REL)
    assert_close("sparse dK", to_host(dk), dk_ref, BF16_ABS, BF16_REL)
    assert_close("sparse dV", to_host(dv), dv_ref, BF16_ABS, BF16_REL)
