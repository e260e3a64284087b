"""Decode step on the GPU (hga_decode_select, hga_decode_attn) against the
fp64 oracle's decode functions, through the C ABI.

Cases cover one and several new tokens, new tokens that straddle a block
boundary, a whole aligned block (which must also equal the prefill kernels'
rows of that query block), no history, K above the history length, the fp32
CUDA-core path with d = 64 and 64-token blocks, and the full 131K-context
decode (992 history blocks, K = 32, a 4,096-token segment buffer).  Segment
positions after the new tokens are filled with NaN on the device: the kernels
must never read them.  Tolerances as the other parity tests: selection
bit-exact except at oracle near-ties; fp32 max abs 1e-4; bf16 max abs 2e-2 and
relative L2 1e-2.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from hga_testutil import BF16_ABS, BF16_REL, F32_ABS, assert_close, dims_of, to_dev, to_host
from segmented_fine_tuning_b200 import (HgaError, hga_attn_fwd, hga_block_summaries, hga_decode_attn,
                                        hga_decode_select, hga_decode_workspace_size, hga_device_status,
                                        hga_select_topk)

pytestmark = pytest.mark.gpu

W_SMALL = synth.Workload("dec-small: Hq8/Hkv2 d128 S512 hist20 K4", 1, 8, 2, 128, 128, 512, 20, 4, "bf16", 91,
                         structured_keys=True)
CASES = [
    (W_SMALL, 1, 300),
    (W_SMALL, 5, 125),       # straddles the block boundary at 128
    (W_SMALL, 1, 0),         # the first segment token: one segment key
    (W_SMALL, 16, 496),      # the buffer's last 16 positions
    (synth.Workload("dec-B2-G4: B2 Hq16/Hkv4 S256 hist9 K3", 2, 16, 4, 128, 128, 256, 9, 3, "bf16", 92), 3, 77),
    (synth.Workload("dec-no-history", 1, 8, 2, 128, 128, 256, 0, 4, "bf16", 93), 2, 40),
    (synth.Workload("dec-K>hist: hist2 K5", 1, 8, 2, 128, 128, 256, 2, 5, "bf16", 94), 1, 200),
    (synth.Workload("dec-f32-d64-blk64: Hq2/Hkv1 S256 hist16 K4", 1, 2, 1, 64, 64, 256, 16, 4, "f32", 95), 3, 100),
    (synth.Workload("dec-bf16-d64-blk32-G3", 1, 6, 2, 64, 32, 128, 7, 2, "bf16", 96), 4, 60),
    # up to 8 rows per KV head (G x n_q) in bf16 take the streaming chunk kernel
    (synth.Workload("dec-stream-d64-blk32: B2 Hq4/Hkv2 d64 S128 hist7 K3", 2, 4, 2, 64, 32, 128, 7, 3, "bf16", 97),
     2, 60),
    (synth.Workload("dec-stream-G8: Hq16/Hkv2 S256 hist6 K3", 1, 16, 2, 128, 128, 256, 6, 3, "bf16", 98), 1, 130),
    (W_SMALL, 2, 126),       # 8 rows, the two tokens straddle the block boundary at 128
    (synth.Workload("dec-stream-blk16: Hq8/Hkv2 S128 hist20 K6", 1, 8, 2, 128, 16, 128, 20, 6, "bf16", 99), 1, 90),
]


def _decode(w, nq, t0, x):
    D = dims_of(w)
    dev = {n: to_dev(getattr(x, n)) for n in ("k_seg", "v_seg", "k_hist", "v_hist")}
    qn = to_dev(x.extra["q_new"])
    # positions after the new tokens hold NaN: they must not be read
    dev["k_seg"][:, t0 + nq:] = float("nan")
    dev["v_seg"][:, t0 + nq:] = float("nan")
    summ = torch.zeros((w.B, max(w.nblk, 1), w.Hkv, w.d), dtype=torch.float32, device="cuda")
    if w.nblk:
        hga_block_summaries(D, dev["k_hist"], 0, w.nblk, summ)
    idx = torch.empty((w.B, w.Hkv, w.topk), dtype=torch.int32, device="cuda")
    scores = torch.empty(idx.shape, dtype=torch.float32, device="cuda")
    ws = torch.empty((hga_decode_workspace_size(D, nq),), dtype=torch.uint8, device="cuda")
    hga_decode_select(D, qn, summ, idx, scores, ws)
    o = torch.empty_like(qn)
    lse = torch.empty((w.B, w.Hq, nq), dtype=torch.float32, device="cuda")
    hga_decode_attn(D, t0, qn, dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], w.nblk, idx, o, lse, ws)
    torch.cuda.synchronize()
    hga_device_status()
    return D, idx.cpu().numpy(), scores.cpu().numpy(), o, lse


def _check_against_oracle(w, nq, t0, x, idx, scores, o, lse):
    od = oracle.Dims(w.B, w.Hq, w.Hkv, w.d, w.blk, w.S, w.nblk, w.topk)
    summ_ref = oracle.block_summaries(od, x.k_hist.f64)
    qn = x.extra["q_new"].f64
    idx_ref, score_ref = oracle.decode_select(od, qn, summ_ref)
    keff = min(w.topk, w.nblk)
    # selection: bit-exact except at near-ties of the oracle's K-th and (K+1)-th scores
    near = oracle.near_tie_positions(od, score_ref[:, :, None, :])[:, :, 0] if keff < w.nblk else \
        np.zeros(idx.shape[:2], dtype=bool)
    diff = np.any(idx != idx_ref, axis=-1)
    assert not (diff & ~near).any(), f"decode selection differs at {np.argwhere(diff & ~near)[:4].tolist()}"
    for b, h in np.argwhere(diff):
        v = idx[b, h][idx[b, h] >= 0]
        kth = np.sort(score_ref[b, h])[::-1][keff - 1]
        assert len(set(v.tolist())) == keff and np.all(score_ref[b, h][v] >= kth - 1e-3 * max(abs(kth), 1e-6))
    ok = idx >= 0
    if ok.any():
        ref_sel = np.take_along_axis(score_ref, np.maximum(idx, 0), axis=-1)
        assert np.abs(scores[ok] - ref_sel[ok]).max() <= 1e-4 * max(1.0, np.abs(score_ref).max())
    assert np.all(idx[~ok] == -1) and np.all(np.isneginf(scores[~ok]))
    o_ref, lse_ref = oracle.decode_attn(od, t0, qn, x.k_seg.f64, x.v_seg.f64, x.k_hist.f64, x.v_hist.f64, idx)
    tol = (F32_ABS, None) if w.dtype == "f32" else (BF16_ABS, BF16_REL)
    assert_close("decode O", to_host(o), o_ref, *tol)
    assert_close("decode LSE", to_host(lse), lse_ref, *tol)


@pytest.mark.parametrize("w,nq,t0", CASES, ids=lambda c: c.name.split(":")[0] if hasattr(c, "name") else str(c))
def test_decode_step_matches_oracle(w, nq, t0):
    x = synth.draw_decode(w, nq, t0)
    D, idx, scores, o, lse = _decode(w, nq, t0, x)
    _check_against_oracle(w, nq, t0, x, idx, scores, o, lse)


def test_decode_whole_block_equals_prefill_kernels():
    """n_q = block new queries at a block boundary: the decode kernels give the
    prefill kernels' selection and (up to summation order) their rows."""
    w, i = W_SMALL, 2
    nq, t0 = w.blk, i * w.blk
    x = synth.draw_decode(w, nq, t0)
    D, idx, scores, o, lse = _decode(w, nq, t0, x)
    _check_against_oracle(w, nq, t0, x, idx, scores, o, lse)
    dev = {n: to_dev(getattr(x, n)) for n in ("q", "k_seg", "v_seg", "k_hist", "v_hist")}
    summ = torch.empty((1, w.nblk, w.Hkv, w.d), device="cuda")
    idx_p = torch.empty((1, w.Hkv, w.nqb, w.topk), dtype=torch.int32, device="cuda")
    hga_block_summaries(D, dev["k_hist"], 0, w.nblk, summ)
    hga_select_topk(D, dev["q"], summ, idx_p)
    o_p = torch.empty_like(dev["q"])
    lse_p = torch.empty((1, w.Hq, w.S), device="cuda")
    hga_attn_fwd(D, dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], w.nblk, idx_p, o_p, lse_p)
    torch.cuda.synchronize()
    # the two kernels sum the query mean in different fp32 orders: equal
    # selections wherever the oracle's K-th and (K+1)-th scores are not a near-tie
    od = oracle.Dims(w.B, w.Hq, w.Hkv, w.d, w.blk, w.S, w.nblk, w.topk)
    _, score_ref = oracle.select(od, x.q.f64, x.k_hist.f64)
    near = oracle.near_tie_positions(od, score_ref)[:, :, i]
    same = np.all(idx == idx_p.cpu().numpy()[:, :, i], axis=-1)
    assert np.all(same | near)
    rows = slice(t0, t0 + nq)
    assert (o.float() - o_p[:, rows].float()).abs().max().item() <= 2e-2
    assert (lse - lse_p[:, :, rows]).abs().max().item() <= 1e-4


def test_decode_131k_context():
    """Full-size decode: 992 history blocks, K = 32, 4,096-token segment buffer,
    one new token at its last position; every head against the oracle."""
    w = synth.DECODE_131K
    nq, t0 = 1, w.S - 1
    x = synth.draw_decode(w, nq, t0)
    D, idx, scores, o, lse = _decode(w, nq, t0, x)
    _check_against_oracle(w, nq, t0, x, idx, scores, o, lse)


def test_decode_rejects_bad_arguments_and_flags_bad_index():
    w = W_SMALL
    x = synth.draw_decode(w, 1, 10)
    D = dims_of(w)
    dev = {n: to_dev(getattr(x, n)) for n in ("k_seg", "v_seg", "k_hist", "v_hist")}
    qn = to_dev(x.extra["q_new"])
    o = torch.empty_like(qn)
    lse = torch.empty((1, w.Hq, 1), device="cuda")
    ws = torch.empty((hga_decode_workspace_size(D, 1),), dtype=torch.uint8, device="cuda")
    idx = torch.tensor([0, 3, 25, -1], dtype=torch.int32, device="cuda").repeat(1, 2, 1)
    with pytest.raises(HgaError) as e:  # new token beyond the buffer
        hga_decode_attn(D, w.S, qn, dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], w.nblk, idx, o, lse,
                        ws)
    assert e.value.status == 2
    with pytest.raises(HgaError) as e:  # short workspace
        hga_decode_attn(D, 10, qn, dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], w.nblk, idx, o, lse,
                        ws[:64])
    assert e.value.status == 1
    # block 25 is outside the 20-block history: skipped and flagged, never read
    hga_decode_attn(D, 10, qn, dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], w.nblk, idx, o, lse, ws)
    with pytest.raises(HgaError) as e:
        hga_device_status()
    assert e.value.status == 4
    idx_ok = torch.tensor([0, 3, -1, -1], dtype=torch.int32, device="cuda").repeat(1, 2, 1)
    o2, lse2 = torch.empty_like(o), torch.empty_like(lse)
    hga_decode_attn(D, 10, qn, dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], w.nblk, idx_ok, o2, lse2,
                    ws)
    torch.cuda.synchronize()
    hga_device_status()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
