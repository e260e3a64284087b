"""GPU parity: every kernel of the HGA step through the C ABI against the fp64
oracle, on the seeded synthetic workloads and on edge cases.

Tolerances: selection bit-exact except at oracle near-ties (K-th vs (K+1)-th
score closer than 1e-3 relative; the alternative must still be a valid top-K);
fp32 workloads max abs 1e-4; bf16 workloads max abs 2e-2 and relative L2 1e-2.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from hga_testutil import (BF16_ABS, BF16_REL, F32_ABS, assert_close, check_selection, dims_of, to_dev, to_host)
from segmented_fine_tuning_b200 import (Dims, HgaError, hga_attn_fwd, hga_block_summaries, hga_device_status,
                                        hga_select_topk, hga_selftest_umma)
from segmented_fine_tuning_b200.step import AttentionStep

pytestmark = pytest.mark.gpu


def _odims(w: synth.Workload, nblk=None):
    return oracle.Dims(w.B, w.Hq, w.Hkv, w.d, w.blk, w.S, w.nblk if nblk is None else nblk, w.topk, w.qblk)


def _tols(w):
    return (F32_ABS, None) if w.dtype == "f32" else (BF16_ABS, BF16_REL)


def _gpu_step(w: synth.Workload, x: synth.Inputs, backward=True):
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


# ------------------------------------------------------------------ tensor-core operand layouts

@pytest.mark.parametrize("form", [0, 1, 2, 3])
def test_selftest_umma_forms(form):
    g = torch.Generator().manual_seed(form)
    a = torch.randn(128, 128, generator=g).to(torch.bfloat16)
    b = torch.randn(128, 128, generator=g).to(torch.bfloat16)
    d = torch.zeros(128, 128, dtype=torch.float32, device="cuda")
    hga_selftest_umma(form, a.cuda(), b.cuda(), d)
    torch.cuda.synchronize()
    hga_device_status()
    A, Bm = a.double(), b.double()
    want = A @ Bm.T if form in (0, 3) else A @ Bm
    err = (d.cpu().double() - want).abs().max().item()
    assert err < 1e-3, f"form {form}: max abs err {err}"


# ------------------------------------------------------------------ summaries and selection

SEL_CASES = [
    synth.TINY_F32,
    synth.Workload("small-bf16-G4", 1, 8, 2, 128, 128, 512, 9, 3, "bf16", 21, structured_keys=True),
    synth.Workload("d64-bf16-blk64-G1", 2, 3, 3, 64, 64, 256, 7, 5, "bf16", 22),
    synth.Workload("k-exceeds-history", 1, 4, 2, 128, 128, 256, 3, 8, "bf16", 23),
    synth.QWEN3_8B_LAYER,
    synth.PREFILL_131K,
    # histories above 256 blocks take the staged scoring path: G = 1, 2, 8, d = 64, fp32, B = 2, and
    # block counts that leave a partial last chunk of 64
    synth.Workload("long-hist-G1-d64: Hq2/Hkv2 d64 blk64 S256 hist300 K8", 1, 2, 2, 64, 64, 256, 300, 8, "bf16", 26),
    synth.Workload("long-hist-G2-f32-B2: B2 Hq4/Hkv2 blk32 S128 hist277 K5", 2, 4, 2, 128, 32, 128, 277, 5, "f32",
                   27),
    synth.Workload("long-hist-G8: Hq16/Hkv2 S256 hist400 K16", 1, 16, 2, 128, 128, 256, 400, 16, "bf16", 28,
                   structured_keys=True),
]


@pytest.mark.parametrize("w", SEL_CASES, ids=lambda w: w.name.split(":")[0])
def test_summaries_and_selection(w):
    x = synth.draw(w)
    D = dims_of(w)
    q, kh = to_dev(x.q), to_dev(x.k_hist)
    summ = torch.zeros((w.B, w.nblk, w.Hkv, w.d), dtype=torch.float32, device="cuda")
    idx = torch.empty((w.B, w.Hkv, w.nqb, w.topk), dtype=torch.int32, device="cuda")
    scores = torch.empty(idx.shape, dtype=torch.float32, device="cuda")
    hga_block_summaries(D, kh, 0, w.nblk, summ)
    hga_select_topk(D, q, summ, idx, scores)
    torch.cuda.synchronize()
    od = _odims(w)
    summ_ref = oracle.block_summaries(od, x.k_hist.f64)
    s = to_host(summ).transpose(0, 2, 1, 3)  # block-major -> oracle layout [B, Hkv, nblk, d]
    assert np.abs(s - summ_ref).max() <= 1e-6 * max(1.0, np.abs(summ_ref).max())
    idx_ref, score_ref = oracle.select(od, x.q.f64, x.k_hist.f64)
    near = oracle.near_tie_positions(od, score_ref)
    n_acc = check_selection(D, idx.cpu().numpy(), idx_ref, score_ref, near)
    print(f"{w.name}: near-tie positions {int(near.sum())}, accepted differences {n_acc}")
    # the reported scores are the selected blocks' scores
    sg = scores.cpu().numpy()
    ig = idx.cpu().numpy()
    ref_sel = np.take_along_axis(score_ref, np.maximum(ig, 0), axis=-1)
    ok = ig >= 0
    assert np.abs(sg[ok] - ref_sel[ok]).max() <= 1e-4 * max(1.0, np.abs(score_ref).max())
    assert np.all(np.isneginf(sg[~ok]))


def test_summaries_partial_range_leaves_rest():
    w = synth.Workload("t", 1, 4, 2, 128, 128, 256, 6, 2, "bf16", 24)
    x = synth.draw(w)
    D = dims_of(w)
    summ = torch.full((1, 6, 2, 128), 7.0, device="cuda")
    hga_block_summaries(D, to_dev(x.k_hist), 2, 4, summ)
    torch.cuda.synchronize()
    s = summ.cpu().numpy().transpose(0, 2, 1, 3)
    ref = oracle.block_summaries(_odims(w), x.k_hist.f64)
    assert np.all(s[:, :, [0, 1, 4, 5]] == 7.0)
    assert np.abs(s[:, :, 2:4] - ref[:, :, 2:4]).max() < 1e-6


def test_select_q_zero_tie_rule():
    """Q = 0: every score is exactly 0; the tie rule picks blocks 0..K-1."""
    w = synth.Workload("t", 1, 4, 2, 128, 128, 256, 10, 4, "bf16", 25)
    x = synth.draw(w)
    D = dims_of(w)
    q = torch.zeros((1, 256, 4, 128), dtype=torch.bfloat16, device="cuda")
    summ = torch.empty((1, 10, 2, 128), device="cuda")
    idx = torch.empty((1, 2, 2, 4), dtype=torch.int32, device="cuda")
    hga_block_summaries(D, to_dev(x.k_hist), 0, 10, summ)
    hga_select_topk(D, q, summ, idx)
    torch.cuda.synchronize()
    assert np.all(idx.cpu().numpy() == np.arange(4))


# ------------------------------------------------------------------ attention forward + backward

ATTN_CASES = [
    synth.TINY_F32,                                                                              # fp32, SIMT
    synth.Workload("tc-small: Hq4/Hkv2 S384 hist5 K3", 1, 4, 2, 128, 128, 384, 5, 3, "bf16", 31),
    synth.Workload("tc-G2-B2: Hq4/Hkv2 S256 hist4 K2", 2, 4, 2, 128, 128, 256, 4, 2, "bf16", 32,
                   structured_keys=True),
    synth.Workload("tc-no-history: S512", 1, 4, 1, 128, 128, 512, 0, 4, "bf16", 33),
    synth.Workload("tc-K>hist: hist2 K5", 1, 8, 2, 128, 128, 256, 2, 5, "bf16", 34),
    synth.Workload("tc-K1: hist6 K1", 1, 4, 2, 128, 128, 256, 6, 1, "bf16", 35),
    synth.Workload("simt-bf16-d64-blk64-G3", 1, 6, 2, 64, 64, 192, 5, 2, "bf16", 36),
    # head dim 64 on the tensor-core path (one 64-column TMA box per tile)
    synth.Workload("tc-d64: Hq8/Hkv2 d64 S384 hist6 K3", 1, 8, 2, 64, 128, 384, 6, 3, "bf16", 41,
                   structured_keys=True),
    synth.Workload("tc-d64-B2-G2: B2 Hq4/Hkv2 d64 S256 hist3 K2", 2, 4, 2, 64, 128, 256, 3, 2, "bf16", 42),
    synth.Workload("simt-f32-d128-blk32", 1, 2, 2, 128, 32, 96, 6, 3, "f32", 37),
    # dK/dV: group sizes up to 8 sum the heads' parts in a thread-block cluster (8 and 6 here; 4 and 2
    # above); 16 heads per KV head add theirs into zeroed outputs
    synth.Workload("tc-G8: Hq16/Hkv2 d64 S256 hist5 K2", 1, 16, 2, 64, 128, 256, 5, 2, "bf16", 53),
    synth.Workload("tc-G6: Hq12/Hkv2 S384 hist4 K2", 1, 12, 2, 128, 128, 384, 4, 2, "bf16", 54),
    synth.Workload("tc-G16: Hq16/Hkv1 d64 S256 hist3 K2", 1, 16, 1, 64, 128, 256, 3, 2, "bf16", 55),
    # query blocks of another size than the history blocks (q_block != block); 128-row query blocks
    # with 64-, 32- or 16-token history blocks run on the tensor-core kernels, 128/block history
    # blocks per 128-key tile (the last tile short when K valid blocks do not fill it)
    synth.Workload("qblk128-blk64: Hq4/Hkv2 S256 hist10 K3", 1, 4, 2, 128, 64, 256, 10, 3, "bf16", 43,
                   structured_keys=True, qblk=128),
    synth.Workload("tc-blk64-K4: Hq8/Hkv2 S384 hist12 K4", 1, 8, 2, 128, 64, 384, 12, 4, "bf16", 46, qblk=128),
    synth.Workload("tc-blk64-d64-B2: B2 Hq4/Hkv2 d64 S256 hist9 K5", 2, 4, 2, 64, 64, 256, 9, 5, "bf16", 47,
                   qblk=128),
    synth.Workload("tc-blk64-K>hist: Hq4/Hkv2 S256 hist3 K8", 1, 4, 2, 128, 64, 256, 3, 8, "bf16", 48, qblk=128),
    synth.Workload("tc-blk32-K6: Hq4/Hkv2 S256 hist20 K6", 1, 4, 2, 128, 32, 256, 20, 6, "bf16", 49,
                   structured_keys=True, qblk=128),
    synth.Workload("tc-blk32-K>hist: Hq4/Hkv2 S256 hist3 K8", 1, 4, 2, 128, 32, 256, 3, 8, "bf16", 50, qblk=128),
    synth.Workload("tc-blk16-d64-K11: Hq8/Hkv2 d64 S384 hist40 K11", 1, 8, 2, 64, 16, 384, 40, 11, "bf16", 51,
                   qblk=128),
    synth.Workload("tc-blk16-K64: B2 Hq4/Hkv2 S256 hist80 K64", 2, 4, 2, 128, 16, 256, 80, 64, "bf16", 52,
                   structured_keys=True, qblk=128),
    synth.Workload("qblk64-blk128: B2 Hq4/Hkv2 d64 S256 hist5 K2", 2, 4, 2, 64, 128, 256, 5, 2, "bf16", 44, qblk=64),
    synth.Workload("qblk16-blk32-f32: Hq2/Hkv1 d64 S96 hist8 K3", 1, 2, 1, 64, 32, 96, 8, 3, "f32", 45, qblk=16),
]


@pytest.mark.parametrize("w", ATTN_CASES, ids=lambda w: w.name.split(":")[0])
def test_attention_small(w):
    x = synth.draw(w)
    st, _ = _gpu_step(w, x)
    od = _odims(w)
    idx_ref, score_ref = oracle.select(od, x.q.f64, x.k_hist.f64)
    idx = st.idx.cpu().numpy()
    check_selection(dims_of(w), idx, idx_ref, score_ref, oracle.near_tie_positions(od, score_ref))
    args = (x.q.f64, x.k_seg.f64, x.v_seg.f64, x.k_hist.f64, x.v_hist.f64, idx)
    o_ref, lse_ref = oracle.attn_fwd(od, *args)
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd(od, *args, x.d_o.f64)
    ma, rl = _tols(w)
    assert_close("O", to_host(st.o), o_ref, ma, rl)
    assert_close("LSE", to_host(st.lse), lse_ref, ma, rl)
    assert_close("dQ", to_host(st.dq), dq_ref, ma, rl)
    assert_close("dK", to_host(st.dk), dk_ref, ma, rl)
    assert_close("dV", to_host(st.dv), dv_ref, ma, rl)


@pytest.mark.parametrize("heads", [1, 2])
@pytest.mark.parametrize("name", ["tc-K>hist", "tc-d64-B2-G2", "tc-blk64-K4", "tc-blk16-d64-K11", "tc-G6"])
def test_forward_heads_per_cta(name, heads):
    """The forward with one query head per CTA and with a pair per CTA (the
    default picks by grid size), on the same tensor-core cases."""
    from segmented_fine_tuning_b200 import hga_set_forward_heads_per_cta
    w = next(c for c in ATTN_CASES if c.name.split(":")[0] == name)
    x = synth.draw(w)
    hga_set_forward_heads_per_cta(heads)
    try:
        st, _ = _gpu_step(w, x)
    finally:
        hga_set_forward_heads_per_cta(0)
    od = _odims(w)
    idx = st.idx.cpu().numpy()
    args = (x.q.f64, x.k_seg.f64, x.v_seg.f64, x.k_hist.f64, x.v_hist.f64, idx)
    o_ref, lse_ref = oracle.attn_fwd(od, *args)
    ma, rl = _tols(w)
    assert_close("O", to_host(st.o), o_ref, ma, rl)
    assert_close("LSE", to_host(st.lse), lse_ref, ma, rl)


def test_rescale_rows_diverge():
    """A history block late in the tile list dominates only the even query
    rows: their running maximum jumps mid-way (the O rescale path) while the
    odd rows of the same warps keep theirs."""
    w = synth.Workload("rescale: Hq2/Hkv1 S256 hist4 K2", 1, 2, 1, 128, 128, 256, 4, 2, "bf16", 40)
    x = synth.draw(w)
    q = x.q.f64.copy()
    kh = x.k_hist.f64.copy()
    q[:, ::2, :, :] = 0.0
    q[:, ::2, :, 0] = 10.0          # even rows: q = 10 e0
    kh[:, 3 * 128:4 * 128, :, 0] = 10.0  # block 3 keys: k0 = 10 -> logit ~8.8 nats for even rows
    x.q = synth._store(q, "bf16")
    x.k_hist = synth._store(kh, "bf16")
    st, _ = _gpu_step(w, x)
    idx = st.idx.cpu().numpy()
    assert np.all(idx[..., 1] == 3) and np.all(idx[..., 0] < 3)
    od = _odims(w)
    args = (x.q.f64, x.k_seg.f64, x.v_seg.f64, x.k_hist.f64, x.v_hist.f64, idx)
    o_ref, lse_ref = oracle.attn_fwd(od, *args)
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd(od, *args, x.d_o.f64)
    assert_close("O", to_host(st.o), o_ref, BF16_ABS, BF16_REL)
    assert_close("LSE", to_host(st.lse), lse_ref, BF16_ABS, BF16_REL)
    assert_close("dQ", to_host(st.dq), dq_ref, BF16_ABS, BF16_REL)
    assert_close("dK", to_host(st.dk), dk_ref, BF16_ABS, BF16_REL)
    assert_close("dV", to_host(st.dv), dv_ref, BF16_ABS, BF16_REL)


def test_dense_equivalence_full():
    """K = every history block: HGA equals dense causal attention; checked
    against the oracle's own dense path too, at full size."""
    w = synth.DENSE_EQUIV
    x = synth.draw(w)
    st, _ = _gpu_step(w, x)
    idx = st.idx.cpu().numpy()
    assert np.all(idx == np.arange(w.nblk))
    od = _odims(w)
    args = (x.q.f64, x.k_seg.f64, x.v_seg.f64, x.k_hist.f64, x.v_hist.f64, idx)
    o_ref, lse_ref = oracle.attn_fwd(od, *args)
    assert_close("O", to_host(st.o), o_ref, BF16_ABS, BF16_REL)
    assert_close("LSE", to_host(st.lse), lse_ref, BF16_ABS, BF16_REL)
    # dense identity on sampled rows
    H = w.nblk * w.blk
    qf = np.concatenate([np.zeros((1, H, w.Hq, w.d)), x.q.f64], 1)
    kf = np.concatenate([x.k_hist.f64, x.k_seg.f64], 1)
    vf = np.concatenate([x.v_hist.f64, x.v_seg.f64], 1)
    o_dense, _ = oracle.dense_causal_fwd(qf[:, :, :4], kf[:, :, :1], vf[:, :, :1])
    assert_close("O vs dense (head group 0)", to_host(st.o)[:, :, :4], o_dense[:, H:], BF16_ABS, BF16_REL)
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd(od, *args, x.d_o.f64)
    assert_close("dQ", to_host(st.dq), dq_ref, BF16_ABS, BF16_REL)
    assert_close("dK", to_host(st.dk), dk_ref, BF16_ABS, BF16_REL)
    assert_close("dV", to_host(st.dv), dv_ref, BF16_ABS, BF16_REL)


def test_qwen3_8b_layer_all_heads():
    """Full-size Qwen3-8B-shaped layer (the benchmark launch): selection over
    all heads; O/LSE/dQ/dK/dV element by element for all 8 KV heads and
    their 32 query heads (every head-dependent path of the kernels: the
    forward's head pairs, the per-head partial sums of dK/dV)."""
    w = synth.QWEN3_8B_LAYER
    x = synth.draw(w)
    st, _ = _gpu_step(w, x)
    od = _odims(w)
    idx_ref, score_ref = oracle.select(od, x.q.f64, x.k_hist.f64)
    idx = st.idx.cpu().numpy()
    check_selection(dims_of(w), idx, idx_ref, score_ref, oracle.near_tie_positions(od, score_ref))
    args = (x.q.f64, x.k_seg.f64, x.v_seg.f64, x.k_hist.f64, x.v_hist.f64, idx)
    o_ref, lse_ref = oracle.attn_fwd(od, *args)
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd(od, *args, x.d_o.f64)
    got = {"O": to_host(st.o), "LSE": to_host(st.lse), "dQ": to_host(st.dq), "dK": to_host(st.dk),
           "dV": to_host(st.dv)}
    for h in range(w.Hkv):
        hs = slice(w.G * h, w.G * h + w.G)
        assert_close(f"O h{h}", got["O"][:, :, hs], o_ref[:, :, hs], BF16_ABS, BF16_REL)
        assert_close(f"LSE h{h}", got["LSE"][:, hs], lse_ref[:, hs], BF16_ABS, BF16_REL)
        assert_close(f"dQ h{h}", got["dQ"][:, :, hs], dq_ref[:, :, hs], BF16_ABS, BF16_REL)
        assert_close(f"dK h{h}", got["dK"][:, :, h], dk_ref[:, :, h], BF16_ABS, BF16_REL)
        assert_close(f"dV h{h}", got["dV"][:, :, h], dv_ref[:, :, h], BF16_ABS, BF16_REL)


def test_prefill_131k_sampled():
    """131K-token prefill, forward only: selection over all heads; O/LSE of two
    rows per query block for KV heads 0 and 5."""
    w = synth.PREFILL_131K
    x = synth.draw(w)
    st, _ = _gpu_step(w, x, backward=False)
    od = _odims(w)
    idx_ref, score_ref = oracle.select(od, x.q.f64, x.k_hist.f64)
    idx = st.idx.cpu().numpy()
    check_selection(dims_of(w), idx, idx_ref, score_ref, oracle.near_tie_positions(od, score_ref))
    rows = sorted({i * w.blk + r for i in range(w.nqb) for r in (0, 127 - (i % 7) * 9)})
    args = (x.q.f64, x.k_seg.f64, x.v_seg.f64, x.k_hist.f64, x.v_hist.f64, idx)
    for h in (0, 5):
        o_ref, lse_ref = oracle.attn_fwd(od, *args, kv_heads=range(h, h + 1), rows=rows)
        hs = slice(4 * h, 4 * h + 4)
        assert_close(f"O h{h}", to_host(st.o)[:, rows][:, :, hs], o_ref[:, rows][:, :, hs], BF16_ABS, BF16_REL)
        assert_close(f"LSE h{h}", to_host(st.lse)[:, hs][:, :, rows], lse_ref[:, hs][:, :, rows], BF16_ABS,
                     BF16_REL)


def test_out_of_range_index_is_flagged_not_faulted():
    """A bad block index in idx is skipped by the kernels and reported."""
    w = synth.Workload("t", 1, 4, 2, 128, 128, 256, 4, 2, "bf16", 38)
    x = synth.draw(w)
    D = dims_of(w)
    dev = {n: to_dev(getattr(x, n)) for n in ("q", "k_seg", "v_seg", "k_hist", "v_hist")}
    idx = torch.tensor([0, 9], dtype=torch.int32).repeat(1, 2, 2, 1).contiguous().cuda()
    o = torch.empty_like(dev["q"])
    lse = torch.empty((1, 4, 256), device="cuda")
    hga_attn_fwd(D, dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], 4, idx, o, lse)
    with pytest.raises(HgaError) as ei:
        hga_device_status()
    assert ei.value.status == 4
    hga_device_status()  # flag cleared
    # the valid part was still computed: equals attention with idx [0, -1]
    idx2 = torch.tensor([0, -1], dtype=torch.int32).repeat(1, 2, 2, 1).contiguous().cuda()
    o2 = torch.empty_like(o)
    lse2 = torch.empty_like(lse)
    hga_attn_fwd(D, dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], 4, idx2, o2, lse2)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_repeat_runs_bit_identical_forward():
    w = synth.Workload("t", 1, 8, 2, 128, 128, 512, 6, 3, "bf16", 39, structured_keys=True)
    x = synth.draw(w)
    st1, dev = _gpu_step(w, x, backward=False)
    o1, lse1, idx1 = st1.o.clone(), st1.lse.clone(), st1.idx.clone()
    st1.select(dev["q"], dev["k_hist"])
    st1.forward(dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"])
    torch.cuda.synchronize()
    assert torch.equal(idx1, st1.idx) and torch.equal(o1, st1.o) and torch.equal(lse1, st1.lse)
