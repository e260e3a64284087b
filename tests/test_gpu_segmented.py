"""The full segmented pass: Qwen3-8B-shaped layers over a 16,384-token
sequence cut into 8 segments of 2,048.  History grows by 16 blocks per
segment and lives in a pinned host tier; the selected blocks reach the
device either through the layer's device block cache or over the host link;
summaries are appended on the device at each segment end.

Three modes, each checked against the fp64 oracle:
  - resident cache (the default): 36 layers; every one of the 288 selections;
    O, LSE, dQ, dK, dV for layers 0, 17 and 35 in every segment (KV heads 0
    and 5 with their 4 query heads each).  Layers are independent and
    identically shaped, so the subset covers every segment shape.  Setting
    HGA_FULL_SWEEP=1 checks outputs for every layer and KV head (a long job).
  - host tier, no insert: layers 0, 17 and 35 with a pool of the largest
    history (112 blocks) and finished segments NOT inserted into it, so every
    step's new blocks are copied from pinned host memory (misses > 0); all
    outputs of the three layers checked, two KV heads per step rotating so
    that all 8 heads are covered.
  - evicting cache: a smaller layer (Hq8/Hkv2, S512, K3) over 8 segments with
    an 18-slot pool, below the 28-block history, so that blocks are evicted
    and fetched again; every selection and every output checked.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from hga_testutil import BF16_ABS, BF16_REL, assert_close, check_selection, to_dev, to_host
from segmented_fine_tuning_b200 import Dims, hga_device_status
from segmented_fine_tuning_b200.segmented import SegmentedPass

pytestmark = pytest.mark.gpu

FULL = os.environ.get("HGA_FULL_SWEEP") == "1"
NS = synth.SEGMENTED_SEGMENTS
SMALL = synth.Workload("segmented-small: B1 Hq8/Hkv2 d128, S512, K3", 1, 8, 2, 128, 128, 512, 0, 3, "bf16", 0,
                       structured_keys=True)


def run_pass(w, layer_ids, check_layers, heads_of, pool_slots=None, keep_new_blocks=True):
    """Runs SegmentedPass over the given layers (layer_ids[l] names the seed of
    pass layer l) and checks it against the oracle.  heads_of(l, s) lists the
    KV heads whose outputs are compared at (pass layer l, segment s).
    Returns the pass (for its fetch statistics)."""
    L = len(layer_ids)
    seg = Dims(1, w.Hq, w.Hkv, w.d, w.blk, w.S, 0, w.topk, "bf16")
    sp = SegmentedPass(seg, L, NS, pool_slots=pool_slots, keep_new_blocks=keep_new_blocks)
    nqb = w.S // w.blk
    # oracle-side state: resident summaries per layer (fp64, oracle layout
    # [B, Hkv, n, d]), full history K/V for the checked layers
    o_summ = [np.zeros((1, w.Hkv, 0, w.d)) for _ in range(L)]
    o_hist = {l: (np.zeros((1, 0, w.Hkv, w.d)), np.zeros((1, 0, w.Hkv, w.d))) for l in check_layers}
    stats = {"near": 0, "accepted": 0, "checked": 0}
    sp.ever_selected = [set() for _ in range(L)]
    for s in range(NS):
        xs = [synth.draw_segment(w, layer_ids[l], s) for l in range(L)]
        dev = [tuple(to_dev(t) for t in (x.q, x.k_seg, x.v_seg, x.d_o)) for x in xs]
        nh = s * nqb
        od = oracle.Dims(1, w.Hq, w.Hkv, w.d, w.blk, w.S, nh, w.topk)
        saved = {}

        def on_step(s_, l, phase):
            x = xs[l]
            if phase == "fwd":
                torch.cuda.synchronize()
                idx = sp.idx[l].cpu().numpy()
                sp.ever_selected[l] |= set(idx.ravel().tolist()) - {-1}
                if nh > 0:
                    score = oracle.block_scores(od, oracle.query_means(od, x.q.f64), o_summ[l])
                    idx_ref = oracle.select_topk(od, score)
                    near = oracle.near_tie_positions(od, score)
                    stats["near"] += int(near.sum())
                    stats["accepted"] += check_selection(sp.dims(s), idx, idx_ref, score, near)
                else:
                    assert np.all(idx == -1)
                if l in check_layers:
                    saved[l] = (idx, to_host(sp.o[l]), to_host(sp.lse[l]))
            elif l in check_layers:
                torch.cuda.synchronize()
                idx, o_g, lse_g = saved[l]
                dq_g, dk_g, dv_g = to_host(sp.dq), to_host(sp.dk), to_host(sp.dv)
                kh, vh = o_hist[l]
                args = (x.q.f64, x.k_seg.f64, x.v_seg.f64, kh, vh, idx)
                for h in heads_of(l, s):
                    hs = slice(h * w.G, (h + 1) * w.G)
                    o_r, lse_r = oracle.attn_fwd(od, *args, kv_heads=range(h, h + 1))
                    dq_r, dk_r, dv_r = oracle.attn_bwd(od, *args, x.d_o.f64, kv_heads=range(h, h + 1))
                    tag = f"layer {layer_ids[l]} segment {s} head {h}"
                    assert_close(f"O {tag}", o_g[:, :, hs], o_r[:, :, hs], BF16_ABS, BF16_REL)
                    assert_close(f"LSE {tag}", lse_g[:, hs], lse_r[:, hs], BF16_ABS, BF16_REL)
                    assert_close(f"dQ {tag}", dq_g[:, :, hs], dq_r[:, :, hs], BF16_ABS, BF16_REL)
                    assert_close(f"dK {tag}", dk_g[:, :, h], dk_r[:, :, h], BF16_ABS, BF16_REL)
                    assert_close(f"dV {tag}", dv_g[:, :, h], dv_r[:, :, h], BF16_ABS, BF16_REL)
                stats["checked"] += 1

        sp.run_segment(s, dev, on_step)
        torch.cuda.synchronize()
        hga_device_status()
        # the segment enters the history: oracle summaries of its blocks, and
        # the device's appended summaries and host tier agree with them
        for l in range(L):
            ks = xs[l].k_seg.f64
            new = oracle.block_summaries(oracle.Dims(1, w.Hq, w.Hkv, w.d, w.blk, w.S, nqb, w.topk), ks)
            o_summ[l] = np.concatenate([o_summ[l], new], axis=2)
            if l in check_layers:
                kh, vh = o_hist[l]
                o_hist[l] = (np.concatenate([kh, ks], 1), np.concatenate([vh, xs[l].v_seg.f64], 1))
        for l in sorted({0, L - 1}):
            g = sp.summ[l][:, : (s + 1) * nqb].cpu().numpy().transpose(0, 2, 1, 3)
            assert np.abs(g - o_summ[l]).max() < 1e-6 * max(1.0, np.abs(o_summ[l]).max())
            # the segment's K/V landed in the host tier at its blocks
            rows = slice(s * nqb * w.blk, (s + 1) * nqb * w.blk)
            for tier, t in ((sp.tier_k[l], xs[l].k_seg), (sp.tier_v[l], xs[l].v_seg)):
                want = torch.from_numpy(np.ascontiguousarray(t.store).view(np.int16)).view(torch.bfloat16)
                assert torch.equal(tier[:, rows], want)
    print(f"{w.name} pool {sp.pool_slots} keep_new_blocks {keep_new_blocks}: {L * (NS - 1)} selections with "
          f"history, near-tie positions {stats['near']}, accepted {stats['accepted']}; outputs checked for "
          f"{stats['checked']} (layer, segment) steps; blocks copied over the host link per step "
          f"{sp.fetched_blocks}; steps remapped on the device {sp.device_remaps}")
    assert stats["checked"] == len(check_layers) * NS
    return sp


def test_segmented_pass_36_layers_8_segments():
    w = synth.QWEN3_8B_LAYER
    L = synth.SEGMENTED_LAYERS
    layers = list(range(L))
    check = set(range(L)) if FULL else {0, 17, 35}
    heads = (lambda l, s: range(8)) if FULL else (lambda l, s: (0, 5))
    sp = run_pass(w, layers, check, heads)
    # finished segments enter each layer's device cache, which holds the whole
    # history: nothing crosses the host link and every step remaps on the device
    copied = np.array(sp.fetched_blocks).reshape(NS - 1, L)
    assert (copied == 0).all() and sp.device_remaps == L * (NS - 1)


def test_segmented_pass_host_tier_fetch():
    """History served from the pinned host tier: the pool (112 slots) is not
    filled at segment end, so each step copies the blocks it has not seen
    (the previous segment's 16) over the host link."""
    w = synth.QWEN3_8B_LAYER
    layers = [0, 17, 35]
    sp = run_pass(w, layers, {0, 1, 2}, lambda l, s: ((l + s) % 8, (l + s + 4) % 8), pool_slots=112,
                  keep_new_blocks=False)
    copied = np.array(sp.fetched_blocks).reshape(NS - 1, len(layers))
    assert sp.device_remaps == 0
    # every selectable block of this workload is selected by some query block
    # of some head, so each step copies exactly the previous segment's blocks
    assert (copied == 16).all(), copied


@pytest.mark.parametrize("keep_new_blocks", [False, True])
def test_segmented_pass_evicting_cache(keep_new_blocks):
    """An 18-slot pool under a history that grows to 28 blocks: blocks are
    evicted (least recently used first) and fetched again later."""
    sp = run_pass(SMALL, [0, 1], {0, 1}, lambda l, s: range(SMALL.Hkv), pool_slots=18,
                  keep_new_blocks=keep_new_blocks)
    copied = np.array(sp.fetched_blocks)
    assert copied.sum() > 0
    if not keep_new_blocks:
        # more copies than distinct blocks ever selected: some block was
        # evicted and later fetched again
        assert copied.sum() > sum(len(x) for x in sp.ever_selected)
