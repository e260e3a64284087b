"""The full segmented pass: 36 Qwen3-8B-shaped layers over a 16,384-token
sequence cut into 8 segments of 2,048.  History grows by 16 blocks per
segment and lives in a pinned host tier; the selected blocks are fetched per
(layer, segment); summaries are appended on the device at each segment end.

Checked against the fp64 oracle: every one of the 288 (layer, segment)
selections; O, LSE, dQ, dK, dV for layers 0, 17 and 35 in every segment
(KV heads 0 and 5 with their 4 query heads each).  Layers are independent and
identically shaped, so the subset covers every segment shape.  Setting
HGA_FULL_SWEEP=1 checks outputs for every layer and KV head (a long job).
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
L, NS = synth.SEGMENTED_LAYERS, synth.SEGMENTED_SEGMENTS
CHECK_LAYERS = range(L) if FULL else (0, 17, 35)
CHECK_HEADS = range(8) if FULL else (0, 5)


def test_segmented_pass_36_layers_8_segments():
    w = synth.QWEN3_8B_LAYER
    seg = Dims(1, w.Hq, w.Hkv, w.d, w.blk, w.S, 0, w.topk, "bf16")
    sp = SegmentedPass(seg, L, NS)
    nqb = w.S // w.blk
    # oracle-side state: resident summaries per layer (fp64, oracle layout
    # [B, Hkv, n, d]), full history K/V for the checked layers
    o_summ = [np.zeros((1, w.Hkv, 0, w.d)) for _ in range(L)]
    o_hist = {l: (np.zeros((1, 0, w.Hkv, w.d)), np.zeros((1, 0, w.Hkv, w.d))) for l in CHECK_LAYERS}
    n_near, n_acc, n_checked = 0, 0, 0
    for s in range(NS):
        xs = [synth.draw_segment(w, l, s) for l in range(L)]
        dev = [tuple(to_dev(t) for t in (x.q, x.k_seg, x.v_seg, x.d_o)) for x in xs]
        nh = s * nqb
        od = oracle.Dims(1, w.Hq, w.Hkv, w.d, w.blk, w.S, nh, w.topk)
        saved = {}

        def on_step(s_, l, phase):
            nonlocal n_near, n_acc, n_checked
            x = xs[l]
            if phase == "fwd":
                torch.cuda.synchronize()
                idx = sp.idx[l].cpu().numpy()
                q64 = x.q.f64
                if nh > 0:
                    score = oracle.block_scores(od, oracle.query_means(od, q64), o_summ[l])
                    idx_ref = oracle.select_topk(od, score)
                    near = oracle.near_tie_positions(od, score)
                    n_near += int(near.sum())
                    n_acc += check_selection(sp.dims(s), idx, idx_ref, score, near)
                else:
                    assert np.all(idx == -1)
                if l in CHECK_LAYERS:
                    saved[l] = (idx, to_host(sp.o[l]), to_host(sp.lse[l]))
            elif l in CHECK_LAYERS:
                torch.cuda.synchronize()
                idx, o_g, lse_g = saved[l]
                dq_g, dk_g, dv_g = to_host(sp.dq), to_host(sp.dk), to_host(sp.dv)
                kh, vh = o_hist[l]
                args = (x.q.f64, x.k_seg.f64, x.v_seg.f64, kh, vh, idx)
                for h in CHECK_HEADS:
                    hs = slice(h * w.G, (h + 1) * w.G)
                    o_r, lse_r = oracle.attn_fwd(od, *args, kv_heads=range(h, h + 1))
                    dq_r, dk_r, dv_r = oracle.attn_bwd(od, *args, x.d_o.f64, kv_heads=range(h, h + 1))
                    tag = f"layer {l} segment {s} head {h}"
                    assert_close(f"O {tag}", o_g[:, :, hs], o_r[:, :, hs], BF16_ABS, BF16_REL)
                    assert_close(f"LSE {tag}", lse_g[:, hs], lse_r[:, hs], BF16_ABS, BF16_REL)
                    assert_close(f"dQ {tag}", dq_g[:, :, hs], dq_r[:, :, hs], BF16_ABS, BF16_REL)
                    assert_close(f"dK {tag}", dk_g[:, :, h], dk_r[:, :, h], BF16_ABS, BF16_REL)
                    assert_close(f"dV {tag}", dv_g[:, :, h], dv_r[:, :, h], BF16_ABS, BF16_REL)
                n_checked += 1

        sp.run_segment(s, dev, on_step)
        torch.cuda.synchronize()
        hga_device_status()
        # the segment enters the history: oracle summaries of its blocks, and
        # the device's appended summaries and host tier agree with them
        for l in range(L):
            ks = xs[l].k_seg.f64
            new = oracle.block_summaries(oracle.Dims(1, w.Hq, w.Hkv, w.d, w.blk, w.S, nqb, w.topk), ks)
            o_summ[l] = np.concatenate([o_summ[l], new], axis=2)
            if l in CHECK_LAYERS:
                kh, vh = o_hist[l]
                o_hist[l] = (np.concatenate([kh, ks], 1), np.concatenate([vh, xs[l].v_seg.f64], 1))
        for l in (0, L - 1):
            g = sp.summ[l][:, : (s + 1) * nqb].cpu().numpy().transpose(0, 2, 1, 3)
            assert np.abs(g - o_summ[l]).max() < 1e-6 * max(1.0, np.abs(o_summ[l]).max())
            # the segment's K/V landed in the host tier at its blocks
            rows = slice(s * nqb * w.blk, (s + 1) * nqb * w.blk)
            for tier, t in ((sp.tier_k[l], xs[l].k_seg), (sp.tier_v[l], xs[l].v_seg)):
                want = torch.from_numpy(np.ascontiguousarray(t.store).view(np.int16)).view(torch.bfloat16)
                assert torch.equal(tier[:, rows], want)
    print(f"selections: {L * (NS - 1)} steps with history, near-tie positions {n_near}, accepted {n_acc}; "
          f"outputs checked for {n_checked} (layer, segment) steps; blocks copied over the host link per step "
          f"mean {np.mean(sp.fetched_blocks):.1f}; steps remapped on the device {sp.device_remaps}")
    assert n_checked == len(CHECK_LAYERS) * NS
    # finished segments enter each layer's device cache, which holds the whole
    # history: nothing crosses the host link and every step remaps on the device
    copied = np.array(sp.fetched_blocks).reshape(NS - 1, L)
    assert (copied == 0).all() and sp.device_remaps == L * (NS - 1)
