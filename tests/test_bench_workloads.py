"""bench.py's algorithmic work model against hand counts (no GPU).

The layer workload (B1, 32 query heads, d 128, S 2,048, K 16 of 128-token
blocks under 128-row query blocks): per query head 16 query blocks x 16
blocks x 128 x 128 history pairs and S(S+1)/2 causal segment pairs, 4d FLOP
per pair.  The 64- and 32-token variants keep the same history keys per query
block (K 32 and 64), so their attention work is the same.
"""
import importlib.util
import os
import sys

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def test_layer_flops_by_hand():
    b = _bench()
    w = synth.QWEN3_8B_LAYER
    flops, bytes_ = b.work_model(w, keff_sum_per_head=16 * 16)
    hist = 16 * 16 * 128 * 128            # query blocks x K x q_block rows x block keys
    seg = 2048 * 2049 // 2
    assert hist == 4_194_304 and seg == 2_098_176
    assert flops["fwd"] == 4 * 128 * (hist + seg) * 32 == 103_095_992_320
    assert flops["bwd_dq"] == flops["fwd"]
    assert flops["bwd_dkdv"] == 4 * 128 * seg * 32
    # summaries: the history keys in bf16 plus the fp32 summaries
    assert bytes_["summaries"] == 112 * 128 * 8 * 128 * 2 + 8 * 112 * 128 * 4
    # preprocess: O and dO in bf16, Dr in fp32
    assert bytes_["bwd_pre"] == 2 * 2048 * 32 * 128 * 2 + 32 * 2048 * 4


def test_smaller_history_blocks_keep_the_work():
    b = _bench()
    ref, _ = b.work_model(synth.QWEN3_8B_LAYER, keff_sum_per_head=16 * 16)
    for w in (synth.QWEN3_8B_LAYER64, synth.QWEN3_8B_LAYER32):
        assert w.qb == 128 and w.blk * w.topk == 128 * 16 and w.nblk * w.blk == 112 * 128
        flops, _ = b.work_model(w, keff_sum_per_head=w.nqb * w.topk)
        assert flops == ref, w.name
