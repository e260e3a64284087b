"""Bounded waits, host side and device side, made to run out on purpose --
without faulting or hanging the GPU.

Host side: hga_fetch_blocks and hga_fetch_blocks_cached wait (at most
timeout_ms) for their small idx copy.  A bounded spin kernel queued on the
compute stream before the call delays that copy past a 1 ms limit: the call
must return HGA_ERR_TIMEOUT, queue no pool copy, and leave the block cache
as it was.

Device side: every mbarrier wait of the attention kernels gives up after 1 s.
hga_selftest_attn_fwd_stalled runs the tensor-core forward with its K/V loads
withheld, so the MMA warp's wait can never be satisfied: the CTA must take its
abort path (free tensor memory, return), hga_device_status must report
HGA_ERR_TIMEOUT, and the context must stay usable (the same forward run
normally afterwards still matches the oracle).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from hga_testutil import BF16_ABS, BF16_REL, assert_close, dims_of, to_dev, to_host
from segmented_fine_tuning_b200 import (BlockCache, HgaError, hga_attn_fwd, hga_device_status, hga_fetch_blocks,
                                        hga_fetch_blocks_cached, hga_selftest_attn_fwd_stalled)

pytestmark = pytest.mark.gpu

HGA_ERR_TIMEOUT = 5
SPIN_CYCLES = 400_000_000  # ~0.2 s of a bounded spin kernel at B200 clocks


def _tier_case():
    w = synth.Workload("timeout: Hq4/Hkv2 S256 hist6 K3", 1, 4, 2, 128, 128, 256, 6, 3, "bf16", 61)
    D = dims_of(w)
    x = synth.draw(w)
    tier_k = torch.from_numpy(np.ascontiguousarray(x.k_hist.store).view(np.int16)).view(torch.bfloat16).pin_memory()
    tier_v = torch.from_numpy(np.ascontiguousarray(x.v_hist.store).view(np.int16)).view(torch.bfloat16).pin_memory()
    idx = torch.tensor([[0, 2, 4], [1, 3, 5]], dtype=torch.int32).reshape(1, 1, 2, 3).repeat(1, 2, 1, 1).cuda()
    return w, D, tier_k, tier_v, idx


def test_fetch_blocks_times_out_and_copies_nothing():
    w, D, tier_k, tier_v, idx = _tier_case()
    scratch = torch.empty(tuple(idx.shape), dtype=torch.int32).pin_memory()
    pool = torch.full((1, 6 * 128, 2, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    pool_v = torch.full_like(pool, float("nan"))
    ip = torch.full_like(idx, -7)
    cs = torch.cuda.Stream()
    done = torch.cuda.Event()
    done.record(cs)
    torch.cuda.synchronize()
    torch.cuda._sleep(SPIN_CYCLES)  # delays the idx copy, which waits for the compute stream
    with pytest.raises(HgaError) as e:
        hga_fetch_blocks(D, tier_k, tier_v, 6, idx, scratch, pool, pool_v, 6, ip, torch.cuda.current_stream(), cs,
                         done, timeout_ms=1)
    assert e.value.status == HGA_ERR_TIMEOUT
    assert "did not complete within 1 ms" in str(e.value)
    # the idx copy into the scratch is still pending on the copy stream: drain it first
    cs.synchronize()
    torch.cuda.synchronize()
    assert torch.isnan(pool.float()).all() and torch.isnan(pool_v.float()).all()
    assert (ip == -7).all()
    # the same call with time to spare succeeds
    nu = hga_fetch_blocks(D, tier_k, tier_v, 6, idx, scratch, pool, pool_v, 6, ip, torch.cuda.current_stream(), cs,
                          done)
    torch.cuda.synchronize()
    assert nu == 6 and torch.equal(pool.cpu(), tier_k)


def test_cached_fetch_timeout_leaves_cache_unchanged():
    w, D, tier_k, tier_v, idx = _tier_case()
    scratch = torch.empty(tuple(idx.shape), dtype=torch.int32).pin_memory()
    cache = BlockCache(6, 6)
    pool = torch.full((1, 6 * 128, 2, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    pool_v = torch.full_like(pool, float("nan"))
    ip = torch.empty_like(idx)
    cs = torch.cuda.Stream()
    done = torch.cuda.Event()
    done.record(cs)
    before = (cache.slot_of_block.copy(), cache.block_of_slot.copy(), cache.last_use.copy(), cache.c.tick)
    torch.cuda.synchronize()
    torch.cuda._sleep(SPIN_CYCLES)
    with pytest.raises(HgaError) as e:
        hga_fetch_blocks_cached(D, tier_k, tier_v, idx, scratch, pool, pool_v, cache, ip,
                                torch.cuda.current_stream(), cs, done, timeout_ms=1)
    assert e.value.status == HGA_ERR_TIMEOUT
    cs.synchronize()
    torch.cuda.synchronize()
    after = (cache.slot_of_block, cache.block_of_slot, cache.last_use, cache.c.tick)
    for a, b in zip(before[:3], after[:3]):
        assert np.array_equal(a, b)
    assert before[3] == after[3]
    assert torch.isnan(pool.float()).all()
    nu, nf = hga_fetch_blocks_cached(D, tier_k, tier_v, idx, scratch, pool, pool_v, cache, ip,
                                     torch.cuda.current_stream(), cs, done)
    torch.cuda.synchronize()
    assert (nu, nf) == (6, 6)


def test_device_wait_timeout_is_reported_and_context_survives():
    w = synth.Workload("stall: Hq4/Hkv2 S256 hist4 K2", 1, 4, 2, 128, 128, 256, 4, 2, "bf16", 62)
    x = synth.draw(w)
    D = dims_of(w)
    dev = {n: to_dev(getattr(x, n)) for n in ("q", "k_seg", "v_seg", "k_hist", "v_hist")}
    idx = torch.tensor([1, 3], dtype=torch.int32).repeat(1, 2, 2, 1).contiguous().cuda()
    o = torch.zeros_like(dev["q"])
    lse = torch.zeros((1, 4, 256), device="cuda")
    hga_device_status()
    hga_selftest_attn_fwd_stalled(D, dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], 4, idx, o,
                                  lse)
    with pytest.raises(HgaError) as e:
        hga_device_status()
    assert e.value.status == HGA_ERR_TIMEOUT
    assert torch.count_nonzero(lse) == 0  # nothing written on the abort path
    hga_device_status()  # the flag was cleared
    # the context is intact: the normal forward still matches the oracle
    hga_attn_fwd(D, dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], 4, idx, o, lse)
    torch.cuda.synchronize()
    hga_device_status()
    od = oracle.Dims(w.B, w.Hq, w.Hkv, w.d, w.blk, w.S, w.nblk, w.topk)
    o_ref, lse_ref = oracle.attn_fwd(od, x.q.f64, x.k_seg.f64, x.v_seg.f64, x.k_hist.f64, x.v_hist.f64,
                                     idx.cpu().numpy())
    assert_close("O after the stalled launch", to_host(o), o_ref, BF16_ABS, BF16_REL)
    assert_close("LSE after the stalled launch", to_host(lse), lse_ref, BF16_ABS, BF16_REL)
