"""Host KV tier: targeted loading of the selected history blocks from pinned
host memory (hga_fetch_blocks) and the segment-end offload
(hga_offload_segment), through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import synth
from hga_testutil import BF16_ABS, BF16_REL, assert_close, dims_of, to_dev, to_host
from segmented_fine_tuning_b200 import (BlockCache, HgaError, hga_attn_bwd, hga_attn_fwd, hga_cache_segment,
                                        hga_device_status, hga_fetch_blocks, hga_fetch_blocks_cached,
                                        hga_offload_segment, hga_remap_idx)
from segmented_fine_tuning_b200.step import AttentionStep

pytestmark = pytest.mark.gpu


def _pinned(t: synth.Tensor):
    return torch.from_numpy(np.ascontiguousarray(t.store).view(np.int16)).view(torch.bfloat16).pin_memory()


def _oracle_check(tag, w, x, idx_blocks, o, lse, dq=None, dk=None, dv=None):
    """Outputs computed over a fetched pool against the fp64 oracle run on
    the resident history with the block numbers the pool slots stand for."""
    od = oracle.Dims(w.B, w.Hq, w.Hkv, w.d, w.blk, w.S, w.nblk, w.topk)
    args = (x.q.f64, x.k_seg.f64, x.v_seg.f64, x.k_hist.f64, x.v_hist.f64, idx_blocks)
    o_r, lse_r = oracle.attn_fwd(od, *args)
    assert_close(f"{tag} O", to_host(o), o_r, BF16_ABS, BF16_REL)
    assert_close(f"{tag} LSE", to_host(lse), lse_r, BF16_ABS, BF16_REL)
    if dq is not None:
        dq_r, dk_r, dv_r = oracle.attn_bwd(od, *args, x.d_o.f64)
        assert_close(f"{tag} dQ", to_host(dq), dq_r, BF16_ABS, BF16_REL)
        assert_close(f"{tag} dK", to_host(dk), dk_r, BF16_ABS, BF16_REL)
        assert_close(f"{tag} dV", to_host(dv), dv_r, BF16_ABS, BF16_REL)


@pytest.mark.parametrize("capacity_extra", [0, 3])
def test_fetch_into_pool_matches_oracle(capacity_extra):
    """The selected blocks fetched from a pinned host tier into a compact pool
    (slots in ascending block order), then forward and backward over the
    pool: O, LSE, dQ, dK, dV against the fp64 oracle over the full history,
    and equal to the same kernels run over the resident history."""
    w = synth.Workload("tier: Hq8/Hkv2 S512 hist20 K3", 1, 8, 2, 128, 128, 512, 20, 3, "bf16", 41,
                       structured_keys=True)
    x = synth.draw(w)
    D = dims_of(w)
    dev = {n: to_dev(getattr(x, n)) for n in ("q", "k_seg", "v_seg", "k_hist", "v_hist", "d_o")}
    st = AttentionStep(D)
    st.run(dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], dev["d_o"])
    torch.cuda.synchronize()
    o_ref, lse_ref, dq_ref = st.o.clone(), st.lse.clone(), st.dq.clone()
    dk_ref, dv_ref = st.dk.clone(), st.dv.clone()

    cap = w.nblk + capacity_extra
    tier_k = torch.zeros((1, cap * 128, 2, 128), dtype=torch.bfloat16).pin_memory()
    tier_v = torch.zeros_like(tier_k).pin_memory()
    tier_k[:, : w.nblk * 128] = _pinned(x.k_hist)
    tier_v[:, : w.nblk * 128] = _pinned(x.v_hist)
    scratch = torch.empty(tuple(st.idx.shape), dtype=torch.int32).pin_memory()
    n_sel = len(set(st.idx.cpu().numpy().ravel().tolist()) - {-1})
    pool_slots = n_sel + 1
    pool_k = torch.full((1, pool_slots * 128, 2, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    pool_v = torch.full_like(pool_k, float("nan"))
    idx_pool = torch.empty_like(st.idx)
    copy_stream = torch.cuda.Stream()
    done = torch.cuda.Event()
    done.record(copy_stream)
    nu = hga_fetch_blocks(D, tier_k, tier_v, cap, st.idx, scratch, pool_k, pool_v, pool_slots, idx_pool,
                          torch.cuda.current_stream(), copy_stream, done)
    torch.cuda.current_stream().wait_event(done)
    assert nu == n_sel
    # pool slot s holds the s-th smallest selected block
    sel = sorted(set(st.idx.cpu().numpy().ravel().tolist()) - {-1})
    ip = idx_pool.cpu().numpy()
    ig = st.idx.cpu().numpy()
    assert np.array_equal(np.where(ig >= 0, np.searchsorted(sel, np.maximum(ig, 0)), -1), ip)
    o = torch.empty_like(st.o)
    lse = torch.empty_like(st.lse)
    hga_attn_fwd(D, dev["q"], dev["k_seg"], dev["v_seg"], pool_k, pool_v, pool_slots, idx_pool, o, lse)
    dq, dk, dv = torch.empty_like(st.dq), torch.empty_like(st.dk), torch.empty_like(st.dv)
    hga_attn_bwd(D, dev["q"], dev["k_seg"], dev["v_seg"], pool_k, pool_v, pool_slots, idx_pool, o, lse,
                 dev["d_o"], dq, dk, dv, st.ws)
    torch.cuda.synchronize()
    hga_device_status()
    _oracle_check("pool", w, x, st.idx.cpu().numpy(), o, lse, dq, dk, dv)
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref) and torch.equal(dq, dq_ref)
    # dK/dV accumulate per-head partials with atomics: equal up to summation order
    assert torch.allclose(dk, dk_ref, rtol=0, atol=1e-5) and torch.allclose(dv, dv_ref, rtol=0, atol=1e-5)


def test_fetch_rejects_small_pool_and_bad_index():
    w = synth.Workload("t", 1, 4, 2, 128, 128, 256, 6, 3, "bf16", 42)
    D = dims_of(w)
    idx = torch.tensor([[0, 2, 4], [1, 3, 5]], dtype=torch.int32).reshape(1, 1, 2, 3).repeat(1, 2, 1, 1).cuda()
    tier = torch.zeros((1, 6 * 128, 2, 128), dtype=torch.bfloat16).pin_memory()
    scratch = torch.empty((1, 2, 2, 3), dtype=torch.int32).pin_memory()
    pool = torch.empty((1, 4 * 128, 2, 128), dtype=torch.bfloat16, device="cuda")
    ip = torch.empty_like(idx)
    cs = torch.cuda.Stream()
    ev = torch.cuda.Event()
    ev.record(cs)
    with pytest.raises(HgaError) as e:
        hga_fetch_blocks(D, tier, tier, 6, idx, scratch, pool, pool, 4, ip, torch.cuda.current_stream(), cs, ev)
    assert e.value.status == 1
    bad = idx.clone()
    bad[0, 0, 0, 0] = 17
    pool6 = torch.empty((1, 6 * 128, 2, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(HgaError) as e:
        hga_fetch_blocks(D, tier, tier, 6, bad, scratch, pool6, pool6, 6, ip, torch.cuda.current_stream(), cs, ev)
    assert e.value.status == 4
    torch.cuda.synchronize()


def test_offload_segment_into_tier():
    w = synth.Workload("t", 2, 4, 2, 128, 128, 256, 3, 2, "bf16", 43)
    x = synth.draw(w)
    D = dims_of(w)
    ks, vs = to_dev(x.k_seg), to_dev(x.v_seg)
    cap = 8
    tk = torch.zeros((2, cap * 128, 2, 128), dtype=torch.bfloat16).pin_memory()
    tv = torch.zeros_like(tk).pin_memory()
    hga_offload_segment(D, ks, vs, tk, tv, cap, 5)
    torch.cuda.synchronize()
    assert torch.equal(tk[:, 5 * 128: 7 * 128], ks.cpu()) and torch.equal(tv[:, 5 * 128: 7 * 128], vs.cpu())
    assert torch.count_nonzero(tk[:, : 5 * 128]) == 0 and torch.count_nonzero(tk[:, 7 * 128:]) == 0
    with pytest.raises(HgaError):
        hga_offload_segment(D, ks, vs, tk, tv, cap, 7)


def test_cached_fetch_reuses_resident_blocks_and_evicts():
    """hga_fetch_blocks_cached: a repeated selection copies nothing; a new
    selection through a pool that cannot hold both copies only the missing
    blocks, evicting the least recently used; the forward over the pool
    equals the forward over the resident history each time."""
    w = synth.Workload("tier-cache: Hq8/Hkv2 S512 hist20 K3", 1, 8, 2, 128, 128, 512, 20, 3, "bf16", 44,
                       structured_keys=True)
    x = synth.draw(w)
    D = dims_of(w)
    dev = {n: to_dev(getattr(x, n)) for n in ("q", "k_seg", "v_seg", "k_hist", "v_hist")}
    st = AttentionStep(D)
    st.select(dev["q"], dev["k_hist"])
    rng = np.random.default_rng(5)
    idx2 = np.sort(np.stack([rng.choice(w.nblk, w.topk, replace=False) for _ in range(2 * 4)]), axis=1)
    idx2 = torch.from_numpy(idx2.astype(np.int32).reshape(1, 2, 4, w.topk)).cuda()
    refs = []
    for idx in (st.idx, idx2):
        o, lse = torch.empty_like(st.o), torch.empty_like(st.lse)
        hga_attn_fwd(D, dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], w.nblk, idx, o, lse)
        refs.append((o, lse))
    cap = w.nblk
    tier_k = _pinned(x.k_hist)
    tier_v = _pinned(x.v_hist)
    scratch = torch.empty(tuple(st.idx.shape), dtype=torch.int32).pin_memory()
    sets = [set(i.cpu().numpy().ravel().tolist()) - {-1} for i in (st.idx, idx2)]
    slots = max(len(sets[0]), len(sets[1]))
    cache = BlockCache(cap, slots)
    pool_k = torch.full((1, slots * 128, 2, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    pool_v = torch.full_like(pool_k, float("nan"))
    ip = torch.empty_like(st.idx)
    cs = torch.cuda.Stream()
    done = torch.cuda.Event()
    done.record(cs)

    def run(idx):
        nu, nf = hga_fetch_blocks_cached(D, tier_k, tier_v, idx, scratch, pool_k, pool_v, cache, ip,
                                         torch.cuda.current_stream(), cs, done)
        torch.cuda.current_stream().wait_event(done)
        o, lse = torch.empty_like(st.o), torch.empty_like(st.lse)
        hga_attn_fwd(D, dev["q"], dev["k_seg"], dev["v_seg"], pool_k, pool_v, slots, ip, o, lse)
        torch.cuda.synchronize()
        hga_device_status()
        return nu, nf, o, lse

    nu, nf, o, lse = run(st.idx)
    assert nu == nf == len(sets[0])
    assert torch.equal(o, refs[0][0]) and torch.equal(lse, refs[0][1])
    _oracle_check("first fetch", w, x, st.idx.cpu().numpy(), o, lse)
    nu, nf, o, lse = run(st.idx)
    assert nu == len(sets[0]) and nf == 0
    assert torch.equal(o, refs[0][0]) and torch.equal(lse, refs[0][1])
    resident = set(int(b) for b in cache.block_of_slot if b >= 0)
    nu, nf, o, lse = run(idx2)
    assert nu == len(sets[1]) and nf == len(sets[1] - resident)
    _oracle_check("after evictions", w, x, idx2.cpu().numpy(), o, lse)
    # slots are no longer in block order, so the forward visits the history
    # tiles in another order: equal up to fp32 summation order
    assert (o.float() - refs[1][0].float()).abs().max().item() <= 2e-2
    assert (lse - refs[1][1]).abs().max().item() <= 1e-4
    # every resident block sits where the cache says
    for slot, blk in enumerate(cache.block_of_slot.tolist()):
        if blk >= 0:
            assert torch.equal(pool_k[:, slot * 128:(slot + 1) * 128].cpu(), tier_k[:, blk * 128:(blk + 1) * 128])


def test_cache_segment_makes_new_blocks_resident():
    """hga_cache_segment puts a segment's blocks into the device cache (with
    hga_offload_segment they exist in both tiers); selecting them afterwards
    copies nothing over the host link, and the pool holds exactly their K/V."""
    w = synth.Workload("t", 1, 4, 2, 128, 128, 256, 3, 2, "bf16", 45)
    x = synth.draw(w)
    D = dims_of(w)
    ks, vs = to_dev(x.k_seg), to_dev(x.v_seg)
    cap, slots = 8, 4
    tk = torch.zeros((1, cap * 128, 2, 128), dtype=torch.bfloat16).pin_memory()
    tv = torch.zeros_like(tk).pin_memory()
    cache = BlockCache(cap, slots)
    pool_k = torch.zeros((1, slots * 128, 2, 128), dtype=torch.bfloat16, device="cuda")
    pool_v = torch.zeros_like(pool_k)
    hga_offload_segment(D, ks, vs, tk, tv, cap, 5)
    hga_cache_segment(D, ks, vs, pool_k, pool_v, cache, 5)
    torch.cuda.synchronize()
    assert cache.slot_of_block[5:7].tolist() == [0, 1]
    assert torch.equal(pool_k[:, :256], ks) and torch.equal(pool_v[:, :256], vs)
    Dh = D.with_history(7)
    idx = torch.full((1, 2, 2, 2), -1, dtype=torch.int32, device="cuda")
    idx[..., 0], idx[..., 1] = 5, 6
    scratch = torch.empty((1, 2, 2, 2), dtype=torch.int32).pin_memory()
    ip = torch.empty_like(idx)
    cs = torch.cuda.Stream()
    done = torch.cuda.Event()
    done.record(cs)
    nu, nf = hga_fetch_blocks_cached(Dh, tk, tv, idx, scratch, pool_k, pool_v, cache, ip,
                                     torch.cuda.current_stream(), cs, done)
    torch.cuda.synchronize()
    assert (nu, nf) == (2, 0)
    assert ip.cpu().unique().tolist() == [0, 1]
    with pytest.raises(HgaError):
        hga_cache_segment(D, ks, vs, pool_k, pool_v, cache, 7)  # blocks 7, 8 outside the capacity of 8


def test_remap_idx_on_device():
    """hga_remap_idx: idx -> slots through a device copy of the slot map, -1
    kept; a selected block that is not resident is flagged, never read."""
    w = synth.Workload("t", 1, 4, 2, 128, 128, 256, 6, 3, "bf16", 46)
    D = dims_of(w)
    slot_of = torch.tensor([4, 0, 5, 1, 3, 2], dtype=torch.int32, device="cuda")
    idx = torch.tensor([[0, 2, -1], [1, 3, 5], [4, -1, -1], [0, 1, 2]], dtype=torch.int32,
                       device="cuda").reshape(1, 2, 2, 3)
    ip = torch.empty_like(idx)
    hga_remap_idx(D, idx, slot_of, ip)
    hga_device_status()
    want = torch.where(idx >= 0, slot_of[idx.clamp(min=0).long()], torch.full_like(idx, -1))
    assert torch.equal(ip, want)
    slot_of[3] = -1  # block 3 not resident
    hga_remap_idx(D, idx, slot_of, ip)
    with pytest.raises(HgaError) as e:
        hga_device_status()
    assert e.value.status == 4
    assert ip[0, 0, 1, 1].item() == -1


@pytest.mark.parametrize("with_cache,with_tier", [(True, True), (False, True), (True, False), (False, False)])
def test_append_segment_one_pass(with_cache, with_tier):
    """hga_append_segment: the summaries of a finished segment's blocks (against
    the oracle), its K/V in the device cache slots that the cache plan gives
    them (byte-equal), and its K/V in the host tier (byte-equal), from one
    pass over the segment; the rest of every buffer untouched."""
    from segmented_fine_tuning_b200 import hga_append_segment
    w = synth.Workload("append: B2 Hq4/Hkv2 S512", 2, 4, 2, 128, 128, 512, 0, 2, "bf16", 47)
    x = synth.draw(w)
    ks, vs = to_dev(x.k_seg), to_dev(x.v_seg)
    cap, at = 10, 5
    D = dims_of(w, nblk=cap)
    summ = torch.full((2, cap, 2, 128), 7.0, device="cuda")
    cache = BlockCache(cap, 6) if with_cache else None
    if with_cache:
        cache.plan(np.array([0, 1, 2], dtype=np.int32))  # slots 0..2 in use: the new blocks take 3..5
    pool_k = torch.zeros((2, 6 * 128, 2, 128), dtype=torch.bfloat16, device="cuda")
    pool_v = torch.zeros_like(pool_k)
    tk = torch.zeros((2, cap * 128, 2, 128), dtype=torch.bfloat16).pin_memory() if with_tier else None
    tv = torch.zeros_like(tk).pin_memory() if with_tier else None
    cs = torch.cuda.Stream()
    hga_append_segment(D, ks, vs, at, summ, pool_k, pool_v, cache, tk, tv, cap if with_tier else 0, None, cs)
    torch.cuda.synchronize()
    hga_device_status()
    ref = oracle.block_summaries(oracle.Dims(2, 4, 2, 128, 128, 512, 4, 2), x.k_seg.f64)  # [B, Hkv, 4, d]
    got = summ.cpu().numpy().transpose(0, 2, 1, 3)
    assert np.abs(got[:, :, at:at + 4] - ref).max() <= 1e-6 * max(1.0, np.abs(ref).max())
    assert np.all(got[:, :, :at] == 7.0) and np.all(got[:, :, at + 4:] == 7.0)
    if with_cache:
        slots = cache.slot_of_block[at:at + 4].tolist()
        # empty slots 3, 4, 5 first, then the least recently used one (slot 0, block 0 evicted)
        assert slots == [3, 4, 5, 0] and cache.slot_of_block[0] == -1
        for t, sl in enumerate(slots):
            assert torch.equal(pool_k[:, sl * 128:(sl + 1) * 128], ks[:, t * 128:(t + 1) * 128])
            assert torch.equal(pool_v[:, sl * 128:(sl + 1) * 128], vs[:, t * 128:(t + 1) * 128])
        assert cache.block_of_slot[slots].tolist() == list(range(at, at + 4))
    else:
        assert torch.count_nonzero(pool_k) == 0 and torch.count_nonzero(pool_v) == 0
    if with_tier:
        assert torch.equal(tk[:, at * 128:(at + 4) * 128], ks.cpu()) and torch.equal(tv[:, at * 128:(at + 4) * 128],
                                                                                   vs.cpu())
        assert torch.count_nonzero(tk[:, :at * 128]) == 0 and torch.count_nonzero(tk[:, (at + 4) * 128:]) == 0


def test_gather_mapped_matches_fetch_and_oracle():
    """hga_gather_blocks_mapped: the GPU reads the selected blocks from the
    mapped pinned tier itself (no host wait).  Same pool and slot map as
    hga_fetch_blocks, byte for byte; attention over the pool matches the
    oracle; a pool too small for the selection is flagged, its unplaced
    entries are -1; a tier that is not pinned is rejected before launch."""
    from segmented_fine_tuning_b200 import hga_gather_blocks_mapped
    w = synth.Workload("gather: B2 Hq8/Hkv2 S512 hist20 K3", 2, 8, 2, 128, 128, 512, 20, 3, "bf16", 48,
                       structured_keys=True)
    x = synth.draw(w)
    D = dims_of(w)
    dev = {n: to_dev(getattr(x, n)) for n in ("q", "k_seg", "v_seg", "k_hist", "v_hist", "d_o")}
    st = AttentionStep(D)
    st.select(dev["q"], dev["k_hist"])
    cap = w.nblk + 2
    tier_k = torch.zeros((2, cap * 128, 2, 128), dtype=torch.bfloat16).pin_memory()
    tier_v = torch.zeros_like(tier_k).pin_memory()
    tier_k[:, : w.nblk * 128] = _pinned(x.k_hist)
    tier_v[:, : w.nblk * 128] = _pinned(x.v_hist)
    n_sel = len(set(st.idx.cpu().numpy().ravel().tolist()) - {-1})
    slots = n_sel + 1
    pools = {}
    for how in ("fetch", "mapped"):
        pk = torch.full((2, slots * 128, 2, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        pv = torch.full_like(pk, float("nan"))
        ip = torch.full_like(st.idx, -7)
        if how == "fetch":
            cs = torch.cuda.Stream()
            done = torch.cuda.Event()
            done.record(cs)
            scratch = torch.empty(tuple(st.idx.shape), dtype=torch.int32).pin_memory()
            hga_fetch_blocks(D, tier_k, tier_v, cap, st.idx, scratch, pk, pv, slots, ip,
                             torch.cuda.current_stream(), cs, done)
            torch.cuda.current_stream().wait_event(done)
        else:
            hga_gather_blocks_mapped(D, tier_k, tier_v, cap, st.idx, pk, pv, slots, ip)
        torch.cuda.synchronize()
        hga_device_status()
        pools[how] = (pk, pv, ip)
    fk, fv, fi = pools["fetch"]
    mk, mv, mi = pools["mapped"]
    assert torch.equal(fi, mi)
    # slots 0..n_sel-1 hold the same blocks; the spare slot stays untouched
    assert torch.equal(fk[:, : n_sel * 128].cpu(), mk[:, : n_sel * 128].cpu())
    assert torch.equal(fv[:, : n_sel * 128].cpu(), mv[:, : n_sel * 128].cpu())
    assert torch.isnan(mk[:, n_sel * 128:].float()).all()
    o, lse = torch.empty_like(st.o), torch.empty_like(st.lse)
    hga_attn_fwd(D, dev["q"], dev["k_seg"], dev["v_seg"], mk, mv, slots, mi, o, lse)
    dq, dk, dv = torch.empty_like(st.dq), torch.empty_like(st.dk), torch.empty_like(st.dv)
    hga_attn_bwd(D, dev["q"], dev["k_seg"], dev["v_seg"], mk, mv, slots, mi, o, lse, dev["d_o"], dq, dk, dv, st.ws)
    torch.cuda.synchronize()
    hga_device_status()
    _oracle_check("mapped gather", w, x, st.idx.cpu().numpy(), o, lse, dq, dk, dv)
    # too few slots: the last two selected blocks get none
    small = n_sel - 2
    pk = torch.zeros((2, small * 128, 2, 128), dtype=torch.bfloat16, device="cuda")
    pv = torch.zeros_like(pk)
    ip = torch.empty_like(st.idx)
    hga_gather_blocks_mapped(D, tier_k, tier_v, cap, st.idx, pk, pv, small, ip)
    with pytest.raises(HgaError) as e:
        hga_device_status()
    assert e.value.status == 4
    ig, ipn = st.idx.cpu().numpy(), ip.cpu().numpy()
    sel = sorted(set(ig.ravel().tolist()) - {-1})
    assert np.all(ipn[np.isin(ig, sel[small:])] == -1)
    assert np.array_equal(ipn[np.isin(ig, sel[:small])], fi.cpu().numpy()[np.isin(ig, sel[:small])])
    # pageable (not pinned) host memory is refused before any launch
    import ctypes
    from segmented_fine_tuning_b200 import _binding
    pageable = np.zeros(tier_k.numel(), dtype=np.uint16)
    lib = _binding.load_library()
    status = lib.hga_gather_blocks_mapped(ctypes.byref(D.c()), pageable.ctypes.data, pageable.ctypes.data, cap,
                                          st.idx.data_ptr(), pk.data_ptr(), pv.data_ptr(), small, ip.data_ptr(),
                                          None)
    assert status == 1, lib.hga_last_error()
