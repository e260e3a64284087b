"""The full segmented pass over a long sequence, driven through the C ABI.

Article: "Low-VRAM Long-Context Fine-Tuning: Hierarchical Global Attention and
Segmented Backpropagation in Practice", Background: the sequence is processed
one segment at a time; only the active segment is differentiable and kept on
the GPU; the KV of earlier segments lives in system RAM; each query block
loads only its bounded set of history blocks.  Deep analysis: the per-block
summaries stay resident on the GPU.  fr edition, Analyse approfondie: a
finished segment's KV is offloaded right away.

Per segment s (history = segments 0..s-1, 16 blocks each at 2,048 tokens):
  forward,  layers 0..L-1:  select (resident summaries) -> fetch the distinct
                            selected blocks that are not already in the
                            layer's device pool from its pinned host tier (a
                            block cache: slots are reused least recently used
                            first) -> attention forward
  backward, layers L-1..0:  attention backward on the same pool (kept from the
                            forward; no second fetch)
  after the forward, every layer: the segment's K/V (final once the layer's
                            forward has run) copied to the host tier on a
                            side stream, so the copies cross the host link
                            during the backward, when it carries nothing else
  segment end, every layer: one pass over the segment's K/V
                            (hga_append_segment): summaries of its blocks
                            appended to the resident array and the blocks
                            copied into the layer's device cache
Every step is a libhga.so call; this module owns buffers, streams and order.
Batch size 1 (one sequence): the resident summary array of a layer grows as a
prefix, which is a valid summary array of the current history for B = 1.
"""
from __future__ import annotations

import torch

from ._binding import (BlockCache, Dims, hga_append_segment, hga_attn_bwd, hga_attn_bwd_workspace_size,
                       hga_attn_fwd, hga_fetch_blocks_cached, hga_offload_segment, hga_remap_idx, hga_select_topk)


class SegmentedPass:
    def __init__(self, seg: Dims, n_layers: int, n_segments: int, device="cuda", fetch_timeout_ms: int = 10000,
                 pool_slots: int | None = None, keep_new_blocks: bool = True, prefetch: bool = True):
        """pool_slots: device pool (cache) size per layer in blocks; by default
        the largest history, so no block is fetched twice in one sequence.
        keep_new_blocks: a finished segment's blocks also enter the layer's
        device cache (a device-to-device copy) as they are offloaded, so their
        first selection needs no host transfer.
        prefetch: the selection and fetch of layer l+1 are queued while the
        forward of layer l runs (selection on a high-priority side stream,
        block copies on the copy stream), so host-link transfers and the
        host's wait for the selected indices overlap attention compute."""
        self.keep_new_blocks = keep_new_blocks
        self.prefetch = prefetch
        if seg.B != 1:
            raise ValueError("the segmented pass drives one sequence (B = 1)")
        self.seg, self.L, self.NS = seg, n_layers, n_segments
        self.nqb = seg.S // seg.block
        self.cap = n_segments * self.nqb            # host-tier / summary capacity, blocks
        self.max_hist = (n_segments - 1) * self.nqb  # largest history, blocks
        self.device = torch.device(device)
        self.timeout = fetch_timeout_ms
        dt = seg.torch_dtype
        H, d, blk = seg.Hkv, seg.d, seg.block
        pool_blocks = max(1, self.max_hist if pool_slots is None else pool_slots)
        self.pool_slots = pool_blocks
        self.tier_k, self.tier_v, self.summ, self.pool_k, self.pool_v = [], [], [], [], []
        self.idx, self.idx_pool, self.scratch, self.o, self.lse, self.done = [], [], [], [], [], []
        self.cache, self.slot_dev = [], []
        for _ in range(n_layers):
            self.tier_k.append(torch.empty((1, self.cap * blk, H, d), dtype=dt).pin_memory())
            self.tier_v.append(torch.empty((1, self.cap * blk, H, d), dtype=dt).pin_memory())
            self.summ.append(torch.zeros((1, self.cap, H, d), dtype=torch.float32, device=self.device))
            self.pool_k.append(torch.empty((1, pool_blocks * blk, H, d), dtype=dt, device=self.device))
            self.pool_v.append(torch.empty((1, pool_blocks * blk, H, d), dtype=dt, device=self.device))
            self.idx.append(torch.empty((1, H, self.nqb, seg.topk), dtype=torch.int32, device=self.device))
            self.idx_pool.append(torch.empty((1, H, self.nqb, seg.topk), dtype=torch.int32, device=self.device))
            self.scratch.append(torch.empty((1, H, self.nqb, seg.topk), dtype=torch.int32).pin_memory())
            self.o.append(torch.empty((1, seg.S, seg.Hq, d), dtype=dt, device=self.device))
            self.lse.append(torch.empty((1, seg.Hq, seg.S), dtype=torch.float32, device=self.device))
            ev = torch.cuda.Event()
            self.done.append(ev)
            self.cache.append(BlockCache(self.cap, pool_blocks))
            self.slot_dev.append(torch.full((self.cap,), -1, dtype=torch.int32, device=self.device))
        self.dq = torch.empty((1, seg.S, seg.Hq, d), dtype=torch.float32, device=self.device)
        self.dk = torch.empty((1, seg.S, H, d), dtype=torch.float32, device=self.device)
        self.dv = torch.empty((1, seg.S, H, d), dtype=torch.float32, device=self.device)
        self.ws = torch.empty((max(256, hga_attn_bwd_workspace_size(seg)),), dtype=torch.uint8, device=self.device)
        # host -> device block copies and device -> host segment offloads on
        # separate streams, so the two directions of the host link overlap
        self.copy_stream = torch.cuda.Stream(self.device)
        self.offload_stream = torch.cuda.Stream(self.device)
        self.sel_stream = torch.cuda.Stream(self.device, priority=-1)
        self.slots_stale = [False] * n_layers  # slot_dev[l] lags the host cache state
        self.ready = [torch.cuda.Event() for _ in range(n_layers)]
        self.offloaded = [torch.cuda.Event() for _ in range(n_layers)]
        for ev in self.done:
            ev.record(self.copy_stream)  # materialise the handles
        self.fetched_blocks = []   # blocks copied over the host link per (layer, segment) step
        self.selected_blocks = []  # distinct blocks selected, per step that went through the host
        self.device_remaps = 0     # steps whose whole history was resident: idx remapped on the device

    def new_sequence(self) -> None:
        """Start another sequence: its history tier replaces the previous one,
        so nothing resident in the pools is valid any more."""
        for c, d in zip(self.cache, self.slot_dev):
            c.reset()
            d.fill_(-1)
        self.slots_stale = [False] * self.L

    def dims(self, s: int) -> Dims:
        return self.seg.with_history(s * self.nqb)

    def n_kv(self, s: int) -> int:
        return self.pool_slots if s > 0 else 0

    # ------------------------------------------------------------ steps
    def stage(self, s: int, l: int, q, stream) -> list[torch.cuda.Event]:
        """Selection of (segment s, layer l) and the history it needs in the
        layer's pool: queued on `stream` (the block copies on the copy
        stream).  Returns the events the forward must wait for: the end of
        the selection on `stream`, and the end of the copies on the copy
        stream when blocks crossed the host link.  `stream` itself never
        waits for the copies, so the selection of the next layer (and with
        it the host's plan of the next copies) runs while they are in
        flight, and the copy stream goes from one layer's blocks to the
        next without a gap."""
        D = self.dims(s)
        hga_select_topk(D, q, self.summ[l], self.idx[l], None, stream)
        waits = []
        if s > 0:
            if (self.cache[l].slot_of_block[: s * self.nqb] >= 0).all():
                # every selectable block is resident: slots on the device, no host round trip
                if self.slots_stale[l]:
                    self._sync_slots(l, stream)
                hga_remap_idx(D, self.idx[l], self.slot_dev[l], self.idx_pool[l], stream)
                self.fetched_blocks.append(0)
                self.device_remaps += 1
            else:
                # the tier's newest blocks come from this layer's last offload
                self.copy_stream.wait_event(self.offloaded[l])
                nu, nf = hga_fetch_blocks_cached(D, self.tier_k[l], self.tier_v[l], self.idx[l], self.scratch[l],
                                                 self.pool_k[l], self.pool_v[l], self.cache[l], self.idx_pool[l],
                                                 stream, self.copy_stream, self.done[l], self.timeout)
                self.selected_blocks.append(nu)
                self.fetched_blocks.append(nf)
                self.slots_stale[l] = True
                waits.append(self.done[l])
        self.ready[l].record(stream)
        return [self.ready[l]] + waits

    def forward(self, s: int, l: int, q, k_seg, v_seg, ready: list[torch.cuda.Event] | None = None):
        """Attention forward of (segment s, layer l); stages the selection
        and fetch first unless `ready` (the events stage() returned) says
        they are already queued."""
        D = self.dims(s)
        st = torch.cuda.current_stream(self.device)
        if ready is None:
            ready = self.stage(s, l, q, st)
        for ev in ready:
            st.wait_event(ev)
        if s > 0:
            hga_attn_fwd(D, q, k_seg, v_seg, self.pool_k[l], self.pool_v[l], self.pool_slots, self.idx_pool[l],
                         self.o[l], self.lse[l], st)
        else:
            hga_attn_fwd(D, q, k_seg, v_seg, None, None, 0, self.idx[l], self.o[l], self.lse[l], st)
        return self.o[l], self.lse[l]

    def backward(self, s: int, l: int, q, k_seg, v_seg, d_o):
        D = self.dims(s)
        st = torch.cuda.current_stream(self.device)
        if s > 0:
            hga_attn_bwd(D, q, k_seg, v_seg, self.pool_k[l], self.pool_v[l], self.pool_slots, self.idx_pool[l],
                         self.o[l], self.lse[l], d_o, self.dq, self.dk, self.dv, self.ws, st)
        else:
            hga_attn_bwd(D, q, k_seg, v_seg, None, None, 0, self.idx[l], self.o[l], self.lse[l], d_o, self.dq,
                         self.dk, self.dv, self.ws, st)
        return self.dq, self.dk, self.dv

    def offload(self, s: int, l: int, k_seg, v_seg):
        """Copy the segment's K/V of layer l to the host tier on the offload
        stream, ordered after the work queued so far (they are final once the
        layer's forward has been queued)."""
        st = torch.cuda.current_stream(self.device)
        self.offload_stream.wait_stream(st)
        hga_offload_segment(self.seg, k_seg, v_seg, self.tier_k[l], self.tier_v[l], self.cap, s * self.nqb,
                            self.offload_stream)
        self.offloaded[l].record(self.offload_stream)
        # the caller may release k_seg/v_seg once the offload stream has passed here
        k_seg.record_stream(self.offload_stream)
        v_seg.record_stream(self.offload_stream)

    def end_segment(self, s: int, l: int, k_seg, v_seg, offloaded: bool = False):
        """Append the segment's blocks in one pass over its K and V: summaries
        on the device, the blocks into the layer's device cache (unless
        keep_new_blocks is off), and -- unless `offloaded` says offload() has
        queued it already -- K/V to the host tier on the side stream (ordered
        after the work queued so far)."""
        st = torch.cuda.current_stream(self.device)
        cache = self.cache[l] if (self.keep_new_blocks and s + 1 < self.NS) else None
        tier = (None, None) if offloaded else (self.tier_k[l], self.tier_v[l])
        hga_append_segment(self.seg.with_history(self.cap), k_seg, v_seg, s * self.nqb, self.summ[l],
                           self.pool_k[l], self.pool_v[l], cache, tier[0], tier[1], self.cap, st,
                           self.offload_stream)
        if not offloaded:
            self.offloaded[l].record(self.offload_stream)
            k_seg.record_stream(self.offload_stream)
            v_seg.record_stream(self.offload_stream)
        if cache is not None:
            self.slots_stale[l] = True

    def _sync_slots(self, l: int, st) -> None:
        """Device copy of layer l's slot map, queued on st (a fresh pinned
        staging buffer each time, so a pending copy is never overwritten).
        Done only when a device remap is about to read it, so steps that
        take the host path queue no extra transfer behind their block
        copies."""
        staged = torch.from_numpy(self.cache[l].slot_of_block[: self.cap].copy()).pin_memory()
        with torch.cuda.stream(st):
            self.slot_dev[l].copy_(staged, non_blocking=True)
        self.slots_stale[l] = False

    def run_segment(self, s: int, inputs, on_step=None):
        """inputs[l] = (q, k_seg, v_seg, d_o) device tensors of layer l for
        segment s.  on_step(s, l, phase) is called after each layer's forward
        ("fwd") and backward ("bwd") calls are queued."""
        st = torch.cuda.current_stream(self.device)
        ahead = self.prefetch and s > 0
        if ahead:
            # the side stream starts after everything queued so far (earlier
            # readers of the pools), then runs one layer ahead of the forward
            self.sel_stream.wait_stream(st)
            ready = self.stage(s, 0, inputs[0][0], self.sel_stream)
        for l in range(self.L):
            self.forward(s, l, *inputs[l][:3], ready=ready if ahead else None)
            if ahead and l + 1 < self.L:
                ready = self.stage(s, l + 1, inputs[l + 1][0], self.sel_stream)
            if on_step:
                on_step(s, l, "fwd")
        # every layer's K/V is final: the tier copies run during the backward
        for l in range(self.L):
            self.offload(s, l, inputs[l][1], inputs[l][2])
        for l in reversed(range(self.L)):
            q, k, v, do = inputs[l]
            self.backward(s, l, q, k, v, do)
            if on_step:
                on_step(s, l, "bwd")
        for l in range(self.L):
            self.end_segment(s, l, inputs[l][1], inputs[l][2], offloaded=True)
