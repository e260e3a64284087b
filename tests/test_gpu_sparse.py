"""SpaCO-style sparse segment backward (hga_attn_bwd_sparse) against the
fp64 oracle's attn_bwd_sparse, through the C ABI.

Only the chosen query blocks propagate gradient, every gradient is scaled by
the correction factor.  The gradient is linear in that factor, so the stated
bf16 tolerance (max abs 2e-2, relative L2 1e-2 vs the oracle) is applied to
the gradient divided by it; fp32 keeps max abs 1e-4 the same way.  dQ rows of
unchosen blocks must be exactly zero.  Cases: the tensor-core path (small,
and the full Qwen3-8B-shaped layer with 4 of 16 blocks chosen), and the
CUDA-core path (fp32, d = 64).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from hga_testutil import BF16_ABS, BF16_REL, F32_ABS, assert_close, dims_of, to_dev, to_host
from segmented_fine_tuning_b200 import (hga_attn_bwd_sparse, hga_attn_bwd_workspace_size, hga_device_status,
                                        spaco_sample_blocks)
from segmented_fine_tuning_b200.step import AttentionStep

pytestmark = pytest.mark.gpu

CASES = [
    (synth.Workload("sparse-tc: Hq8/Hkv2 S512 hist6 K3", 1, 8, 2, 128, 128, 512, 6, 3, "bf16", 111,
                    structured_keys=True), 2),
    (synth.Workload("sparse-tc-B2: B2 Hq4/Hkv2 S384 hist4 K2", 2, 4, 2, 128, 128, 384, 4, 2, "bf16", 112), 1),
    (synth.QWEN3_8B_LAYER, 4),
    (synth.TINY_F32, 2),
    (synth.Workload("sparse-qblk64-blk128: Hq4/Hkv2 S384 hist4 K2", 1, 4, 2, 128, 128, 384, 4, 2, "bf16", 113,
                    qblk=64), 2),
    (synth.Workload("sparse-tc-blk64: Hq4/Hkv2 S512 hist11 K5", 1, 4, 2, 128, 64, 512, 11, 5, "bf16", 114,
                    qblk=128), 2),
    (synth.Workload("sparse-tc-blk16: Hq4/Hkv2 S512 hist30 K13", 1, 4, 2, 128, 16, 512, 30, 13, "bf16", 115,
                    qblk=128), 2),
]


@pytest.mark.parametrize("w,k", CASES, ids=lambda c: c.name.split(":")[0] if hasattr(c, "name") else str(c))
def test_sparse_backward_matches_oracle(w, k):
    x = synth.draw(w)
    D = dims_of(w)
    dev = {n: to_dev(getattr(x, n)) for n in ("q", "k_seg", "v_seg", "k_hist", "v_hist", "d_o")}
    st = AttentionStep(D)
    st.select(dev["q"], dev["k_hist"])
    st.forward(dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"])
    g = torch.Generator().manual_seed(w.seed)
    mask, scale = spaco_sample_blocks(w.B, w.nqb, k, g, cap=8.0)
    dq = torch.full_like(dev["q"], float("nan"), dtype=torch.float32)
    dk = torch.full_like(dev["k_seg"], float("nan"), dtype=torch.float32)
    dv = torch.full_like(dev["v_seg"], float("nan"), dtype=torch.float32)
    hga_attn_bwd_sparse(D, dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], w.nblk, st.idx,
                        st.o, st.lse, dev["d_o"], mask.cuda(), scale, dq, dk, dv, st.ws)
    torch.cuda.synchronize()
    hga_device_status()
    od = oracle.Dims(w.B, w.Hq, w.Hkv, w.d, w.blk, w.S, w.nblk, w.topk, w.qblk)
    idx = st.idx.cpu().numpy()
    ref = oracle.attn_bwd_sparse(od, x.q.f64, x.k_seg.f64, x.v_seg.f64, x.k_hist.f64, x.v_hist.f64, idx, x.d_o.f64,
                                 mask.numpy().astype(np.int8), scale)
    tol = (F32_ABS, None) if w.dtype == "f32" else (BF16_ABS, BF16_REL)
    for name, got, want in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref):
        assert_close(f"sparse {name} / scale", to_host(got) / scale, want / scale, *tol)
    # unchosen query blocks: exactly zero dQ
    dqh = dq.cpu().numpy()
    for b in range(w.B):
        for i in range(w.nqb):
            if not mask[b, i]:
                assert np.all(dqh[b, i * w.qb:(i + 1) * w.qb] == 0.0)
    print(f"{w.name}: {k} of {w.nqb} query blocks, scale {scale}")


def test_sparse_backward_all_blocks_equals_backward():
    """Every block chosen with scale 1: the plain backward's result."""
    w = CASES[0][0]
    x = synth.draw(w)
    D = dims_of(w)
    dev = {n: to_dev(getattr(x, n)) for n in ("q", "k_seg", "v_seg", "k_hist", "v_hist", "d_o")}
    st = AttentionStep(D)
    st.run(dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], dev["d_o"])
    dq, dk, dv = torch.empty_like(st.dq), torch.empty_like(st.dk), torch.empty_like(st.dv)
    mask = torch.ones((w.B, w.nqb), dtype=torch.uint8, device="cuda")
    ws = torch.empty((hga_attn_bwd_workspace_size(D),), dtype=torch.uint8, device="cuda")
    hga_attn_bwd_sparse(D, dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], w.nblk, st.idx, st.o,
                        st.lse, dev["d_o"], mask, 1.0, dq, dk, dv, ws)
    torch.cuda.synchronize()
    hga_device_status()
    assert torch.equal(dq, st.dq)
    assert torch.allclose(dk, st.dk, rtol=0, atol=1e-5) and torch.allclose(dv, st.dv, rtol=0, atol=1e-5)
