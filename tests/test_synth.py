"""The seeded input generator: determinism, rounding, and the recipe's structure."""
import numpy as np
import torch

import synth


def test_bf16_rounding_matches_torch_rne():
    r = np.random.Generator(np.random.PCG64(0))
    x = np.concatenate([r.standard_normal(100000), r.standard_normal(1000) * 1e-30, r.standard_normal(1000) * 1e30])
    x32 = synth.round_f32(x)
    ours = synth.f32_to_bf16_bits(x32)
    theirs = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, theirs)
    back = synth.bf16_bits_to_f64(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(x32).to(torch.bfloat16).double().numpy())


def test_draw_is_deterministic_and_sliced():
    w = synth.DENSE_EQUIV
    a = synth.draw(w)
    b = synth.draw(w)
    for n in ("q", "k_hist", "v_hist", "k_seg", "v_seg", "d_o"):
        np.testing.assert_array_equal(getattr(a, n).store, getattr(b, n).store)
    assert a.q.shape == (1, 512, 32, 128)
    assert a.k_hist.shape == (1, 12 * 128, 8, 128)
    assert a.k_seg.shape == (1, 512, 8, 128)
    assert a.q.store.dtype == np.uint16


def test_structured_keys_have_block_means():
    w = synth.Workload("t", 1, 4, 2, 64, 16, 32, 20, 4, "f32", 9, structured_keys=True, dominant_frac=0.1)
    x = synth.draw(w)
    k = x.k_hist.f64.reshape(1, 20, 16, 2, 64)
    # block means of the keys are ~0.5*m (or 1.0*m for the 2 dominant blocks)
    norms = np.linalg.norm(k.mean(axis=2), axis=-1)[0]  # [20, 2]
    assert (norms > 5.0).sum() >= 2 * 2 - 1  # dominant blocks stand out in both heads
    assert np.median(norms) > 2.0  # 0.5*sqrt(64)=4 vs noise sqrt(64/16)=2


def test_tiny_f32_is_float32():
    x = synth.draw(synth.TINY_F32)
    assert x.q.store.dtype == np.float32 and x.q.shape == (1, 256, 2, 64)
    assert x.k_hist.shape == (1, 1024, 1, 64)
