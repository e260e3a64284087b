"""Seeded synthetic inputs for the HGA attention step.

This module is shared by the oracle-side tests and the GPU side (tests and
benchmark).  It holds none of the method's arithmetic: it only draws random
numbers, rounds them to the storage type, and slices a sequence into history
and segment.

Recipe (one generator per workload, numpy ``PCG64(seed)``, float64 normals,
drawn in this order):
  1. Q   [B, S, Hq, d]            ~ N(0, 1)
  2. if the keys are block-structured:
       m  [B, T/blk, Hkv, d]      ~ N(0, 1)   one mean vector per 128-token block
       (if a fraction of dominant blocks is asked for) a permutation of the
       history blocks; the first round(frac * nblk) of them get scale 2
     K = 0.5 * scale_block * m_block + eps,  eps [B, T, Hkv, d] ~ N(0, 1)
     else K [B, T, Hkv, d] ~ N(0, 1)
  3. V   [B, T, Hkv, d]            ~ N(0, 1)
  4. dO  [B, S, Hq, d]            ~ N(0, 1)
T = nblk*blk + S tokens; history is tokens [0, nblk*blk), the active segment
the last S.  Values are then rounded to the storage dtype: float32 (round to
nearest even), or bfloat16 by float64 -> float32 -> bfloat16, each step round
to nearest even.  Both sides consume exactly these rounded values (the oracle
widens them to float64).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    blk: int
    S: int
    nblk: int
    topk: int
    dtype: str  # "f32" or "bf16"
    seed: int
    structured_keys: bool = False
    dominant_frac: float = 0.0
    fwd_only: bool = False
    qblk: int = 0  # query-block size; 0 = blk

    @property
    def T(self) -> int:
        return self.nblk * self.blk + self.S

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def qb(self) -> int:
        return self.qblk or self.blk

    @property
    def nqb(self) -> int:
        return self.S // self.qb


# The five workloads of the HGA attention step.
TINY_F32 = Workload("tiny-fp32: B1 Hq2/Hkv1 d64, hist 16x64, S256, K4", 1, 2, 1, 64, 64, 256, 16, 4, "f32", 0)
QWEN3_8B_LAYER = Workload("qwen3-8b-layer: B1 Hq32/Hkv8 d128, hist 112x128, S2048, K16", 1, 32, 8, 128, 128, 2048, 112,
                          16, "bf16", 2, structured_keys=True)
DENSE_EQUIV = Workload("dense-equivalence: B1 Hq32/Hkv8 d128, hist 12x128, S512, K12=all", 1, 32, 8, 128, 128, 512,
                       12, 12, "bf16", 3)
PREFILL_131K = Workload("prefill-131k: B1 Hq32/Hkv8 d128, hist 992x128, S4096, K32, fwd only", 1, 32, 8, 128, 128,
                        4096, 992, 32, "bf16", 4, structured_keys=True, dominant_frac=0.01, fwd_only=True)
# The layer with history blocks of 64 tokens under 128-row query blocks: the same history keys per query
# block (32 x 64 = 16 x 128) and the same history length (224 x 64 = 112 x 128).
QWEN3_8B_LAYER64 = Workload("qwen3-8b-layer-blk64: B1 Hq32/Hkv8 d128, hist 224x64, S2048, q_block 128, K32", 1, 32,
                            8, 128, 64, 2048, 224, 32, "bf16", 6, structured_keys=True, qblk=128)
# The same with 32-token history blocks: K = 64 (the largest K) keeps 64 x 32 = 16 x 128 history keys per
# query block over 448 x 32 = 112 x 128 history tokens.
QWEN3_8B_LAYER32 = Workload("qwen3-8b-layer-blk32: B1 Hq32/Hkv8 d128, hist 448x32, S2048, q_block 128, K64", 1, 32,
                            8, 128, 32, 2048, 448, 64, "bf16", 9, structured_keys=True, qblk=128)

WORKLOADS = {"tiny_f32": TINY_F32, "qwen3_8b_layer": QWEN3_8B_LAYER, "dense_equiv": DENSE_EQUIV,
             "prefill_131k": PREFILL_131K}

# Full segmented pass: 36 layers of the Qwen3-8B-shaped layer over 8 segments of
# 2,048 tokens; segment s of layer l is drawn from its own generator.
SEGMENTED_LAYERS = 36
SEGMENTED_SEGMENTS = 8


def segmented_seed(layer: int, segment: int) -> int:
    return 1_000_003 * layer + segment + 5


def round_f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even.
    Inputs are finite by construction, so the 32-bit sum cannot overflow
    (the largest finite pattern is 0xFF7FFFFF)."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    r = (u >> 16) & 1
    r += 0x7FFF
    r += u
    r >>= 16
    return r.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@dataclass
class Tensor:
    """One input tensor in its storage form plus the exact float64 values."""
    store: np.ndarray  # float32 or uint16 (bf16 bits)
    dtype: str

    @property
    def f64(self) -> np.ndarray:
        if self.dtype == "bf16":
            return bf16_bits_to_f64(self.store)
        return self.store.astype(np.float64)

    @property
    def shape(self):
        return self.store.shape


def _store(x: np.ndarray, dtype: str) -> Tensor:
    x32 = round_f32(x)
    if dtype == "bf16":
        return Tensor(f32_to_bf16_bits(x32), "bf16")
    return Tensor(x32, "f32")


@dataclass
class Inputs:
    w: Workload
    q: Tensor
    k_hist: Tensor
    v_hist: Tensor
    k_seg: Tensor
    v_seg: Tensor
    d_o: Tensor
    extra: dict = field(default_factory=dict)


def draw(w: Workload, seed: int | None = None, nblk: int | None = None) -> Inputs:
    """Draw one workload's inputs.  ``nblk`` overrides the history length
    (used by the segmented pass, whose history grows)."""
    seed = w.seed if seed is None else seed
    nblk = w.nblk if nblk is None else nblk
    rng = np.random.Generator(np.random.PCG64(seed))
    B, S, Hq, Hkv, d, blk = w.B, w.S, w.Hq, w.Hkv, w.d, w.blk
    T = nblk * blk + S
    q = rng.standard_normal((B, S, Hq, d))
    if w.structured_keys:
        nb_tot = T // blk
        means = rng.standard_normal((B, nb_tot, Hkv, d))
        scale = np.ones(nb_tot)
        if w.dominant_frac > 0 and nblk > 0:
            perm = rng.permutation(nblk)
            scale[perm[: int(round(w.dominant_frac * nblk))]] = 2.0
        eps = rng.standard_normal((B, T, Hkv, d))
        k = 0.5 * np.repeat(scale[None, :, None, None] * means, blk, axis=1) + eps
    else:
        k = rng.standard_normal((B, T, Hkv, d))
    v = rng.standard_normal((B, T, Hkv, d))
    d_o = rng.standard_normal((B, S, Hq, d))
    H = nblk * blk
    return Inputs(w, _store(q, w.dtype), _store(k[:, :H], w.dtype), _store(v[:, :H], w.dtype),
                  _store(k[:, H:], w.dtype), _store(v[:, H:], w.dtype), _store(d_o, w.dtype))


# Decode step at 131K context: the prefill's history (992 blocks) and a full
# 4,096-token segment buffer, one new token at the last position.
DECODE_131K = Workload("decode-131k: B1 Hq32/Hkv8 d128, hist 992x128, segment buffer 4096, K32, 1 new token", 1, 32,
                       8, 128, 128, 4096, 992, 32, "bf16", 8, structured_keys=True, dominant_frac=0.01,
                       fwd_only=True)


def draw_decode(w: Workload, nq: int, t0: int, seed: int | None = None) -> Inputs:
    """Inputs of a decode step: the workload's draw, whose segment tensors
    serve as the segment KV buffer (capacity w.S); the new queries are the
    segment's query rows t0 .. t0+nq-1 (in ``extra["q_new"]``)."""
    x = draw(w, seed=seed)
    x.extra["q_new"] = Tensor(np.ascontiguousarray(x.q.store[:, t0:t0 + nq]), x.q.dtype)
    return x


def draw_segment(w: Workload, layer: int, segment: int) -> Inputs:
    """Active-segment tensors of (layer, segment) for the segmented pass.  The
    history of that step is the concatenation of the earlier segments' K/V of
    the same layer, so only the segment part of the draw is used."""
    return draw(w, seed=segmented_seed(layer, segment), nblk=0)
