"""Pins for the fp64 oracle: each check compares the oracle with something other
than itself (closed forms, hand-worked fixtures, brute force, torch's float64
attention and autograd, finite differences), chosen so that a dropped term, a
wrong sign or index, or a transposed operand fails at least one of them."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import Dims

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _rand_inputs(D: Dims, seed, hist_blocks=None):
    r = _rng(seed)
    nb = D.nblk if hist_blocks is None else hist_blocks
    q = r.standard_normal((D.B, D.S, D.Hq, D.d))
    ks = r.standard_normal((D.B, D.S, D.Hkv, D.d))
    vs = r.standard_normal((D.B, D.S, D.Hkv, D.d))
    kh = r.standard_normal((D.B, nb * D.blk, D.Hkv, D.d))
    vh = r.standard_normal((D.B, nb * D.blk, D.Hkv, D.d))
    do = r.standard_normal((D.B, D.S, D.Hq, D.d))
    return q, ks, vs, kh, vh, do


# ---------------------------------------------------------------- summaries

def test_summaries_constant_per_block():
    """Keys = c_block + (+e, -e pairs): the mean is c_block exactly."""
    D = Dims(B=2, Hq=4, Hkv=2, d=8, blk=4, S=4, nblk=5, topk=2)
    r = _rng(1)
    c = r.integers(-8, 8, size=(D.B, D.nblk, D.Hkv, D.d)).astype(np.float64)
    e = r.integers(-4, 4, size=(D.B, D.nblk, 2, D.Hkv, D.d)).astype(np.float64) * 0.25
    noise = np.concatenate([e, -e], axis=2)  # 4 tokens per block summing to zero
    k = (c[:, :, None] + noise).reshape(D.B, D.nblk * D.blk, D.Hkv, D.d)
    summ = oracle.block_summaries(D, k)
    np.testing.assert_array_equal(summ, c.transpose(0, 2, 1, 3))


def test_query_means_constant_per_block():
    D = Dims(B=1, Hq=3, Hkv=1, d=4, blk=2, S=6, nblk=1, topk=1)
    r = _rng(2)
    c = r.integers(-5, 5, size=(D.B, D.nqb, D.Hq, D.d)).astype(np.float64)
    e = r.integers(-3, 3, size=(D.B, D.nqb, 1, D.Hq, D.d)).astype(np.float64)
    q = (c[:, :, None] + np.concatenate([e, -e], axis=2)).reshape(D.B, D.S, D.Hq, D.d)
    np.testing.assert_array_equal(oracle.query_means(D, q), c.transpose(0, 2, 1, 3))


# ---------------------------------------------------------------- selection

def test_select_hand_gqa_golden():
    g = json.load(open(os.path.join(GOLDEN, "hand_select_gqa.json")))
    dm = g["dims"]
    kh = np.array(g["k_hist"], dtype=np.float64).reshape(1, dm["nblk"] * dm["blk"], 1, dm["d"])
    q = np.array(g["q"], dtype=np.float64).reshape(1, dm["S"], dm["Hq"], dm["d"])
    for k_str, want in g["expect"]["idx_by_topk"].items():
        D = Dims(B=1, Hq=dm["Hq"], Hkv=1, d=dm["d"], blk=dm["blk"], S=dm["S"], nblk=dm["nblk"], topk=int(k_str))
        idx, score = oracle.select(D, q, kh)
        np.testing.assert_array_equal(score.reshape(-1), g["expect"]["score"])
        assert idx.reshape(-1).tolist() == want


def _brute_topk(scores, K):
    """Among all K-subsets: the largest score sum; ties -> lexicographically
    smallest sorted index tuple (== lower block index wins a tie)."""
    n = len(scores)
    keff = min(K, n)
    best = None
    for sub in itertools.combinations(range(n), keff):
        key = (-sum(scores[i] for i in sub), sub)
        if best is None or key < best:
            best = key
    return list(best[1]) + [-1] * (K - keff)


@pytest.mark.parametrize("seed", range(6))
def test_topk_bruteforce(seed):
    r = _rng(100 + seed)
    nblk = int(r.integers(1, 9))
    for K in (1, 2, 3, 4, 9):
        D = Dims(B=1, Hq=1, Hkv=1, d=4, blk=1, S=3, nblk=nblk, topk=K)
        # small integers: many exact ties, exact sums
        score = r.integers(-3, 4, size=(1, 1, D.nqb, nblk)).astype(np.float64)
        idx = oracle.select_topk(D, score)
        for i in range(D.nqb):
            assert idx[0, 0, i].tolist() == _brute_topk(score[0, 0, i].tolist(), K)


def test_topk_matches_stable_lexsort():
    D = Dims(B=2, Hq=2, Hkv=2, d=4, blk=1, S=5, nblk=300, topk=17)
    r = _rng(7)
    score = np.round(r.standard_normal((D.B, D.Hkv, D.nqb, D.nblk)), 1)  # rounded: ties
    score[0, 0, 0, :50] = -0.0
    score[0, 0, 0, 50:100] = 0.0
    idx = oracle.select_topk(D, score)
    for b, h, i in itertools.product(range(D.B), range(D.Hkv), range(D.nqb)):
        s = score[b, h, i]
        order = np.lexsort((np.arange(D.nblk), -s))  # primary: score desc, then index asc
        assert idx[b, h, i].tolist() == sorted(order[: D.topk].tolist())


def test_select_q_zero_picks_first_blocks():
    """Q = 0: every score is exactly 0, so the tie rule alone picks 0..K-1."""
    D = Dims(B=1, Hq=4, Hkv=2, d=8, blk=4, S=8, nblk=10, topk=3)
    q, _, _, kh, _, _ = _rand_inputs(D, 3)
    idx, score = oracle.select(D, np.zeros_like(q), kh)
    assert np.all(score == 0)
    assert np.all(idx == np.arange(3))


def test_select_fewer_blocks_than_k():
    D = Dims(B=1, Hq=2, Hkv=1, d=4, blk=2, S=4, nblk=3, topk=5)
    q, _, _, kh, _, _ = _rand_inputs(D, 4)
    idx, _ = oracle.select(D, q, kh)
    assert np.all(idx[..., :3] == np.arange(3)) and np.all(idx[..., 3:] == -1)


def test_scores_max_over_group_not_mean():
    """Scores equal the max over the group's heads of the per-head score
    computed with numpy's dot (a library routine)."""
    D = Dims(B=1, Hq=6, Hkv=2, d=8, blk=4, S=8, nblk=6, topk=2)
    q, _, _, kh, _, _ = _rand_inputs(D, 5)
    summ = oracle.block_summaries(D, kh)
    qm = oracle.query_means(D, q)
    sc = oracle.block_scores(D, qm, summ)
    G = D.Hq // D.Hkv
    for h in range(D.Hkv):
        per_head = np.stack([qm[0, h * G + g] @ summ[0, h].T for g in range(G)]) / math.sqrt(D.d)
        np.testing.assert_allclose(sc[0, h], per_head.max(axis=0), rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- forward

def _eval(expr, sym):
    return eval(expr, {"exp": math.exp, "log": math.log}, sym)


def _load_hand():
    g = json.load(open(os.path.join(GOLDEN, "hand_d4.json")))
    dm = g["dims"]
    D = Dims(**dm)
    sh_q = (1, dm["S"], 1, dm["d"])
    kh = np.array(g["k_hist"], float).reshape(1, 4, 1, 4)
    vh = np.array(g["v_hist"], float).reshape(1, 4, 1, 4)
    q = np.array(g["q"], float).reshape(sh_q)
    ks = np.array(g["k_seg"], float).reshape(sh_q)
    vs = np.array(g["v_seg"], float).reshape(sh_q)
    do = np.array(g["d_o"], float).reshape(sh_q)
    sym = {}
    for k, v in g["symbols"].items():
        sym[k] = _eval(v, sym)
    return g, D, q, ks, vs, kh, vh, do, sym


def test_hand_d4_forward_and_selection():
    g, D, q, ks, vs, kh, vh, do, sym = _load_hand()
    summ = oracle.block_summaries(D, kh)
    np.testing.assert_array_equal(summ.reshape(2, 4), g["expect"]["summ"])
    idx, score = oracle.select(D, q, kh)
    np.testing.assert_array_equal(score.reshape(-1), g["expect"]["score"])
    assert idx.reshape(-1).tolist() == g["expect"]["idx"]
    o, lse = oracle.attn_fwd(D, q, ks, vs, kh, vh, idx)
    want_o = np.array([[_eval(e, sym) for e in row] for row in g["expect"]["o"]])
    want_lse = np.array([_eval(e, sym) for e in g["expect"]["lse"]])
    np.testing.assert_allclose(o.reshape(2, 4), want_o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse.reshape(-1), want_lse, rtol=0, atol=1e-14)


def test_hand_d4_backward():
    g, D, q, ks, vs, kh, vh, do, sym = _load_hand()
    idx = np.array([[[[1]]]], dtype=np.int32)
    dq, dk, dv = oracle.attn_bwd(D, q, ks, vs, kh, vh, idx, do)
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        want = np.array([[_eval(e, sym) for e in row] for row in g["expect"][name]])
        np.testing.assert_allclose(got.reshape(2, 4), want, rtol=0, atol=1e-14, err_msg=name)


def _sdpa_dense(q_full, k_full, v_full):
    """torch float64 scaled-dot-product attention, causal, GQA by repeating KV."""
    G = q_full.shape[2] // k_full.shape[2]
    qt = q_full.permute(0, 2, 1, 3)
    kt = k_full.repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    vt = v_full.repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    return out.permute(0, 2, 1, 3)


@pytest.mark.parametrize("blk,nblk,S,G", [(4, 3, 8, 2), (8, 5, 16, 4), (2, 1, 6, 1)])
def test_all_blocks_selected_equals_dense_causal(blk, nblk, S, G):
    """K = every history block: HGA over the segment == dense causal attention
    over history + segment (torch float64 SDPA), on the segment rows."""
    Hkv = 2
    D = Dims(B=2, Hq=Hkv * G, Hkv=Hkv, d=8, blk=blk, S=S, nblk=nblk, topk=nblk)
    q, ks, vs, kh, vh, _ = _rand_inputs(D, 11)
    idx, _ = oracle.select(D, q, kh)
    assert np.all(idx == np.arange(nblk))
    o, lse = oracle.attn_fwd(D, q, ks, vs, kh, vh, idx)
    H = nblk * blk
    r = _rng(12)
    q_hist = r.standard_normal((D.B, H, D.Hq, D.d))  # history-row queries: irrelevant to segment rows
    qf = torch.from_numpy(np.concatenate([q_hist, q], axis=1))
    kf = torch.from_numpy(np.concatenate([kh, ks], axis=1))
    vf = torch.from_numpy(np.concatenate([vh, vs], axis=1))
    dense = _sdpa_dense(qf, kf, vf).numpy()[:, H:]
    np.testing.assert_allclose(o, dense, rtol=0, atol=1e-12)
    # the oracle's own textbook dense path agrees too, including LSE
    o2, lse2 = oracle.dense_causal_fwd(qf.numpy(), kf.numpy(), vf.numpy())
    np.testing.assert_allclose(o2[:, H:], dense, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse2[:, :, H:], rtol=0, atol=1e-12)
    # LSE against torch's logsumexp of the dense causal logits
    G_ = D.Hq // D.Hkv
    logits = torch.einsum("bthd,bshd->bhts", qf, kf.repeat_interleave(G_, dim=2)) / math.sqrt(D.d)
    T = H + S
    mask = torch.ones(T, T, dtype=torch.bool).tril()
    ref_lse = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=-1).numpy()[:, :, H:]
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_q_zero_gives_uniform_average():
    """Q = 0: all logits 0, so O is the plain mean of V over the key set and
    LSE = log(#keys)."""
    D = Dims(B=1, Hq=2, Hkv=1, d=4, blk=2, S=6, nblk=4, topk=2)
    q, ks, vs, kh, vh, _ = _rand_inputs(D, 13)
    idx = np.array([1, 3, 0, 2, 3, -1], dtype=np.int32)[None, None].reshape(1, 1, 3, 2)
    idx = np.sort(np.where(idx < 0, 99, idx), axis=-1)
    idx = np.where(idx == 99, -1, idx).astype(np.int32)
    o, lse = oracle.attn_fwd(D, np.zeros_like(q), ks, vs, kh, vh, idx)
    for hq in range(D.Hq):
        for p in range(D.S):
            blocks = [n for n in idx[0, 0, p // D.blk] if n >= 0]
            vals = [vh[0, n * D.blk + t, 0] for n in blocks for t in range(D.blk)] + [vs[0, t, 0] for t in range(p + 1)]
            np.testing.assert_allclose(o[0, p, hq], np.mean(vals, axis=0), rtol=0, atol=1e-14)
            assert abs(lse[0, hq, p] - math.log(len(vals))) < 1e-14


def test_value_ones_give_ones():
    """Softmax rows sum to one: with V = 1 every output is 1."""
    D = Dims(B=1, Hq=4, Hkv=2, d=8, blk=4, S=12, nblk=5, topk=3)
    q, ks, _, kh, _, _ = _rand_inputs(D, 14)
    idx, _ = oracle.select(D, q, kh)
    o, _ = oracle.attn_fwd(D, 3 * q, ks, np.ones_like(ks), kh, np.ones_like(kh), idx)
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-13)


def test_segment_first_row_single_key():
    """A one-token segment with no history: O = V."""
    D = Dims(B=1, Hq=2, Hkv=1, d=4, blk=1, S=1, nblk=0, topk=1)
    q, ks, vs, kh, vh, _ = _rand_inputs(D, 15)
    o, lse = oracle.attn_fwd(D, q, ks, vs, kh, vh, -np.ones((1, 1, 1, 1), np.int32))
    np.testing.assert_array_equal(o[0, 0, 0], vs[0, 0, 0])
    np.testing.assert_array_equal(o[0, 0, 1], vs[0, 0, 0])


def test_kv_head_subset_is_exact_restriction():
    D = Dims(B=1, Hq=4, Hkv=2, d=8, blk=4, S=8, nblk=4, topk=2)
    q, ks, vs, kh, vh, do = _rand_inputs(D, 16)
    idx, _ = oracle.select(D, q, kh)
    o, lse = oracle.attn_fwd(D, q, ks, vs, kh, vh, idx)
    o1, lse1 = oracle.attn_fwd(D, q, ks, vs, kh, vh, idx, kv_heads=range(1, 2))
    np.testing.assert_array_equal(o1[:, :, 2:], o[:, :, 2:])
    assert np.all(np.isnan(o1[:, :, :2]))
    o2, lse2 = oracle.attn_fwd(D, q, ks, vs, kh, vh, idx, rows=[0, 5, 7])
    np.testing.assert_array_equal(o2[:, [0, 5, 7]], o[:, [0, 5, 7]])
    np.testing.assert_array_equal(lse2[:, :, [0, 5, 7]], lse[:, :, [0, 5, 7]])
    assert np.all(np.isnan(o2[:, [1, 2, 3, 4, 6]]))
    g = oracle.attn_bwd(D, q, ks, vs, kh, vh, idx, do)
    g1 = oracle.attn_bwd(D, q, ks, vs, kh, vh, idx, do, kv_heads=range(1, 2))
    np.testing.assert_array_equal(g1[0][:, :, 2:], g[0][:, :, 2:])
    np.testing.assert_array_equal(g1[1][:, :, 1:], g[1][:, :, 1:])
    np.testing.assert_array_equal(g1[2][:, :, 1:], g[2][:, :, 1:])


# ---------------------------------------------------------------- backward

def test_backward_finite_differences():
    """Central differences of L = <O, dO> with the selection held fixed."""
    D = Dims(B=1, Hq=4, Hkv=2, d=4, blk=2, S=4, nblk=3, topk=2)
    q, ks, vs, kh, vh, do = _rand_inputs(D, 17)
    idx, _ = oracle.select(D, q, kh)
    dq, dk, dv = oracle.attn_bwd(D, q, ks, vs, kh, vh, idx, do)

    def loss(q_, ks_, vs_):
        o, _ = oracle.attn_fwd(D, q_, ks_, vs_, kh, vh, idx)
        return float(np.sum(o * do))

    h = 1e-5
    for name, x, g in (("q", q, dq), ("k_seg", ks, dk), ("v_seg", vs, dv)):
        fd = np.zeros_like(x)
        for ix in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[ix] += h
            xm[ix] -= h
            args_p = {"q": (xp, ks, vs), "k_seg": (q, xp, vs), "v_seg": (q, ks, xp)}[name]
            args_m = {"q": (xm, ks, vs), "k_seg": (q, xm, vs), "v_seg": (q, ks, xm)}[name]
            fd[ix] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.abs(fd - g).max() / max(np.abs(g).max(), 1e-12)
        assert err < 1e-6, (name, err)


@pytest.mark.parametrize("G", [1, 2, 4])
def test_backward_all_blocks_equals_dense_autograd(G):
    """K = every history block, dO = 0 on history rows: the segment gradients
    equal torch autograd through float64 dense causal attention (history
    K/V are detached there too)."""
    Hkv = 2
    D = Dims(B=1, Hq=Hkv * G, Hkv=Hkv, d=8, blk=4, S=12, nblk=3, topk=3)
    q, ks, vs, kh, vh, do = _rand_inputs(D, 18 + G)
    idx, _ = oracle.select(D, q, kh)
    dq, dk, dv = oracle.attn_bwd(D, q, ks, vs, kh, vh, idx, do)
    H = D.nblk * D.blk
    qt = torch.from_numpy(q).requires_grad_()
    kst = torch.from_numpy(ks).requires_grad_()
    vst = torch.from_numpy(vs).requires_grad_()
    q_hist = torch.zeros((D.B, H, D.Hq, D.d), dtype=torch.float64)
    out = _sdpa_dense(torch.cat([q_hist, qt], 1), torch.cat([torch.from_numpy(kh), kst], 1),
                      torch.cat([torch.from_numpy(vh), vst], 1))
    (out[:, H:] * torch.from_numpy(do)).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, kst.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, vst.grad.numpy(), rtol=0, atol=1e-12)


def test_backward_partial_selection_autograd():
    """K < #blocks: autograd through a float64 gather-then-softmax written with
    torch ops (keys assembled from the oracle's selection) matches."""
    D = Dims(B=1, Hq=4, Hkv=2, d=8, blk=4, S=8, nblk=5, topk=2)
    q, ks, vs, kh, vh, do = _rand_inputs(D, 30)
    idx, _ = oracle.select(D, q, kh)
    dq, dk, dv = oracle.attn_bwd(D, q, ks, vs, kh, vh, idx, do)
    qt = torch.from_numpy(q).requires_grad_()
    kst = torch.from_numpy(ks).requires_grad_()
    vst = torch.from_numpy(vs).requires_grad_()
    khT, vhT = torch.from_numpy(kh), torch.from_numpy(vh)
    G = D.Hq // D.Hkv
    total = 0
    for hq in range(D.Hq):
        h = hq // G
        for p in range(D.S):
            blocks = [int(n) for n in idx[0, h, p // D.blk] if n >= 0]
            rows = [n * D.blk + t for n in blocks for t in range(D.blk)]
            keys = torch.cat([khT[0, rows, h], kst[0, : p + 1, h]], 0)
            vals = torch.cat([vhT[0, rows, h], vst[0, : p + 1, h]], 0)
            w = torch.softmax(keys @ qt[0, p, hq] / math.sqrt(D.d), 0)
            total = total + (w @ vals * torch.from_numpy(do[0, p, hq])).sum()
    total.backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, kst.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, vst.grad.numpy(), rtol=0, atol=1e-12)


def test_near_tie_flag():
    D = Dims(B=1, Hq=1, Hkv=1, d=4, blk=1, S=2, nblk=4, topk=2)
    score = np.array([[[[3.0, 2.0, 1.9999, 0.0], [3.0, 2.0, 1.0, 0.0]]]])
    flags = oracle.near_tie_positions(D, score)
    assert flags.tolist() == [[[True, False]]]


# ---------------------------------------------------------------- decode step

def _summ_oracle_layout(D: Dims, kh):
    return oracle.block_summaries(D, kh)


@pytest.mark.parametrize("i", [0, 2, 3])
def test_decode_whole_block_equals_prefill_block(i):
    """nq = block new queries starting at a block boundary form a whole query
    block: decode selection and attention equal the prefill oracle's for that
    block (itself pinned by the tests above)."""
    D = Dims(B=2, Hq=6, Hkv=2, d=8, blk=4, S=16, nblk=7, topk=3)
    q, ks, vs, kh, vh, _ = _rand_inputs(D, 71 + i)
    summ = oracle.block_summaries(D, kh)
    idx_p, score_p = oracle.select(D, q, kh)
    o_p, lse_p = oracle.attn_fwd(D, q, ks, vs, kh, vh, idx_p)
    rows = slice(i * D.blk, (i + 1) * D.blk)
    idx_d, score_d = oracle.decode_select(D, q[:, rows], summ)
    np.testing.assert_array_equal(idx_d, idx_p[:, :, i])
    np.testing.assert_allclose(score_d, score_p[:, :, i], rtol=0, atol=1e-14)
    o_d, lse_d = oracle.decode_attn(D, i * D.blk, q[:, rows], ks, vs, kh, vh, idx_d)
    np.testing.assert_allclose(o_d, o_p[:, rows], rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse_d, lse_p[:, :, rows], rtol=0, atol=1e-13)


@pytest.mark.parametrize("nq,t0", [(1, 0), (1, 9), (3, 5), (5, 2)])
def test_decode_bruteforce(nq, t0):
    """Straight numpy restatement on a tiny case: mean of the new queries,
    group-max scores, the best K-subset by enumeration, and a softmax over
    the explicit key list of every new row."""
    D = Dims(B=1, Hq=4, Hkv=2, d=4, blk=2, S=12, nblk=6, topk=2)
    r = _rng(80 + nq + t0)
    qn = r.standard_normal((1, nq, D.Hq, D.d))
    ks = r.standard_normal((1, D.S, D.Hkv, D.d))
    vs = r.standard_normal((1, D.S, D.Hkv, D.d))
    kh = r.standard_normal((1, D.nblk * D.blk, D.Hkv, D.d))
    vh = r.standard_normal((1, D.nblk * D.blk, D.Hkv, D.d))
    summ = oracle.block_summaries(D, kh)
    idx, score = oracle.decode_select(D, qn, summ)
    G = D.Hq // D.Hkv
    o, lse = oracle.decode_attn(D, t0, qn, ks, vs, kh, vh, idx)
    for h in range(D.Hkv):
        sm = kh[0, :, h].reshape(D.nblk, D.blk, D.d).mean(axis=1)
        qm = qn[0, :, h * G:(h + 1) * G].mean(axis=0)                  # [G, d]
        want = (qm @ sm.T).max(axis=0) / math.sqrt(D.d)
        np.testing.assert_allclose(score[0, h], want, rtol=0, atol=1e-13)
        assert idx[0, h].tolist() == list(_brute_topk(want.tolist(), D.topk))
        for g in range(G):
            hq = h * G + g
            for u in range(nq):
                keys = [kh[0, n * D.blk + t, h] for n in idx[0, h] for t in range(D.blk)]
                vals = [vh[0, n * D.blk + t, h] for n in idx[0, h] for t in range(D.blk)]
                keys += [ks[0, t, h] for t in range(t0 + u + 1)]
                vals += [vs[0, t, h] for t in range(t0 + u + 1)]
                s = np.array([qn[0, u, hq] @ k for k in keys]) / math.sqrt(D.d)
                p = np.exp(s - s.max())
                np.testing.assert_allclose(o[0, u, hq], (p / p.sum()) @ np.array(vals), rtol=0, atol=1e-13)
                assert abs(lse[0, hq, u] - (s.max() + math.log(p.sum()))) < 1e-13


def test_decode_q_zero_and_short_history():
    """Q = 0: every score is 0, so blocks 0..K-1 are chosen (padding -1 when the
    history is shorter than K) and each row is the plain mean of its values,
    LSE = log(number of keys)."""
    D = Dims(B=1, Hq=2, Hkv=1, d=4, blk=2, S=8, nblk=3, topk=5)
    r = _rng(90)
    qn = np.zeros((1, 2, 2, 4))
    ks, vs = r.standard_normal((1, 8, 1, 4)), r.standard_normal((1, 8, 1, 4))
    kh, vh = r.standard_normal((1, 6, 1, 4)), r.standard_normal((1, 6, 1, 4))
    idx, score = oracle.decode_select(D, qn, oracle.block_summaries(D, kh))
    assert idx.reshape(-1).tolist() == [0, 1, 2, -1, -1]
    np.testing.assert_array_equal(score, 0.0)
    t0 = 3
    o, lse = oracle.decode_attn(D, t0, qn, ks, vs, kh, vh, idx)
    for u in range(2):
        vals = np.concatenate([vh[0, :, 0], vs[0, : t0 + u + 1, 0]])
        for hq in range(2):
            np.testing.assert_allclose(o[0, u, hq], vals.mean(axis=0), rtol=0, atol=1e-14)
            assert abs(lse[0, hq, u] - math.log(len(vals))) < 1e-14


# ---------------------------------------------------------------- sparse backward

def test_sparse_backward_all_blocks_scale_one_is_the_backward():
    D = Dims(B=2, Hq=4, Hkv=2, d=8, blk=4, S=12, nblk=5, topk=2)
    q, ks, vs, kh, vh, do = _rand_inputs(D, 101)
    idx, _ = oracle.select(D, q, kh)
    ref = oracle.attn_bwd(D, q, ks, vs, kh, vh, idx, do)
    got = oracle.attn_bwd_sparse(D, q, ks, vs, kh, vh, idx, do, np.ones((2, 3), dtype=np.int8), 1.0)
    for a, b in zip(got, ref):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-14)


def test_sparse_backward_matches_autograd_of_the_masked_loss():
    """torch float64 autograd of L = c * sum over the chosen query blocks of
    <O, dO>, with O from a dense masked softmax over the selected history
    blocks and the causal segment (written out in torch, not the oracle)."""
    D = Dims(B=1, Hq=4, Hkv=2, d=8, blk=4, S=16, nblk=6, topk=2)
    q, ks, vs, kh, vh, do = _rand_inputs(D, 102)
    idx, _ = oracle.select(D, q, kh)
    mask = np.array([[1, 0, 0, 1]], dtype=np.int8)
    c = 2.0
    got = oracle.attn_bwd_sparse(D, q, ks, vs, kh, vh, idx, do, mask, c)
    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(ks, requires_grad=True)
    tv = torch.tensor(vs, requires_grad=True)
    G = D.Hq // D.Hkv
    T = D.nblk * D.blk
    keys = torch.cat([torch.tensor(kh), tk], dim=1)       # [1, T+S, Hkv, d]
    vals = torch.cat([torch.tensor(vh), tv], dim=1)
    loss = 0
    for hq in range(D.Hq):
        h = hq // G
        for p in range(D.S):
            i = p // D.blk
            if not mask[0, i]:
                continue
            cols = [n * D.blk + t for n in idx[0, h, i] if n >= 0 for t in range(D.blk)] + list(range(T, T + p + 1))
            s = keys[0, cols, h] @ tq[0, p, hq] / math.sqrt(D.d)
            o = torch.softmax(s, 0) @ vals[0, cols, h]
            loss = loss + c * (o * torch.tensor(do[0, p, hq])).sum()
    loss.backward()
    np.testing.assert_allclose(got[0], tq.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[1], tk.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[2], tv.grad.numpy(), rtol=0, atol=1e-12)
    # rows of unchosen blocks get exactly zero dQ
    assert np.all(got[0][:, 4:12] == 0.0)


def test_sparse_backward_ignores_unchosen_rows_of_d_o():
    D = Dims(B=1, Hq=2, Hkv=1, d=4, blk=2, S=8, nblk=3, topk=2)
    q, ks, vs, kh, vh, do = _rand_inputs(D, 103)
    idx, _ = oracle.select(D, q, kh)
    mask = np.array([[0, 1, 0, 1]], dtype=np.int8)
    a = oracle.attn_bwd_sparse(D, q, ks, vs, kh, vh, idx, do, mask, 0.5)
    do2 = do.copy()
    do2[:, 0:2] = 1e3
    do2[:, 4:6] = -7.0
    b = oracle.attn_bwd_sparse(D, q, ks, vs, kh, vh, idx, do2, mask, 0.5)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


# ---------------------------------------------------------------- query blocks of another size than history blocks

def test_query_means_over_query_blocks_of_two_history_blocks():
    """qblk = 2*blk: a query block's mean is the average of the means of its
    two halves (computed with qblk = blk), exactly for integer inputs."""
    D2 = Dims(B=2, Hq=3, Hkv=1, d=4, blk=2, S=12, nblk=1, topk=1, qblk=4)
    D1 = Dims(B=2, Hq=3, Hkv=1, d=4, blk=2, S=12, nblk=1, topk=1)
    q = _rng(31).integers(-8, 8, size=(D2.B, D2.S, D2.Hq, D2.d)).astype(np.float64)
    qm2, qm1 = oracle.query_means(D2, q), oracle.query_means(D1, q)
    assert qm2.shape[2] == 3 and qm1.shape[2] == 6
    np.testing.assert_array_equal(qm2, 0.5 * (qm1[:, :, 0::2] + qm1[:, :, 1::2]))


def test_scores_over_query_blocks_of_two_history_blocks_g1():
    """G = 1, qblk = 2*blk: the score is linear in the query mean, so a query
    block's scores are the average of its halves' scores."""
    D2 = Dims(B=1, Hq=2, Hkv=2, d=8, blk=4, S=16, nblk=5, topk=2, qblk=8)
    D1 = Dims(B=1, Hq=2, Hkv=2, d=8, blk=4, S=16, nblk=5, topk=2)
    q, _, _, kh, _, _ = _rand_inputs(D2, 32)
    _, s2 = oracle.select(D2, q, kh)
    _, s1 = oracle.select(D1, q, kh)
    np.testing.assert_allclose(s2, 0.5 * (s1[:, :, 0::2] + s1[:, :, 1::2]), rtol=0, atol=1e-13)


@pytest.mark.parametrize("blk,qblk", [(2, 4), (4, 2), (3, 6)])
def test_query_zero_k1_closed_form_with_other_query_block_size(blk, qblk):
    """Q = 0, K = 1, history block n holding the value n+1, segment values 0:
    row p attends to the blk tokens of the block chosen for query block
    p // qblk and to the p+1 segment keys, all with equal weight, so
    O[p] = blk * (n + 1) / (blk + p + 1).  A row mapped to the wrong query
    block, or a block of the wrong length, fails it."""
    nblk, S = 5, 12
    D = Dims(B=1, Hq=2, Hkv=1, d=3, blk=blk, S=S, nblk=nblk, topk=1, qblk=qblk)
    nqb = S // qblk
    chosen = (np.arange(nqb) * 2 + 1) % nblk  # a different block for neighbouring query blocks
    idx = chosen.astype(np.int32).reshape(1, 1, nqb, 1)
    vh = np.repeat((np.arange(nblk, dtype=np.float64) + 1.0), blk)[None, :, None, None] * np.ones((1, 1, 1, D.d))
    kh = _rng(33).standard_normal((1, nblk * blk, 1, D.d))
    ks = _rng(34).standard_normal((1, S, 1, D.d))
    o, lse = oracle.attn_fwd(D, np.zeros((1, S, D.Hq, D.d)), ks, np.zeros_like(ks), kh, vh, idx)
    for p in range(S):
        n = chosen[p // qblk]
        want = blk * (n + 1.0) / (blk + p + 1.0)
        np.testing.assert_allclose(o[0, p], want, rtol=0, atol=1e-14)
        assert abs(lse[0, 0, p] - math.log(blk + p + 1.0)) < 1e-14


def test_all_blocks_selected_equals_dense_with_other_query_block_size():
    """K = every history block makes the query-block size irrelevant: HGA
    equals dense causal attention over history + segment for qblk != blk."""
    Hkv, G, blk, nblk, S = 2, 2, 4, 3, 16
    D = Dims(B=1, Hq=Hkv * G, Hkv=Hkv, d=8, blk=blk, S=S, nblk=nblk, topk=nblk, qblk=8)
    q, ks, vs, kh, vh, _ = _rand_inputs(D, 35)
    idx, _ = oracle.select(D, q, kh)
    assert idx.shape == (1, Hkv, 2, nblk) and np.all(idx == np.arange(nblk))
    o, lse = oracle.attn_fwd(D, q, ks, vs, kh, vh, idx)
    H = nblk * blk
    qf = np.concatenate([_rng(36).standard_normal((1, H, D.Hq, D.d)), q], axis=1)
    o2, lse2 = oracle.dense_causal_fwd(qf, np.concatenate([kh, ks], axis=1), np.concatenate([vh, vs], axis=1))
    np.testing.assert_allclose(o, o2[:, H:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse2[:, :, H:], rtol=0, atol=1e-12)


def test_sparse_backward_mask_counts_query_blocks_of_qblk_rows():
    """qmask has one entry per query block of qblk rows: with only query block
    1 chosen, dQ is zero outside rows [qblk, 2*qblk) and non-zero inside."""
    D = Dims(B=1, Hq=2, Hkv=1, d=4, blk=2, S=12, nblk=4, topk=2, qblk=4)
    q, ks, vs, kh, vh, do = _rand_inputs(D, 37)
    idx, _ = oracle.select(D, q, kh)
    mask = np.zeros((1, D.nqb), np.int8)
    mask[0, 1] = 1
    dq, dk, dv = oracle.attn_bwd_sparse(D, q, ks, vs, kh, vh, idx, do, mask, 1.0)
    rows = np.abs(dq[0]).sum(axis=(1, 2))
    assert np.all(rows[:4] == 0) and np.all(rows[8:] == 0) and np.all(rows[4:8] > 0)
    # keys after the chosen rows get no gradient
    assert np.all(dk[0, 8:] == 0) and np.all(dv[0, 8:] == 0)
