"""Pins of the oracle's key-key proxy score and token selection.

* the window mean and the scores against a long-double numpy restatement;
* the kept-token count rule and the pages' "60% eviction -> 2.5x fewer
  tokens" (NexusQuant, "Token eviction"; dev.to, step 2 and the summary);
* BOS and the recent window are always kept (same passages);
* the kept set equals a numpy lexsort top-k with ties to the lower position.
"""
import numpy as np
import pytest
import torch

from e8_lattice_vector_nq_b200 import synth


def test_kept_count_rule(oq):
    assert oq.kept_count(32768, 64, 60) == 13147
    assert 32768 / 13147 == pytest.approx(2.49, abs=0.01)  # "about 2.5x fewer tokens"
    assert oq.kept_count(65536, 128, 35) == 42644
    assert oq.kept_count(100, 99, 50) == 100  # T <= 1 + W: keep all
    assert oq.kept_count(100, 10, 0) == 100
    assert oq.kept_count(100, 10, 100) == 11  # only BOS + window
    for T, W, p in [(1000, 64, 60), (777, 5, 33), (66, 64, 99)]:
        mid = T - 1 - W
        assert oq.kept_count(T, W, p) == T - (mid * p) // 100


def lexsort_select(score, W, pct):
    T = score.size
    mid = T - 1 - W
    if T <= 1 + W or pct == 0:
        return np.arange(T, dtype=np.int32)
    n_mid = mid - (mid * pct) // 100
    pos = np.arange(1, T - W)
    order = np.lexsort((pos, -score[1:T - W]))  # primary: score desc, then position asc
    chosen = pos[order[:n_mid]]
    return np.sort(np.concatenate([[0], chosen, np.arange(T - W, T)])).astype(np.int32)


@pytest.mark.parametrize("T,W,pct", [(5000, 64, 60), (3000, 128, 35), (200, 16, 90), (100, 99, 50)])
def test_select_matches_lexsort(oq, T, W, pct):
    rng = np.random.default_rng(T + W + pct)
    score = rng.normal(0, 1, T)
    kept = oq.select(score, W, pct)
    assert np.array_equal(kept, lexsort_select(score, W, pct))
    assert kept[0] == 0 and set(range(T - W, T)) <= set(kept.tolist())
    assert np.all(np.diff(kept) > 0)
    assert kept.size == oq.kept_count(T, W, pct)


def test_select_ties_prefer_lower_position(oq):
    T, W = 1000, 10
    score = np.repeat(np.arange(10, dtype=np.float64), 100)[::-1].copy()  # 100-way ties
    score[5] = -0.0
    kept = oq.select(score, W, 55)
    assert np.array_equal(kept, lexsort_select(score, W, 55))
    # the boundary score level is split by position: the lower ones are kept
    n_mid = (T - 1 - W) - ((T - 1 - W) * 55) // 100
    assert kept.size == 1 + n_mid + W


def test_score_matches_long_double(oq):
    wl = synth.WORKLOADS["tiny"]
    K, _ = synth.gen_layer(wl, 0, "cpu", tokens=700)
    kb = K.view(torch.int16).numpy().view(np.uint16)
    W = 64
    score, mean = oq.score_unit(kb, W, return_mean=True)
    k = oq.bf16_bits_to_f32(kb).reshape(kb.shape).astype(np.longdouble)
    m = (k[:, -W:, :].sum(1) / W)
    assert np.array_equal(mean, m.astype(np.float32))
    ref = np.einsum("htd,hd->t", k, mean.astype(np.longdouble))
    assert np.max(np.abs(score - ref.astype(np.float64)) / np.abs(ref).max()) < 1e-13
    # signed score, the largest are kept
    kept = oq.select(score, W, 60)
    mid = np.arange(1, 700 - W)
    dropped = np.setdiff1d(mid, kept)
    assert score[np.intersect1d(mid, kept)].min() >= score[dropped].max()
