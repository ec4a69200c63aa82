"""Pins of the parity accounting: the decision margins the oracle reports, and
the counting in oracle/parity.py that excuses a GPU/oracle mismatch only near
a decision boundary.  CPU only.
"""
import numpy as np

from e8_lattice_vector_nq_b200 import synth


def test_e8_margin_hand_worked(oq):
    # integer coset: f = 0, |e| = |y|, nearest rounding tie |0.3 - 0.5| = 0.2 -> 0.4;
    # half coset: u = y - 1/2, the closest to a tie is u = -0.45 -> 0.1; even sums;
    # d0 = 0.2775, d1 = 0.9275 -> 0.70; so the margin is the half coset's 0.1
    y = np.array([[0.1, 0.2, 0.15, 0.3, -0.2, -0.1, 0.05, 0.25]], np.float32)
    assert abs(oq.e8_margins(y)[0] - 0.1) < 1e-6
    # odd integer sum (f = (1, 0, ...)): |e| = (0.3, 0.1, 0.2, 0.1 ...) -> parity gap
    # (0.3 - 0.2) / 0.3 = 1/3; the other margins are larger (rounding 0.4 / 0.6 / 0.8,
    # half coset rounding 0.6, 0.2 ... -> 0.2 is the smallest)
    y = np.array([[0.7, 0.1, 0.2, 0.1, 0.1, 0.1, 0.1, 0.1]], np.float32)
    assert abs(oq.e8_margins(y)[0] - 0.2) < 1e-6


def test_e8_margin_zero_on_each_kind_of_boundary(oq):
    y = np.array([
        [0.5, 0.1, 0.2, 0.1, 0.3, 0.1, 0.2, 0.1],     # integer-coset rounding tie
        [0.25] * 8,                                   # coset tie (d0 = d1 = 0.5)
        [0.6, 0.4, 0.1, 0.1, 0.1, 0.1, 0.1, 0.1],     # parity move: two |e| = 0.4
        [1.0, 0.1, 0.2, 0.1, 0.3, 0.1, 0.2, 0.1],     # half-coset rounding tie (u = 0.5)
    ], np.float32)
    m = oq.e8_margins(y)
    assert np.all(m < 1e-6), m


def test_e8_margin_grows_with_distance_from_a_tie(oq):
    # moving a coordinate off the integer rounding tie by d gives margin 2 d / 1
    for d in (1e-6, 1e-4, 1e-2):
        y = np.array([[0.5 + d, 0.1, 0.2, 0.1, 0.3, 0.1, 0.2, 0.1]], np.float32)
        got = oq.e8_margins(y)[0]
        assert abs(got - 2 * d) <= 1e-6 + 1e-3 * d, (d, got)


def test_encode_margin_bounded_by_the_scale_rounding(oq):
    # the scale decision: P = fp32(M * G_2) against the midpoint of its fp16
    # neighbours, restated with numpy's float16 (a library routine)
    import torch

    wl = synth.WORKLOADS["tiny"]
    _, V = synth.gen_layer(wl, 0, "cpu", tokens=64)
    xv = V.reshape(-1, 128).contiguous().view(torch.int16).numpy().view(np.uint16)
    m = oq.encode_margins(xv, 2)
    v = oq.fwht(oq.bf16_bits_to_f32(xv).reshape(-1, 128))
    M = np.abs(v).max(axis=1).astype(np.float32)
    G = np.float32(1.0 / (1.5 * np.sqrt(128.0)))  # fp32 nearest to 1 / (A_2 sqrt(128))
    P = (M * G).astype(np.float32)
    h = P.astype(np.float16)
    up = np.nextafter(h, np.float16(np.inf))
    dn = np.nextafter(h, np.float16(0))
    other = np.where(P.astype(np.float64) >= h.astype(np.float64), up, dn)
    mid = 0.5 * (h.astype(np.float64) + other.astype(np.float64))
    sig_margin = np.abs(P.astype(np.float64) - mid) / P.astype(np.float64)
    assert np.all(m <= sig_margin + 1e-12)
    assert np.all(m >= 0) and np.all(m <= 1)
    assert oq.encode_margins(np.zeros((1, 128), np.uint16), 3)[0] == 1.0


def test_parity_counts_excuse_only_near_boundaries(oq):
    from oracle import parity

    wl = synth.WORKLOADS["mistral7b_32k"]
    T, W, pct, H = 700, 16, 60, 2
    import torch

    K, V = synth.gen_layer(wl, 0, "cpu", tokens=T)
    K, V = K[:H], V[:H]
    k16 = K.contiguous().view(torch.int16).numpy().view(np.uint16)
    v16 = V.contiguous().view(torch.int16).numpy().view(np.uint16)
    s = oq.score_unit(k16, W)
    kept = oq.select(s, W, pct)
    r = oq.encode_unit(k16, v16, kept.size, kept=kept, theta=wl.theta)
    Ko, Vo = oq.decode_unit(r["k_codes"], r["k_meta"], r["v_codes"], r["v_meta"],
                            positions=kept, theta=wl.theta)
    job = {"K": k16, "V": v16, "theta": wl.theta, "bits_k": 3, "bits_v": 2, "window": W,
           "pct": pct, "gpu_scores": s.copy(), "gpu_kept": kept.copy(),
           "gk_codes": r["k_codes"].copy(), "gk_meta": r["k_meta"].copy(),
           "gv_codes": r["v_codes"].copy(), "gv_meta": r["v_meta"].copy(), "gK": Ko.copy(),
           "gV": Vo.copy()}
    ok = parity.check_layer(job)
    assert parity.verdict(ok) == [] and ok["mismatch_codes"] == 0 and ok["bf16_diff"] == 0
    assert ok["vectors"] == 2 * H * kept.size and ok["kept_diff"] == 0

    # a flipped code bit far from any boundary: one unexcused mismatch
    bad = dict(job, gk_codes=job["gk_codes"].copy())
    bad["gk_codes"][1, 5, 0] ^= 1
    res = parity.check_layer(bad)
    assert res["unexcused_codes"] == 1 and res["mismatch_vectors"] == 1
    assert parity.verdict(res)

    # a kept-set swap at the threshold is excused, one elsewhere is not
    mid = kept[(kept > 0) & (kept < T - W)]
    thr_pos = mid[np.argmin(s[mid])]
    dropped = np.setdiff1d(np.arange(1, T - W), kept)
    nxt = dropped[np.argmax(s[dropped])]
    s2 = s.copy()
    s2[nxt] = s[thr_pos] * (1 + 1e-7 * np.sign(s[thr_pos]))  # within 1e-5 of the threshold
    near = parity.kept_set_parity(s2, kept, np.sort(np.r_[np.setdiff1d(kept, [thr_pos]), nxt]),
                                  W, pct)
    assert near["kept_diff"] == 2 and near["kept_excused"] == 2 and near["kept_unexcused"] == 0
    far_pos = dropped[np.argmin(s[dropped])]
    far = parity.kept_set_parity(s, kept, np.sort(np.r_[np.setdiff1d(kept, [thr_pos]), far_pos]),
                                 W, pct)
    assert far["kept_unexcused"] == 1
    # a decoded element that differs
    dec = dict(job, gV=job["gV"].copy())
    dec["gV"][0, 3, 7] ^= 1
    assert parity.check_layer(dec)["bf16_diff"] == 1


def test_code_fields_unpack_every_coordinate(oq):
    from oracle import parity

    rng = np.random.default_rng(5)
    for bits in (2, 3):
        j = rng.integers(0, 1 << bits, size=(7, 128)).astype(np.uint64)
        words = np.zeros((7, 4 * bits), np.uint64)
        for c in range(128):
            p = bits * c
            words[:, p >> 5] |= (j[:, c] << np.uint64(p & 31)) & np.uint64(0xFFFFFFFF)
            if (p & 31) + bits > 32:
                words[:, (p >> 5) + 1] |= j[:, c] >> np.uint64(32 - (p & 31))
        assert np.array_equal(parity.code_fields(words.astype(np.uint32), bits), j)


def test_parity_jobs_run_in_spawn_workers(oq):
    """The worker pool the full-size GPU tests use: spawn processes, lazily
    built jobs, merged counts."""
    import torch

    from oracle import parity

    wl = synth.WORKLOADS["tiny"]
    K, V = synth.gen_layer(wl, 0, "cpu", tokens=40)
    k16 = K.contiguous().view(torch.int16).numpy().view(np.uint16)
    v16 = V.contiguous().view(torch.int16).numpy().view(np.uint16)
    r = oq.encode_unit(k16, v16, 40, theta=wl.theta)

    def jobs():
        for i in range(3):
            gv = r["v_codes"].copy()
            if i == 2:
                gv[0, 0, 0] ^= 4  # one planted mismatch in the last job
            yield {"K": k16, "V": v16, "theta": wl.theta, "bits_k": 3, "bits_v": 2, "window": 0,
                   "pct": 0, "gk_codes": r["k_codes"], "gk_meta": r["k_meta"], "gv_codes": gv,
                   "gv_meta": r["v_meta"]}

    pool = parity.make_pool(2)
    try:
        tot = parity.merge(parity.run_jobs(pool, jobs(), inflight=2))
    finally:
        pool.shutdown()
    assert tot["units"] == 3 and tot["vectors"] == 3 * 2 * 8 * 40
    assert tot["mismatch_vectors"] == 1 and tot["unexcused_codes"] == 1
    assert parity.verdict(tot) and "code mismatches" in parity.verdict(tot)[0]


def test_parity_counts_exact_layout(oq):
    """The exact-layout path of the accounting: the oracle's own folded
    store passes; one flipped coset bit (the low bit of a code 7) fails."""
    import torch

    from oracle import parity

    wl = synth.WORKLOADS["tiny"]
    K, V = synth.gen_layer(wl, 0, "cpu", tokens=24)
    k16 = K.contiguous().view(torch.int16).numpy().view(np.uint16)
    v16 = V.contiguous().view(torch.int16).numpy().view(np.uint16)
    H, n = k16.shape[0], 24
    c, s = oq.rope_cs(wl.theta, np.arange(n))
    kw, ks = oq.fold_exact(*oq.encode_vectors_box(k16.reshape(-1, 128), 3, rope=True,
                                                  c=np.tile(c, (H, 1)), s=np.tile(s, (H, 1))), 3)
    vw, vs = oq.fold_exact(*oq.encode_vectors_box(v16.reshape(-1, 128), 2), 2)
    job = {"K": k16, "V": v16, "theta": wl.theta, "bits_k": 3, "bits_v": 2, "window": 0, "pct": 0,
           "exact": True, "gk_codes": kw.reshape(H, n, 12), "gk_meta": ks.reshape(H, n),
           "gv_codes": vw.reshape(H, n, 8), "gv_meta": vs.reshape(H, n)}
    assert parity.verdict(parity.check_layer(job)) == []
    bad = dict(job, gk_codes=job["gk_codes"].copy())
    bad["gk_codes"][0, 3, 0] ^= 1 << 21  # group 0's coset bit
    r = parity.check_layer(bad)
    assert r["unexcused_codes"] >= 1 and parity.verdict(r)
