"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these compares the oracle with itself: they use hand-worked fixtures
(tests/golden), closed forms, invariants, brute force on tiny inputs, and
library routines (torch's scaled_dot_product_attention and softmax in fp64).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import hkv_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(12345)


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

@pytest.mark.parametrize("nq,nk,d,pos0", [(1, 1, 4, 0), (5, 9, 16, 4), (7, 7, 64, 0),
                                          (3, 40, 128, 37)])
def test_attention_matches_torch_sdpa(nq, nk, d, pos0):
    q = rng.standard_normal((nq, d)) * 2
    k = rng.standard_normal((nk, d))
    v = rng.standard_normal((nk, d))
    o, p = O.causal_attention(q, k, v, q_pos0=pos0)
    mask = torch.tensor([[j <= pos0 + i for j in range(nk)] for i in range(nq)])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None], attn_mask=mask[None])
    np.testing.assert_allclose(o, ref[0].numpy(), rtol=0, atol=1e-12)
    w = torch.softmax((torch.tensor(q) @ torch.tensor(k).T / math.sqrt(d)).masked_fill(~mask, -math.inf), -1)
    np.testing.assert_allclose(p, w.numpy(), rtol=0, atol=1e-14)
    np.testing.assert_allclose(p.sum(1), 1.0, atol=1e-14)
    assert np.all(p[~mask.numpy()] == 0.0)


def test_attention_single_key_returns_its_value():
    q = rng.standard_normal((1, 8))
    k = rng.standard_normal((3, 8))
    v = rng.standard_normal((3, 8))
    o, p = O.causal_attention(q, k, v, q_pos0=0)  # position 0 sees key 0 only
    assert p[0].tolist() == [1.0, 0.0, 0.0]
    np.testing.assert_array_equal(o[0], v[0])


# --------------------------------------------------------------------------
# head grouping
# --------------------------------------------------------------------------

def test_classify_golden():
    g = _load("classify_worked.json")
    for c in g["cases"]:
        n_tau, label, _ = O.classify(c["p"], c["W"], g["tau"])
        assert (n_tau, label) == (c["n_tau"], c["label"]), c["why"]


@pytest.mark.parametrize("N", [7, 13, 23, 51, 97, 383])
def test_classify_uniform_closed_form(N):
    # uniform weights: C(k) = k / N, so n_tau = ceil(0.9 N) (0.9 N not an integer)
    n_tau, _, cw = O.classify(np.full(N, 1.0 / N), W=10_000, tau=0.9)
    assert n_tau == math.ceil(0.9 * N)
    for W in (n_tau, n_tau + 1):
        _, label, _ = O.classify(np.full(N, 1.0 / N), W=W, tau=0.9)
        assert label == (1 if n_tau < W else 0)


@pytest.mark.parametrize("a,N", [(0.5, 40), (0.8, 100), (0.95, 300), (0.99, 384)])
def test_classify_geometric_closed_form(a, N):
    # p(delta) = (1-a) a^delta / (1 - a^N): C(k) = (1 - a^k) / (1 - a^N), so
    # n_tau = ceil(log(1 - tau (1 - a^N)) / log a)
    delta = np.arange(N)
    p_delta = (1 - a) * a ** delta / (1 - a ** N)
    row = p_delta[::-1]  # row index j = position; delta = N-1-j
    expect = math.ceil(math.log(1 - 0.9 * (1 - a ** N)) / math.log(a))
    n_tau, _, _ = O.classify(row, W=10_000, tau=0.9)
    assert n_tau == expect


def test_classify_direction_and_strictness():
    # mass piled on the oldest token: accumulating from the newest needs them all
    row = np.array([0.91] + [0.09 / 9] * 9)
    assert O.classify(row, W=11, tau=0.9)[:2] == (10, 1)
    assert O.classify(row, W=10, tau=0.9)[:2] == (10, 0)  # 10 < 10 is false
    # the current token counts: all mass on it gives n_tau = 1
    row = np.zeros(10); row[-1] = 1.0
    assert O.classify(row, W=2, tau=0.9)[:2] == (1, 1)


def test_windowed_sum_identity():
    # Local <=> the W-1 newest weights already reach tau (C is monotone)
    for _ in range(300):
        n = int(rng.integers(2, 200))
        row = rng.dirichlet(np.full(n, float(rng.choice([0.05, 0.3, 1.0]))))
        W = int(rng.integers(1, n + 2))
        n_tau, label, cw = O.classify(row, W=W, tau=0.9)
        assert label == (1 if cw >= 0.9 else 0)
        assert cw == pytest.approx(row[::-1][: W - 1].sum(), abs=1e-12)
        cum = np.cumsum(row[::-1])
        assert cum[n_tau - 1] >= 0.9 - 1e-12 and (n_tau == 1 or cum[n_tau - 2] < 0.9 + 1e-12)


def test_planted_heads_clear_cut():
    """A head whose last query is aimed at its left neighbour with a logit
    gap >= 20 must be Local; one aimed at far-away keys must be Global."""
    d, P, W = 64, 97, 28
    k = rng.standard_normal((P, d))
    q = np.zeros((P, d))
    target = k[P - 2] / np.linalg.norm(k[P - 2])
    q[P - 1] = target * 60.0 * math.sqrt(d)
    _, p = O.causal_attention(q[P - 1:], k, k, q_pos0=P - 1)
    s = (q[P - 1] @ k.T) / math.sqrt(d)
    assert (s[P - 2] - np.delete(s, P - 2)).min() >= 20
    assert O.classify(p[0], W=W, tau=0.9)[:2] == (2, 1)
    far = rng.choice(np.arange(0, P - 40), size=8, replace=False)
    q[P - 1] = 8.0 * k[far].mean(0) * 4
    _, p = O.causal_attention(q[P - 1:], k, k, q_pos0=P - 1)
    n_tau, label, _ = O.classify(p[0], W=W, tau=0.9)
    assert label == 0 and n_tau > P - 40


# --------------------------------------------------------------------------
# budgets
# --------------------------------------------------------------------------

def test_budgets_golden():
    g = _load("budgets_worked.json")
    for c in g["cases"]:
        labels = np.array([1] * c["n_local"] + [0] * (c["H"] - c["n_local"]))
        rng.shuffle(labels)
        nl, bg, T = O.budgets(labels, c["L"], c["W"], *c["rho"])
        assert (nl, T, bg) == (c["n_local"], c["T"], c["budget_g"]), c["why"]
        assert nl * c["W"] + (c["H"] - nl) * bg <= T


def test_budgets_reject_too_small_ratio():
    with pytest.raises(ValueError):
        O.budgets(np.zeros(8), L=100, W=30, rho_num=1, rho_den=4)  # 200 < 240


def test_budgets_invariants_random():
    for _ in range(200):
        H = int(rng.integers(1, 40)); L = int(rng.integers(50, 3000)); W = int(rng.integers(1, 60))
        den = int(rng.choice([1, 2, 4, 6, 8]))
        labels = rng.integers(0, 2, H)
        if (H * L) // den < H * W:
            continue
        nl, bg, T = O.budgets(labels, L, W, 1, den)
        ng = H - nl
        assert nl * W + ng * bg <= T
        if ng:
            assert T - nl * W - ng * bg < ng  # only the rounding remainder is left over
            assert bg >= W


# --------------------------------------------------------------------------
# stratified token eviction
# --------------------------------------------------------------------------

def test_ste_select_golden():
    g = _load("ste_select_worked.json")
    for c in g["cases"]:
        ev, _, _ = O.ste_select(c["score"], c["pos"], c["t"], c["D"], c["k_near"], c["k_far"],
                                c["stratified"])
        got = sorted(np.asarray(c["pos"])[ev].tolist())
        assert got == c["evicted"], c["why"]


def _brute_bottom_k(keys, k):
    """The unique k-subset whose largest key is below every other key."""
    if k == 0:
        return set()
    idx = range(len(keys))
    winners = [set(s) for s in itertools.combinations(idx, k)
               if all(max(keys[i] for i in s) < keys[j] for j in idx if j not in s)]
    assert len(winners) == 1
    return winners[0]


def test_ste_select_brute_force_tiny():
    for trial in range(150):
        t = 40
        n = int(rng.integers(3, 20))
        pos = np.sort(rng.choice(np.arange(t + 1), size=n, replace=False))
        if pos[-1] != t:
            pos[-1] = t  # the current token is always cached
        score = rng.choice([0.1, 0.2, 0.3, 0.5], size=n) if trial % 2 else rng.random(n)
        D = int(rng.integers(1, 20))
        kn, kf = int(rng.integers(0, 4)), int(rng.integers(0, 4))
        ev, _, _ = O.ste_select(score, pos, t, D, kn, kf, True)
        delta = t - pos
        near = [i for i in range(n) if 1 <= delta[i] <= D]
        far = [i for i in range(n) if delta[i] > D]
        # shortfall rule
        a, b = kn, kf
        if a > len(near): b += a - len(near); a = len(near)
        if b > len(far): a += b - len(far); b = len(far); a = min(a, len(near))
        if len(near) > 12 or len(far) > 12:
            continue
        expect = set()
        for group, kk in ((near, a), (far, b)):
            keys = [(score[i], pos[i]) for i in group]
            expect |= {group[i] for i in _brute_bottom_k(keys, kk)}
        assert set(np.flatnonzero(ev)) == expect
        assert not ev[pos == t].any()  # current token never evicted


def test_ste_scores_against_torch_softmax():
    d, L, t, r = 32, 60, 50, 8
    qa = rng.standard_normal((L, d)); ka = rng.standard_normal((L, d))
    kept = np.sort(np.concatenate([rng.choice(np.arange(40), 20, replace=False),
                                   np.arange(41, t + 1)]))
    s = O.ste_scores(qa, ka, kept, t, r)
    ref = np.zeros(kept.size)
    for step in range(t - r + 1, t + 1):
        vis = kept <= step
        w = torch.softmax(torch.tensor(ka[kept[vis]]) @ torch.tensor(qa[step]) / math.sqrt(d), 0)
        ref[vis] += w.numpy()
    np.testing.assert_allclose(s, ref, rtol=0, atol=1e-13)
    assert s.sum() == pytest.approx(r, abs=1e-12)  # each query's weights sum to 1
    assert s[kept == t][0] == pytest.approx(
        torch.softmax(torch.tensor(ka[kept]) @ torch.tensor(qa[t]) / math.sqrt(d), 0)[-1].item())


# --------------------------------------------------------------------------
# whole unit
# --------------------------------------------------------------------------

def _small_unit(H=6, d=16, L=90, P=30, W=6, M=8, D=10, r=4, rho=(1, 3), seed=0, amp=8.0):
    g = np.random.default_rng(seed)
    k = g.standard_normal((H, L, d)); v = g.standard_normal((H, L, d))
    q = g.standard_normal((H, L, d))
    for h in range(H):
        for t in range(1, L):
            if h % 2 == 0:
                idx = [t - o for o in (1, 2, 3) if t - o >= 0]
            else:
                idx = g.integers(0, t, 6)
            q[h, t] += amp * k[h, idx].mean(0)
    prm = O.UnitParams(num_heads=H, head_dim=d, max_len=L, prefill_len=P, local_window=W,
                       ste_m=M, near_dist=D, score_window=r, rho_num=rho[0], rho_den=rho[1])
    return prm, q, k, v


def test_unit_invariants():
    prm, q, k, v = _small_unit()
    res = O.run_unit(prm, q, k, v)
    H, L, P, W, M, D = 6, prm.max_len, prm.prefill_len, prm.local_window, prm.ste_m, prm.near_dist
    assert set(res.labels.tolist()) == {0, 1}  # both kinds appear in this unit
    nl, bg, T = O.budgets(res.labels, L, W, prm.rho_num, prm.rho_den)
    assert (res.n_local, res.budget_g) == (nl, bg)
    assert res.n_local * W + (H - res.n_local) * res.budget_g <= T
    assert res.stats["n_events"] > 0
    kept = {h: set(range(P)) if res.labels[h] == 0 else set(range(P - W, P)) for h in range(H)}
    events = dict(zip(res.event_step.tolist(), range(len(res.event_step))))
    for t in range(P - 1, L):
        if t >= P:
            for h in range(H):
                kept[h].add(t)
                if res.labels[h] == 1:
                    kept[h].discard(t - W)
        if t in events:
            e = events[t]
            for h in range(H):
                if res.labels[h] != 0:
                    continue
                gone = [x for x in res.evicted[e, h] if x >= 0]
                n_before = len(kept[h])
                assert set(gone) <= kept[h]
                assert t not in gone  # never the current token
                if t >= P:
                    assert n_before == bg + M
                    near = [x for x in gone if t - x <= D]
                    assert len(near) == M // 2 and len(gone) == M  # M/2 + M/2
                kept[h] -= set(gone)
                assert len(kept[h]) == bg  # exactly the budget after eviction
        for h in range(H):
            if res.labels[h] == 1 and t >= P:
                assert kept[h] == set(range(t - W + 1, t + 1))
    for h in range(H):
        assert set(res.kept_final[h].tolist()) == kept[h]


def test_unit_decode_matches_sdpa_on_kept_set():
    prm, q, k, v = _small_unit(seed=3)
    res = O.run_unit(prm, q, k, v)
    L, P = prm.max_len, prm.prefill_len
    t = L - 1
    last_event = res.event_step.tolist()[-1] == t
    for h in range(prm.num_heads):
        kept = res.kept_final[h]
        if last_event and res.labels[h] == 0:  # output was taken before that eviction
            kept = np.sort(np.concatenate([kept, [x for x in res.evicted[-1, h] if x >= 0]]))
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.tensor(q[h, t])[None, None], torch.tensor(k[h, kept])[None],
            torch.tensor(v[h, kept])[None])
        np.testing.assert_allclose(res.o_decode[t - P, h], ref[0, 0].numpy(), atol=1e-12)


def test_full_cache_equality():
    """rho = 1 and W = L: nothing is truncated or evicted, so the compressed
    path gives full-cache attention exactly."""
    prm, q, k, v = _small_unit(seed=5, L=70, P=20)
    prm.rho_num, prm.rho_den, prm.local_window = 1, 1, prm.max_len
    res = O.run_unit(prm, q, k, v, want_prefill=True)
    prm_full = O.UnitParams(**{**prm.__dict__, "mode": O.MODE_FULL})
    full = O.run_unit(prm_full, q, k, v, want_prefill=True)
    assert res.stats["n_events"] == 0
    np.testing.assert_allclose(res.o_decode, full.o_decode, rtol=0, atol=1e-13)
    np.testing.assert_allclose(res.o_prefill, full.o_prefill, rtol=0, atol=0)
    for h in range(prm.num_heads):
        o_all, _ = O.causal_attention(q[h], k[h], v[h])
        np.testing.assert_allclose(full.o_decode[:, h], o_all[prm.prefill_len:], atol=1e-13)
        np.testing.assert_allclose(full.o_prefill[h], o_all[:prm.prefill_len], atol=1e-13)


def test_initial_ste_when_prefill_exceeds_budget():
    # P = 60 > budget: one STE at classification, E = P - budget, split floor/ceil
    prm, q, k, v = _small_unit(seed=7, L=120, P=60, W=6, M=8, rho=(1, 4))
    res = O.run_unit(prm, q, k, v)
    bg = res.budget_g
    assert prm.prefill_len > bg
    assert res.event_step[0] == prm.prefill_len - 1
    E = prm.prefill_len - bg
    for h in np.flatnonzero(res.labels == 0):
        gone = [x for x in res.evicted[0, h] if x >= 0]
        assert len(gone) == E
        near = [x for x in gone if prm.prefill_len - 1 - x <= prm.near_dist]
        assert len(near) == E // 2


def test_unstratified_and_uniform_variants():
    prm, q, k, v = _small_unit(seed=9)
    prm_u = O.UnitParams(**{**prm.__dict__, "stratified": False})
    res_u = O.run_unit(prm_u, q, k, v)
    assert res_u.stats["n_events"] > 0
    prm_b = O.UnitParams(**{**prm.__dict__, "mode": O.MODE_UNIFORM})
    res_b = O.run_unit(prm_b, q, k, v)
    T = (prm.num_heads * prm.max_len * prm.rho_num) // prm.rho_den
    assert (res_b.labels == 0).all() and res_b.budget_g == T // prm.num_heads
    assert all(len(x) <= res_b.budget_g + prm.ste_m for x in res_b.kept_final)


def test_hints_adopt_only_near_ties():
    prm, q, k, v = _small_unit(seed=11)
    base = O.run_unit(prm, q, k, v)
    H, E = prm.num_heads, len(base.event_step)
    # replay the oracle's own decisions as hints: everything agrees
    kept_log = np.full((E, H, base.budget_g), -1, np.int32)
    state = {h: set(range(prm.prefill_len)) if base.labels[h] == 0 else None for h in range(H)}
    last = prm.prefill_len - 1
    for e, t in enumerate(base.event_step.tolist()):
        for h in range(H):
            if base.labels[h] != 0:
                continue
            state[h] |= set(range(last + 1, t + 1))
            state[h] -= {x for x in base.evicted[e, h] if x >= 0}
            kept_log[e, h] = sorted(state[h])
        last = t
    hints = {"labels": base.labels, "event_step": base.event_step, "kept": kept_log}
    same = O.run_unit(prm, q, k, v, hints=hints)
    assert same.stats["n_select_hard"] == 0 and same.stats["n_select_ties"] == 0
    # a hint that swaps a clearly-kept token for an evicted one is a hard mismatch
    bad = kept_log.copy()
    h = int(np.flatnonzero(base.labels == 0)[0])
    gone = [x for x in base.evicted[0, h] if x >= 0]
    bad[0, h, 0] = gone[0]
    bad[0, h] = np.sort(bad[0, h])
    res = O.run_unit(prm, q, k, v, hints={**hints, "kept": bad})
    assert res.stats["n_select_hard"] >= 1
    # a flipped label far from the threshold is a hard mismatch too
    lab = base.labels.copy()
    far = int(np.argmax(np.abs(base.c_window - 0.9)))
    lab[far] ^= 1
    res = O.run_unit(prm, q, k, v, hints={"labels": lab})
    assert res.stats["n_label_hard"] == 1


def _event_states(prm, res):
    """Cached positions of every Global head just before each event of an
    oracle run (from its labels, event steps and evicted logs)."""
    H, P = prm.num_heads, prm.prefill_len
    state = {h: set(range(P)) for h in range(H) if res.labels[h] == 0}
    last, before = P - 1, []
    for e, t in enumerate(res.event_step.tolist()):
        for h in state:
            state[h] |= set(range(last + 1, t + 1))
        before.append({h: sorted(x) for h, x in state.items()})
        for h in state:
            state[h] -= {x for x in res.evicted[e, h] if x >= 0}
        last = t
    return before


def _scores_numpy(q, k, kept, t, r):
    """STE scores written out with numpy: for each of the last r steps, the
    softmax (scale 1/sqrt(d)) of that step's query over the cached keys not
    newer than the step, summed per key."""
    kept = np.asarray(kept)
    s = np.zeros(kept.size)
    for step in range(t - r + 1, t + 1):
        vis = kept <= step
        x = k[kept[vis]] @ q[step] / np.sqrt(q.shape[1])
        w = np.exp(x - x.max())
        s[vis] += w / w.sum()
    return s


def test_hints_adopt_inside_the_band_and_only_there():
    """The near-tie band is relative and two-sided in the right direction:
    a hint that keeps the highest-scored evicted token g of a stratum and
    evicts the lowest-scored kept token c in its place exceeds the exact
    answer by x = (s_c - s_g) / s_g; with band 1.01 x it is
    adopted as a tie, with band 0.99 x it is a hard mismatch.  Scores are
    well below 1, so an absolute band (s_c - s_g <= band) would adopt the
    second one, and a band on the wrong side (s_c <= s_g (1 - band)) would
    reject the first.  A flipped label is adopted exactly when
    |C(W-1) - tau| is inside its band, on either side of tau."""
    prm, q, k, v = _small_unit(seed=11)
    base = O.run_unit(prm, q, k, v)
    H, E = prm.num_heads, len(base.event_step)
    assert E >= 2
    before = _event_states(prm, base)
    kept_log = np.full((E, H, base.budget_g), -1, np.int32)
    for e in range(E):
        for h in before[e]:
            gone = {x for x in base.evicted[e, h] if x >= 0}
            kept_log[e, h] = sorted(set(before[e][h]) - gone)
    hints = {"labels": base.labels, "event_step": base.event_step, "kept": kept_log}
    # the swap goes into the last event, so no later event sees its effect
    e, t = E - 1, int(base.event_step[-1])
    cases = []
    for h in before[e]:
        cached = np.array(before[e][h])
        sc = _scores_numpy(q[h], k[h], cached, t, prm.score_window)
        gone = {x for x in base.evicted[e, h] if x >= 0}
        far = (t - cached) > prm.near_dist
        ev = np.array([p in gone for p in cached])
        if not (far & ev).any() or not (far & ~ev).any():
            continue
        ig = np.flatnonzero(far & ev)[np.argmax(sc[far & ev])]
        ic = np.flatnonzero(far & ~ev)[np.argmin(sc[far & ~ev])]
        x = (sc[ic] - sc[ig]) / sc[ig]
        if x > 1e-9:
            cases.append((x, h, int(cached[ig]), int(cached[ic]), sc[ig]))
    assert cases
    x, h, pg, pc, sg = min(cases)
    assert sg < 0.5  # an absolute band would differ from the relative one here
    swapped = kept_log.copy()
    row = [p for p in swapped[e, h] if p != pc] + [pg]
    swapped[e, h] = np.sort(row)
    for factor, ties, hard in ((1.01, 1, 0), (0.99, 0, 1)):
        prm_b = O.UnitParams(**{**prm.__dict__, "select_band": x * factor})
        res = O.run_unit(prm_b, q, k, v, hints={**hints, "kept": swapped})
        assert (res.stats["n_select_ties"], res.stats["n_select_hard"]) == (ties, hard), factor
        if ties:
            assert res.stats["max_select_tie_gap"] == pytest.approx(x, rel=1e-9)
            assert sorted(res.kept_final[h]) == sorted(set(swapped[e, h]) | set(range(t + 1, prm.max_len)))
    # labels: the head closest to tau above it and below it
    gap = base.c_window - prm.tau
    for side in (gap > 0, gap < 0):
        hh = int(np.flatnonzero(side)[np.argmin(np.abs(gap[side]))])
        lab = base.labels.copy()
        lab[hh] ^= 1
        for factor, ties, hard in ((1.01, 1, 0), (0.99, 0, 1)):
            prm_b = O.UnitParams(**{**prm.__dict__, "label_band": abs(gap[hh]) * factor})
            res = O.run_unit(prm_b, q, k, v, hints={"labels": lab})
            assert (res.stats["n_label_ties"], res.stats["n_label_hard"]) == (ties, hard), (hh, factor)
            assert res.labels[hh] == lab[hh]


# --------------------------------------------------------------------------
# classifier variants: distance-averaged rows, CFG-tied rows
# --------------------------------------------------------------------------

@pytest.mark.parametrize("P,nq", [(9, 1), (9, 4), (30, 8), (97, 8), (12, 12)])
def test_class_row_uniform_closed_form(P, nq):
    """q = 0: query i spreads 1/(i+1) over positions 0..i, so the weight at
    distance delta averaged over i = P-nq..P-1 is
    (H_P - H_max(delta, P-nq)) / nq with H_n the n-th harmonic number."""
    d = 8
    q = np.zeros((P, d)); k = rng.standard_normal((P, d)); v = rng.standard_normal((P, d))
    row = O.class_row(q, k, v, nq)
    harm = np.concatenate([[0.0], np.cumsum(1.0 / np.arange(1, P + 1))])
    for delta in range(P):
        expect = (harm[P] - harm[max(delta, P - nq)]) / nq
        assert row[P - 1 - delta] == pytest.approx(expect, rel=1e-12, abs=1e-15), delta
    assert row.sum() == pytest.approx(1.0, abs=1e-12)


def test_class_row_aligns_by_distance():
    """Every query aimed at one fixed position j0 puts its weight at a
    different distance; the averaged row holds 1/nq at each distance
    i - j0, i = P-nq..P-1.  The last query alone holds it all at P-1-j0."""
    P, d, nq, j0 = 40, 16, 8, 10
    k = 0.01 * rng.standard_normal((P, d))
    e = np.zeros(d); e[3] = 1.0
    k[j0] = e * 40.0
    q = np.tile(e * 40.0, (P, 1))
    v = rng.standard_normal((P, d))
    row = O.class_row(q, k, v, nq)
    for i in range(P - nq, P):
        assert row[P - 1 - (i - j0)] == pytest.approx(1.0 / nq, abs=1e-9)
    one = O.class_row(q, k, v, 1)
    assert one[j0] == pytest.approx(1.0, abs=1e-9)
    # grouping follows: the neighbour-aimed head stays Local under averaging
    W = 28
    kk = rng.standard_normal((P, d))
    qq = np.zeros((P, d))
    for i in range(1, P):
        qq[i] = 60.0 * math.sqrt(d) * kk[i - 1] / np.linalg.norm(kk[i - 1])
    for n in (1, nq):
        assert O.classify(O.class_row(qq, kk, kk, n), W=W, tau=0.9)[:2] == (2, 1)


def test_class_row_one_query_is_last_weight_row():
    P, d = 33, 16
    q, k, v = (rng.standard_normal((P, d)) for _ in range(3))
    _, p = O.causal_attention(q[P - 1:], k, v, q_pos0=P - 1)
    np.testing.assert_array_equal(O.class_row(q, k, v, 1), p[0])


def test_cfg_partner_pairs():
    for S in (2, 4, 64):
        for pairing in (O.CFG_HALVES, O.CFG_ADJACENT):
            part = [O.cfg_partner(s, S, pairing) for s in range(S)]
            assert sorted(part) == list(range(S))
            assert all(part[p] == s and p != s for s, p in enumerate(part))
        assert [O.cfg_partner(s, S, O.CFG_HALVES) for s in range(S)][: S // 2] == \
            list(range(S // 2, S))
        assert all(O.cfg_partner(s, S, O.CFG_UNTIED) == s for s in range(S))
    with pytest.raises(ValueError):
        O.cfg_partner(0, 3, O.CFG_HALVES)


def test_tied_rows_decide_one_label_for_the_pair():
    """Two rows whose own windows hold 0.95 and 0.80 of the mass: alone one
    is Local and one Global; tied (mean 0.875 < 0.9) both are Global."""
    P, W = 20, 5

    def row_with(c_window):
        r = np.zeros(P)
        r[P - (W - 1):] = c_window / (W - 1)   # the W-1 newest tokens
        r[: P - (W - 1)] = (1 - c_window) / (P - (W - 1))
        return r

    a, b = row_with(0.95), row_with(0.80)
    assert O.classify(a, W, 0.9)[1] == 1 and O.classify(b, W, 0.9)[1] == 0
    t = O.tied_rows(a, b)
    assert O.classify(t, W, 0.9)[1] == 0
    assert O.classify(t, W, 0.9)[2] == pytest.approx(0.875, abs=1e-12)
    np.testing.assert_array_equal(O.tied_rows(a, b), O.tied_rows(b, a))


def test_unit_classifier_variants():
    """cls_queries = r runs the whole unit with both labels present and the
    budget invariants intact; a unit given its own one-query rows as
    cls_rows reproduces the default run exactly; a unit given a tied row
    takes its labels from that row."""
    prm, q, k, v = _small_unit(seed=5)
    base = O.run_unit(prm, q, k, v)
    H, P = prm.num_heads, prm.prefill_len
    own = np.stack([O.class_row(q[h, :P], k[h, :P], v[h, :P], 1) for h in range(H)])
    same = O.run_unit(prm, q, k, v, cls_rows=own)
    np.testing.assert_array_equal(same.labels, base.labels)
    np.testing.assert_array_equal(same.o_decode, base.o_decode)
    prm_r = O.UnitParams(**{**prm.__dict__, "cls_queries": prm.score_window})
    res_r = O.run_unit(prm_r, q, k, v)
    avg = np.stack([O.class_row(q[h, :P], k[h, :P], v[h, :P], prm.score_window)
                    for h in range(H)])
    for h in range(H):
        assert res_r.labels[h] == O.classify(avg[h], prm.local_window, 0.9)[1]
    nl, bg, _ = O.budgets(res_r.labels, prm.max_len, prm.local_window, prm.rho_num, prm.rho_den)
    assert res_r.n_local == nl and res_r.budget_g == bg
    assert all(len(x) <= (bg + prm.ste_m if res_r.labels[h] == 0 else prm.local_window)
               for h, x in enumerate(res_r.kept_final))
    g = np.random.default_rng(3)
    q2, k2 = q + 0.5 * g.standard_normal(q.shape), k + 0.5 * g.standard_normal(k.shape)
    other = np.stack([O.class_row(q2[h, :P], k2[h, :P], v[h, :P], 1) for h in range(H)])
    tied = O.tied_rows(own, other)
    res_t = O.run_unit(prm, q, k, v, cls_rows=tied)
    for h in range(H):
        assert res_t.labels[h] == O.classify(tied[h], prm.local_window, 0.9)[1]
    with pytest.raises(ValueError):
        O.run_unit(O.UnitParams(**{**prm.__dict__, "cls_queries": prm.score_window + 1}),
                   q, k, v)


def test_class_row_from_weights_worked_example():
    """P = 3, the last two queries.  Query at position 1 puts 0.3, 0.7 on
    positions 0, 1 (distances 1, 0); query at position 2 puts 0.2, 0.3, 0.5
    on positions 0, 1, 2 (distances 2, 1, 0).  Per distance, averaged:
    delta 0: (0.7 + 0.5) / 2 = 0.6; delta 1: (0.3 + 0.3) / 2 = 0.3;
    delta 2: (0 + 0.2) / 2 = 0.1 (the query at 1 cannot reach distance 2).
    In the last query's position order: [0.1, 0.3, 0.6]."""
    w = np.array([[0.3, 0.7, 0.0], [0.2, 0.3, 0.5]])
    np.testing.assert_allclose(O.class_row_from_weights(w), [0.1, 0.3, 0.6], atol=1e-15)
    # the entries past a query's own position are never read
    w2 = w.copy(); w2[0, 2] = 123.0
    np.testing.assert_array_equal(O.class_row_from_weights(w2), O.class_row_from_weights(w))
    # from q, k, v: the same as averaging the causal weights of those queries
    P, d, nq = 25, 8, 6
    q, k, v = (rng.standard_normal((P, d)) for _ in range(3))
    _, p = O.causal_attention(q[P - nq:], k, v, q_pos0=P - nq)
    np.testing.assert_array_equal(O.class_row(q, k, v, nq), O.class_row_from_weights(p))
