"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Integer decisions (labels, kept sets, evicted sets) are compared bit-exactly
(outside the near-tie bands of tests/lockstep.py); attention outputs within
the tolerance of the arithmetic: max-abs relative error per decode call
<= 2e-2 for bf16 caches and <= 1e-5 for fp32.
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_hkv_b200 as hkv
from kv_cache_compression_hkv_b200.inputs import WORKLOADS
from oracle import hkv_oracle as O

from lockstep import assert_lockstep, compare_unit, generate, run_gpu

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
TOL = {"f32": 1e-5, "bf16": 2e-2}


@pytest.fixture(scope="module", autouse=True)
def built():
    from kv_cache_compression_hkv_b200 import build
    build.build()
    assert torch.cuda.is_available(), "these tests need a CUDA device"


# ---------------------------------------------------------------------------
# standalone primitives: identical inputs on both sides, bit-exact answers
# ---------------------------------------------------------------------------

def test_classify_rows_bitexact():
    g = np.random.default_rng(0)
    rows, Ws = [], []
    for i in range(600):
        n = int(g.integers(2, 700))
        a = float(g.choice([0.02, 0.2, 1.0, 5.0]))
        x = g.dirichlet(np.full(n, a))
        if i % 5 == 0:
            x = np.zeros(n); x[-1 - int(g.integers(0, n))] = 1.0
        rows.append(x.astype(np.float32)); Ws.append(int(g.integers(1, 60)))
    for W in (1, 20, 28, 56):
        for n in (65, 97, 384):
            N = 13 if n == 65 else n
            rows.append(np.full(n, 1.0 / N, np.float32) * (np.arange(n) >= n - N)); Ws.append(W)
    n_max = max(r.size for r in rows)
    for W in sorted(set(Ws)):
        sel = [r for r, w in zip(rows, Ws) if w == W]
        for n in sorted({r.size for r in sel}):
            batch = np.stack([r for r in sel if r.size == n])
            nt, lab = hkv.classify_rows(torch.tensor(batch, device=DEV), W)
            nt, lab = nt.cpu().numpy(), lab.cpu().numpy()
            for i, row in enumerate(batch):
                e_nt, e_lab, _ = O.classify(row.astype(np.float64), W, 0.9)
                assert (nt[i], lab[i]) == (e_nt, e_lab), (n, W, i)
    assert n_max < 1000


def _weight_blocks(g, U, r, n):
    """[U, r, n] fp32 kept weight rows: row q is a softmax over positions
    0..n-r+q (zero after), with a per-unit mix of recency and spread so
    that the grouping lands on both sides of tau."""
    blocks = np.zeros((U, r, n), np.float32)
    for u in range(U):
        gamma = float(g.choice([0.02, 0.1, 0.3, 1.0, 3.0]))
        for q in range(r):
            i = n - r + q
            logits = gamma * (np.arange(i + 1) - i) + g.standard_normal(i + 1)
            w = np.exp(logits - logits.max())
            blocks[u, q, : i + 1] = w / w.sum()
    return blocks


@pytest.mark.parametrize("n,nq", [(40, 1), (97, 4), (97, 8), (384, 8), (130, 3), (9, 8)])
def test_classify_groups_bitexact(n, nq):
    """Grouping by the last nq queries' per-distance weights, alone and tied
    in pairs, on identical fp32 rows: n_tau and labels equal the oracle's
    (averaging in the same order; only the running sum's order differs,
    which decides nothing unless a sum lands within a few ulps of tau)."""
    g = np.random.default_rng(n * 10 + nq)
    U, r, W = 96, 8, 28 if n > 28 else 4
    blocks = _weight_blocks(g, U, r, n)
    partner = np.arange(U, dtype=np.int32)
    partner[: U // 2] ^= 1                                   # adjacent pairs
    partner[48:88] = 48 + (np.arange(40) + 20) % 40         # halves of the next 40
    # the last 8 stay alone
    for part in (None, partner):
        nt, lab = hkv.classify_groups(torch.tensor(blocks, device=DEV), nq, W,
                                      partner=None if part is None else torch.tensor(part, device=DEV))
        nt, lab = nt.cpu().numpy(), lab.cpu().numpy()
        rows = [O.class_row_from_weights(blocks[u, r - nq:].astype(np.float64)) for u in range(U)]
        for u in range(U):
            p = u if part is None else int(part[u])
            row = rows[u] if p == u else O.tied_rows(rows[min(u, p)], rows[max(u, p)])
            e_nt, e_lab, _ = O.classify(row, W, 0.9)
            assert (nt[u], lab[u]) == (e_nt, e_lab), (u, p)
        assert 0 < lab.sum() < U  # both kinds present
        if part is not None:
            assert all(nt[u] == nt[int(part[u])] for u in range(U))
    bad = torch.tensor(np.full(U, U, np.int32), device=DEV)
    nt, lab = hkv.classify_groups(torch.tensor(blocks, device=DEV), nq, W, partner=bad)
    assert (nt.cpu().numpy() == -1).all() and (lab.cpu().numpy() == 255).all()


@pytest.mark.parametrize("n,stratified", [(40, True), (230, True), (834, True), (2480, True),
                                          (230, False), (33, True), (1, True)])
def test_select_batch_bitexact(n, stratified):
    g = np.random.default_rng(n)
    P = 96
    score = np.zeros((P, n), np.float32)
    pos = np.zeros((P, n), np.int32)
    count = np.zeros(P, np.int32)
    tt = np.zeros(P, np.int32)
    for i in range(P):
        m = n if i % 3 else int(g.integers(1, n + 1))
        t = int(g.integers(m - 1, 3 * n + 5))
        p = np.sort(g.choice(np.arange(t), size=m - 1, replace=False)) if m > 1 else np.zeros(0, int)
        p = np.concatenate([p, [t]])
        g.shuffle(p)
        if i % 4 == 0:     # heavy ties
            s = g.choice([0.0, 0.125, 0.25, 1.0], size=m)
        elif i % 4 == 1:   # tiny and denormal-free spread
            s = g.random(m) ** 8
        else:
            s = g.random(m)
        score[i, :m] = s; pos[i, :m] = p; count[i] = m; tt[i] = t
    D, kn, kf = 48, 16, 16
    ev = hkv.ste_select_batch(*(torch.tensor(a, device=DEV) for a in (score, pos, count, tt)),
                              D=D, k_near=kn, k_far=kf, stratified=stratified).cpu().numpy()
    for i in range(P):
        m = count[i]
        e, _, _ = O.ste_select(score[i, :m].astype(np.float64), pos[i, :m], int(tt[i]), D, kn, kf,
                               stratified)
        np.testing.assert_array_equal(ev[i, :m].astype(bool), e, err_msg=f"problem {i}")
        assert not ev[i, m:].any()


# ---------------------------------------------------------------------------
# whole hot path, lock-step with the oracle
# ---------------------------------------------------------------------------

def _lockstep(w, units, seed=0, fused=True, mode=hkv.MODE_HEADKV, stratified=True,
              cls_queries=1, pairing=hkv.CFG_UNTIED, tau=0.9, expect_label=None):
    cfg = hkv.config_for(w, mode=mode, stratified=stratified, cls_queries=cls_queries,
                         cfg_pairing=pairing)
    cfg.tau = tau
    data = generate(w, seed, DEV)
    cache, rec, _ = run_gpu(w, cfg, data, units, fused=fused)
    rc, detail = cache.check()
    assert rc == 0, (rc, detail)
    omode = {hkv.MODE_HEADKV: O.MODE_HEADKV, hkv.MODE_FULL: O.MODE_FULL,
             hkv.MODE_UNIFORM: O.MODE_UNIFORM}[mode]
    stats = []
    for u in units:
        res, err = compare_unit(w, data, u, rec[u], omode, stratified, cls_queries, pairing,
                                tau)
        assert_lockstep(res, err, TOL[w.dtype], len(rec[u]["events"]), unit=(w.name,) + u)
        if mode == hkv.MODE_HEADKV:
            np.testing.assert_array_equal(res.labels, rec[u]["labels"])
        if expect_label is not None:
            assert (rec[u]["labels"] == expect_label).all(), rec[u]["labels"]
        stats.append(res.stats)
    return stats


def test_llamagen_1layer_f32_full_config():
    w = WORKLOADS["llamagen_1layer_f32"]
    stats = _lockstep(w, [(0, 0)])
    assert stats[0]["n_events"] >= 1 and stats[0]["n_select"] > 0


def test_evict_counters_match_the_events():
    """hkv_get_evict_stats: every Global head evicts once per event, scoring
    its whole cache (budget + M tokens) and moving at most M rows."""
    w = WORKLOADS["llamagen_xl"].scaled(num_seqs=2, num_layers=2)
    units = [(s, l) for s in range(2) for l in range(2)]
    cfg = hkv.config_for(w)
    data = generate(w, 31, DEV)
    cache, rec, _ = run_gpu(w, cfg, data, units)
    st = cache.evict_stats()
    heads = tokens = 0
    for (s, l) in units:
        ln, bd = cache.lens(l)
        glob = rec[(s, l)]["labels"] == 0
        n_ev = sum(1 for t, _ in rec[(s, l)]["events"] if t >= w.prefill_len)
        heads += n_ev * int(glob.sum())
        tokens += n_ev * int((bd[s][glob] + w.ste_m).sum())
    assert st["heads"] == heads and st["tokens"] == tokens, (st, heads, tokens)
    assert 0 < st["rows_moved"] <= heads * w.ste_m
    cache.reset()
    assert cache.evict_stats() == {"heads": 0, "tokens": 0, "rows_moved": 0}


@pytest.mark.parametrize("name", ["llamagen_xl", "janus_pro_1b", "janus_pro_7b_rho4",
                                  "janus_pro_7b_rho6", "janus_pro_7b_rho8", "lumina_mgpt_768"])
def test_lockstep_scaled_stacks(name):
    """Every shape of the stacks, full sequence length, few sequences/layers."""
    w = WORKLOADS[name]
    w = w.scaled(num_seqs=3 if w.max_len < 1000 else 2, num_layers=2)
    units = [(s, l) for s in range(w.num_seqs) for l in range(w.num_layers)]
    if w.max_len > 1000:
        units = units[:2]
    _lockstep(w, units, seed=11)


def test_long_sequence_large_strata():
    """A 4096-token sequence: Global caches of about 2000 tokens, so each
    eviction selects 32 of ~1900 far keys and 32 of 128 near keys (the
    block select's bins hold several keys per thread), in lock step."""
    w = WORKLOADS["lumina_mgpt_768"].scaled(
        name="long_4096", num_seqs=1, num_layers=1, num_heads=4, local_heads=2, head_dim=128,
        prefix_len=64, image_tokens=4032, prefill_image=448, row_pitch=64, local_window=64,
        rho=(1, 4), ste_m=64, near_dist=128, images=1)
    assert w.max_len == 4096
    stats = _lockstep(w, [(0, 0)], seed=41, tau=0.5)
    assert stats[0]["n_events"] >= 2


@pytest.mark.parametrize("name", ["llamagen_xl", "janus_pro_1b"])
def test_lockstep_fp32_caches(name):
    """fp32 caches at d = 64 and d = 128 (chunks of 16 and 8 rows)."""
    w = WORKLOADS[name].scaled(num_seqs=2, num_layers=1, dtype="f32")
    _lockstep(w, [(0, 0), (1, 0)], seed=12)


def test_unfused_append_attend_matches_oracle():
    w = WORKLOADS["janus_pro_1b"].scaled(num_seqs=2, num_layers=1)
    _lockstep(w, [(0, 0), (1, 0)], seed=5, fused=False)


def test_full_cache_mode_matches_oracle():
    w = WORKLOADS["janus_pro_7b_rho4"].scaled(num_seqs=2, num_layers=1)
    _lockstep(w, [(0, 0), (1, 0)], seed=6, mode=hkv.MODE_FULL)


def test_unstratified_and_uniform_variants():
    w = WORKLOADS["llamagen_xl"].scaled(num_seqs=2, num_layers=1)
    _lockstep(w, [(0, 0), (1, 0)], seed=7, stratified=False)
    _lockstep(w, [(0, 0)], seed=8, mode=hkv.MODE_UNIFORM)


@pytest.mark.parametrize("nq,pairing", [(8, hkv.CFG_UNTIED), (1, hkv.CFG_HALVES),
                                         (8, hkv.CFG_ADJACENT)])
def test_classifier_variants(nq, pairing):
    """Grouping by the last nq queries' per-distance weights, and tied
    across CFG pairs: labels and the whole unit in lock step with the
    oracle; a tied pair's two streams carry identical labels."""
    w = WORKLOADS["llamagen_xl"].scaled(num_seqs=4, num_layers=1)
    units = [(s, 0) for s in range(4)]
    cfg = hkv.config_for(w, cls_queries=nq, cfg_pairing=pairing)
    _lockstep(w, units, seed=13, cls_queries=nq, pairing=pairing)
    if pairing != hkv.CFG_UNTIED:
        data = generate(w, 13, DEV)
        cache, _, _ = run_gpu(w.scaled(image_tokens=w.prefill_image + 1), cfg, data, [])
        lab, ntau = cache.labels(0)
        for s in range(4):
            sp = O.cfg_partner(s, 4, pairing)
            np.testing.assert_array_equal(lab[s], lab[sp])
            np.testing.assert_array_equal(ntau[s], ntau[sp])


def test_head_sharded_contexts_match_unsharded_and_oracle():
    """Heads split over two contexts (as over two GPUs; the sum of their
    Local counts stands for the all-reduce): sampled units of the sharded
    run, concatenated over the shards, are in lock step with the oracle;
    every label, length and kept set equals the unsharded context's and the
    outputs agree within the bf16 tolerance; a total no shard split allows
    latches INVALID_ARG."""
    from lockstep import HeadShardedView
    w = WORKLOADS["llamagen_xl"].scaled(num_seqs=2, num_layers=2)
    S, H, P = w.num_seqs, w.num_heads, w.prefill_len
    data = generate(w, 21, DEV)
    base = hkv.config_for(w)
    shards = [range(0, 7), range(7, H)]  # unequal on purpose
    view = HeadShardedView(base, shards, DEV)
    parts = view.parts
    sl = HeadShardedView._sl
    with pytest.raises(hkv.HkvError):  # a sharded context cannot group alone
        parts[0].prefill_classify(0, *(sl(x[:, :, :P], shards[0]) for x in data[0]))
    with pytest.raises(hkv.HkvError):  # compress before label
        k0, v0 = (sl(x[:, :, :P], shards[0]) for x in data[0][1:])
        parts[0].prefill_compress(0, k0, v0, torch.zeros(S, dtype=torch.int32, device=DEV))
    units = [(s, l) for s in range(S) for l in range(w.num_layers)]
    _, rec_v, _ = run_gpu(w, base, data, units, cache=view)
    full, rec_f, _ = run_gpu(w, base, data, units)
    assert view.check()[0] == 0 and full.check()[0] == 0
    for u in units:
        # the sharded run against the oracle (budgets over all heads)
        res, err = compare_unit(w, data, u, rec_v[u])
        assert_lockstep(res, err, TOL["bf16"], len(rec_v[u]["events"]), unit=("sharded",) + u)
        np.testing.assert_array_equal(res.labels, rec_v[u]["labels"])
        # and against the unsharded context
        np.testing.assert_array_equal(rec_v[u]["labels"], rec_f[u]["labels"])
        assert [t for t, _ in rec_v[u]["events"]] == [t for t, _ in rec_f[u]["events"]]
        for (_, kv), (_, kf) in zip(rec_v[u]["events"], rec_f[u]["events"]):
            assert kv.keys() == kf.keys()
            for h in kv:
                np.testing.assert_array_equal(kv[h], kf[h])
        a, b = rec_v[u]["o"].double(), rec_f[u]["o"].double()
        assert float((a - b).abs().max() / b.abs().max()) <= TOL["bf16"]
    for l in range(w.num_layers):
        for x, y in zip(view.labels(l), full.labels(l)):
            np.testing.assert_array_equal(x, y)
        for x, y in zip(view.lens(l), full.lens(l)):
            np.testing.assert_array_equal(x, y)
        for s in range(S):
            for h in (0, 6, 7, H - 1):
                np.testing.assert_array_equal(view.kept(s, l, h), full.kept(s, l, h))
    # a Local total no split of the heads allows
    c = parts[0]
    c.reset()
    q, k, v = (sl(x[:, :, :P], shards[0]) for x in data[0])
    n = c.prefill_label(0, q, k, v)
    c.prefill_compress(0, k, v, n + (H - len(shards[0])) + 1)
    assert c.check()[0] == 1  # HKV_ERR_INVALID_ARG


@pytest.mark.parametrize("tau,kind", [(1e-6, 1), (0.999, 0)])
def test_every_head_one_kind(tau, kind):
    """tau so low that every head is Local (no Global head: nG = 0, windows
    only), or so high that every head is Global (T / H each, below the
    prefill length: an initial eviction of E > M tokens on every head, then
    the regular ones); the whole unit in lock step with the oracle."""
    w = WORKLOADS["janus_pro_1b"].scaled(num_seqs=2, num_layers=1)
    stats = _lockstep(w, [(0, 0), (1, 0)], seed=15, tau=tau, expect_label=kind)
    if kind == 0:
        assert all(st["n_events"] >= 2 for st in stats)
    else:
        assert all(st["n_events"] == 0 for st in stats)


@pytest.mark.parametrize("name,W", [("llamagen_xl", 2), ("llamagen_xl", 31), ("llamagen_xl", 33),
                                    ("janus_pro_1b", 32), ("janus_pro_1b", 33)])
def test_local_windows_around_a_chunk(name, W):
    """Every head Local (tau = 1e-9: with W = 2 the newest token's own
    weight, at least ~1e-6 here, decides) with windows of 2 tokens and of
    one 32-token chunk minus, exactly, and plus one: ring wrap-around and a
    one-row last chunk, at d = 64 and d = 128, in lock step."""
    w = WORKLOADS[name].scaled(num_seqs=2, num_layers=1, local_window=W)
    _lockstep(w, [(0, 0), (1, 0)], seed=16 + W, tau=1e-9, expect_label=1)


def test_prefill_sharded_one_rank_equals_prefill_classify():
    """dist.prefill_sharded with no process group (one rank holding every
    head): label, its own counts, compress; the same labels, lengths and
    kept sets as hkv_prefill_classify."""
    from kv_cache_compression_hkv_b200 import dist
    w = WORKLOADS["janus_pro_1b"].scaled(num_seqs=2, num_layers=1)
    P = w.prefill_len
    q, k, v = (x[:, :, :P] for x in generate(w, 23, DEV)[0])
    a = hkv.HeadKVCache(hkv.config_for(w), device=DEV)
    b = hkv.HeadKVCache(hkv.config_for(w), device=DEV)
    a.prefill_classify(0, q, k, v)
    n = dist.prefill_sharded(b, 0, q, k, v)
    la, ta = a.labels(0)
    lb, tb = b.labels(0)
    np.testing.assert_array_equal(la, lb)
    np.testing.assert_array_equal(ta, tb)
    np.testing.assert_array_equal(n.cpu().numpy(), (la == 1).sum(1))
    for x, y in zip(a.lens(0), b.lens(0)):
        np.testing.assert_array_equal(x, y)
    for s in range(2):
        for h in range(w.num_heads):
            np.testing.assert_array_equal(a.kept(s, 0, h), b.kept(s, 0, h))
    assert a.check()[0] == 0 and b.check()[0] == 0


def test_prefill_outputs_match_oracle():
    w = WORKLOADS["janus_pro_7b_rho6"].scaled(num_seqs=2, num_layers=1)
    cfg = hkv.config_for(w)
    data = generate(w, 3, DEV)
    _, _, pre = run_gpu(w.scaled(image_tokens=w.prefill_image + 1), cfg, data, [], with_prefill_out=True)
    q, k, v = data[0]
    P = w.prefill_len
    for s in range(2):
        for h in range(0, w.num_heads, 7):
            o, _ = O.causal_attention(q[s, h, :P].double().cpu().numpy(),
                                      k[s, h, :P].double().cpu().numpy(),
                                      v[s, h, :P].double().cpu().numpy())
            got = pre[0][s, h].double().cpu().numpy()
            assert np.abs(got - o).max() / np.abs(o).max() < 2e-2


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("P", [33, 65, 97, 128, 130, 192, 255, 384])
def test_prefill_shapes_against_oracle(d, P):
    """Tensor-core prefill: one or several 128-query tiles, ragged tails, the
    last r rows straddling two tiles; outputs and labels against the oracle."""
    w = WORKLOADS["janus_pro_1b"].scaled(num_seqs=2, num_layers=1, num_heads=6, local_heads=3,
                                          head_dim=d, prefix_len=1, prefill_image=P - 1,
                                          image_tokens=P + 39, local_window=min(28, P))
    cfg = hkv.config_for(w, mode=hkv.MODE_HEADKV)
    cfg.rho_num, cfg.rho_den = 1, 2
    data = generate(w, 17 + P, DEV)
    q, k, v = data[0]
    cache = hkv.HeadKVCache(cfg, device=DEV)
    out = torch.empty(2, 6, P, d, dtype=torch.bfloat16, device=DEV)
    cache.prefill_classify(0, q[:, :, :P], k[:, :, :P], v[:, :, :P], out=out)
    lab, ntau = cache.labels(0)
    assert cache.check()[0] == 0
    for s in range(2):
        for h in range(6):
            qq, kk, vv = (x[s, h, :P].double().cpu().numpy() for x in (q, k, v))
            o, p = O.causal_attention(qq, kk, vv)
            got = out[s, h].double().cpu().numpy()
            assert np.abs(got - o).max() / np.abs(o).max() < 2e-2, (s, h)
            e_nt, e_lab, cw = O.classify(p[-1], w.local_window, 0.9)
            if abs(cw - 0.9) > 1e-5:
                assert lab[s, h] == e_lab, (s, h, cw)
            if e_nt > 1 and abs(np.cumsum(p[-1][::-1])[e_nt - 2] - 0.9) > 1e-5 and \
                    abs(np.cumsum(p[-1][::-1])[e_nt - 1] - 0.9) > 1e-5:
                assert ntau[s, h] == e_nt, (s, h)


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_rescales_against_oracle(d):
    """Logits that climb about 25 (log2) per 64-key tile along the keys, so
    every row raises its reference maximum and rescales its O accumulator in
    TMEM on every tile (and at d = 128 both column groups do, with the
    second group's rows below key 32 starting from an empty maximum);
    outputs and labels against the oracle."""
    P, H = 300, 2
    w = WORKLOADS["janus_pro_1b"].scaled(num_seqs=1, num_layers=1, num_heads=H, local_heads=1,
                                          head_dim=d, prefix_len=1, prefill_image=P - 1,
                                          image_tokens=P + 39, local_window=28)
    cfg = hkv.config_for(w, mode=hkv.MODE_HEADKV)
    g = torch.Generator().manual_seed(31 + d)
    u = torch.ones(d) / d ** 0.5
    slope = 0.4 / 1.4426950408889634  # per key, natural-log units of q.k / sqrt(d)
    j = torch.arange(P, dtype=torch.float64)
    q = u + 0.05 * torch.randn(1, H, P, d, generator=g)
    k = (slope * j)[:, None] * u * d ** 0.5 + 0.05 * torch.randn(1, H, P, d, generator=g)
    v = torch.randn(1, H, P, d, generator=g)
    q, k, v = (x.to(torch.bfloat16).to(DEV).contiguous() for x in (q, k, v))
    cache = hkv.HeadKVCache(cfg, device=DEV)
    out = torch.empty(1, H, P, d, dtype=torch.bfloat16, device=DEV)
    cache.prefill_classify(0, q, k, v, out=out)
    lab, _ = cache.labels(0)
    assert cache.check()[0] == 0
    for h in range(H):
        qq, kk, vv = (x[0, h].double().cpu().numpy() for x in (q, k, v))
        o, p = O.causal_attention(qq, kk, vv)
        # the logits do climb past the threshold within every tile
        s_last = qq[-1] @ kk.T / d ** 0.5 * 1.4426950408889634
        assert s_last[63] - s_last[0] > 16 and s_last[-1] - s_last[-65] > 16
        got = out[0, h].double().cpu().numpy()
        assert np.abs(got - o).max() / np.abs(o).max() < 2e-2, h
        _, e_lab, cw = O.classify(p[-1], w.local_window, 0.9)
        if abs(cw - 0.9) > 1e-5:
            assert lab[0, h] == e_lab, (h, cw)


def test_full_size_sampled_units():
    """The bench's workload at full size and launch configuration; two
    sampled units go through the oracle in lock step."""
    w = WORKLOADS["llamagen_xl"]
    units = [(5, 0), (62, 35)]
    _lockstep(w, units, seed=2024)


def test_full_size_lumina_sampled_units():
    """The default bench workload (Lumina-mGPT-768: 16 sequences, 32
    layers) at full size and launch configuration; two sampled units go
    through the oracle in lock step."""
    w = WORKLOADS["lumina_mgpt_768"]
    _lockstep(w, [(3, 0), (12, 31)], seed=2025)


# ---------------------------------------------------------------------------
# errors: argument checks, call order, device-side status
# ---------------------------------------------------------------------------

def test_call_order_and_arguments():
    w = WORKLOADS["llamagen_1layer_f32"]
    cfg = hkv.config_for(w)
    cache = hkv.HeadKVCache(cfg, device=DEV)
    x = torch.zeros(1, 20, 64, device=DEV)
    with pytest.raises(hkv.HkvError) as e:
        cache.decode_step(0, x, x, x, x.clone())
    assert e.value.code == 2  # STATE: not classified
    with pytest.raises(hkv.HkvError) as e:
        cache.ste_evict(0, 2)
    assert e.value.code == 1
    q = torch.randn(1, 20, 300, 64, device=DEV)
    with pytest.raises(hkv.HkvError) as e:  # prefill longer than max_len
        cache.prefill_classify(0, q[:, :, :257], q[:, :, :257], q[:, :, :257])
    assert e.value.code == 1
    cache.prefill_classify(0, q[:, :, :65], q[:, :, :65], q[:, :, :65])
    with pytest.raises(hkv.HkvError) as e:
        cache.prefill_classify(0, q[:, :, :65], q[:, :, :65], q[:, :, :65])
    assert e.value.code == 2
    for t in range(65, 257):
        cache.decode_step(0, x, x, x, x.clone())
        cache.ste_evict()
    with pytest.raises(hkv.HkvError) as e:  # beyond max_len
        cache.decode_step(0, x, x, x, x.clone())
    assert e.value.code == 3
    assert cache.check()[0] == 0


def test_nan_input_latches_numeric_status():
    w = WORKLOADS["llamagen_1layer_f32"]
    cache = hkv.HeadKVCache(hkv.config_for(w), device=DEV)
    q = torch.randn(1, 20, 65, 64, device=DEV)
    cache.prefill_classify(0, q, q, q)
    x = torch.randn(1, 20, 64, device=DEV)
    bad = x.clone(); bad[0, 3, 5] = float("nan")
    cache.decode_step(0, bad, x, x, x.clone())
    rc, detail = cache.check()
    assert rc == 4 and detail % 20 == 3
    cache.clear_error()
    assert cache.check()[0] == 0
