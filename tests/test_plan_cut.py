"""The decode plan's range cutting, restated in Python: the arithmetic by
which plan_kernel (csrc/decode.cu) turns the heads' cost intervals into
warp starts, with equal shares (cut_ranges) and with per-warp weights
(cut_ranges_weighted).  Checked on random layers: every warp gets exactly
one start, the starts never go backwards, and equal weights reproduce the
equal shares.  (The GPU lock-step tests run the kernel itself.)"""
import random

CHUNK_COST = 3


def cut_equal(cnt, head_cost, tcost, gw):
    starts = {}
    for i in range(len(cnt)):
        c0, c1 = (cnt[i - 1] if i else 0), cnt[i]
        e0 = CHUNK_COST * c0 + head_cost * i
        e1 = CHUNK_COST * c1 + head_cost * (i + 1)
        w_lo = (e0 * gw + tcost - 1) // tcost
        w_hi = min((e1 * gw + tcost - 1) // tcost, gw)
        for w in range(w_lo, w_hi):
            bnd = w * tcost // gw
            k = (bnd - e0 + CHUNK_COST - 1) // CHUNK_COST if bnd > e0 else 0
            assert w not in starts
            starts[w] = c0 + min(k, c1 - c0)
    return starts


def cut_weighted(cnt, head_cost, tcost, gw, nw, pre):
    s_blk = pre[nw]
    units = (gw // nw) * s_blk
    starts = {}
    for i in range(len(cnt)):
        c0, c1 = (cnt[i - 1] if i else 0), cnt[i]
        e0 = CHUNK_COST * c0 + head_cost * i
        e1 = CHUNK_COST * c1 + head_cost * (i + 1)
        x_lo = (e0 * units + tcost - 1) // tcost
        x_hi = min((e1 * units + tcost - 1) // tcost, units)
        if x_lo >= x_hi:
            continue
        b, r, k = x_lo // s_blk, x_lo % s_blk, 0
        while k < nw and pre[k] < r:
            k += 1
        if k == nw:
            b, k = b + 1, 0
        while b * s_blk + pre[k] < x_hi:
            u = b * s_blk + pre[k]
            w = b * nw + k
            bnd = u * tcost // units
            kk = (bnd - e0 + CHUNK_COST - 1) // CHUNK_COST if bnd > e0 else 0
            assert w not in starts
            starts[w] = c0 + min(kk, c1 - c0)
            k += 1
            if k == nw:
                b, k = b + 1, 0
    return starts


def sub_partition_prefix(nw, lone, shared=11):
    per = [0] * 4
    for k in range(nw):
        per[k & 3] += 1
    top = max(per)
    pre = [0]
    for k in range(nw):
        pre.append(pre[-1] + (lone if per[k & 3] < top else shared))
    return pre


def test_weighted_cut_gives_every_warp_one_start():
    rng = random.Random(7)
    for _ in range(200):
        n = rng.randint(1, 400)
        cnt, s = [], 0
        for _ in range(n):
            s += rng.choice([0, 1, 2, 2, 3, 5, 10, 25])
            cnt.append(s)
        head_cost = rng.choice([1, 5, 8])
        tcost = CHUNK_COST * cnt[-1] + head_cost * n
        nw = rng.choice([3, 5, 6, 12])
        gw = nw * rng.randint(1, 148)
        for lone in (11, 12, 13):
            pre = sub_partition_prefix(nw, lone)
            starts = cut_weighted(cnt, head_cost, tcost, gw, nw, pre)
            assert sorted(starts) == list(range(gw))
            seq = [starts[w] for w in range(gw)]
            assert all(a <= b for a, b in zip(seq, seq[1:]))
            assert seq[0] == 0
            if lone == 11:
                assert starts == cut_equal(cnt, head_cost, tcost, gw)


def test_six_warp_blocks_weigh_the_lone_warps():
    # six warps: sub-partitions 0 and 1 hold two each, 2 and 3 one each
    assert sub_partition_prefix(6, 13) == [0, 11, 22, 35, 48, 59, 70]
    # twelve warps spread evenly: every weight is the shared one
    assert sub_partition_prefix(12, 13) == [11 * k for k in range(13)]
