"""The split-K decode's row split, modelled on the CPU.

dec::producer (csrc/decode_splitk.cuh) lays the eligible rows of every
(virtual) lane end to end, each non-empty lane preceded by `pad` virtual
rows, and CTA c takes [c*per, (c+1)*per).  This model walks the same way and
checks what the kernel relies on: every real row is read by exactly one CTA,
the (c0, np) a stage header carries are exactly the CTAs holding that lane
(the merge counts arrivals against np), the partial slot lane + CTA is
never shared, and no two split lanes (np > 1) share a first CTA c0 (the
arrival counter of a split lane is the workspace word indexed by c0), with
c0 below the grid size, and no CTA holds more than two split lanes (its
first and its last segment; the kernel keeps two pending counts).  The GPU parity tests check the numbers; this checks the plan
over thousands of length mixes that the GPU tests cannot afford.
"""
import random


def walk(lens, VL, G, min_rows, pad, ROWS=112):
    ext = [n + pad if n > 0 else 0 for n in lens]
    total = sum(e * VL for e in ext)
    per = max(-(-total // G), min_rows)
    cover, segs = {}, []
    for c in range(G):
        start, end = c * per, min(total, c * per + per)
        if start >= end:
            continue
        cum, b = 0, None
        for bb in range(len(lens)):
            if cum + ext[bb] * VL > start:
                b = bb
                break
            cum += ext[bb] * VL
        cum_b = cum
        off0 = start - cum_b
        vl = off0 // ext[b]
        row = off0 - vl * ext[b] - pad
        pos = start
        while pos < end:
            if row < 0:
                pos -= row
                row = 0
                if pos >= end:
                    break
            L = b * VL + vl
            SR = cum_b + vl * ext[b] + pad
            nrows = min(ROWS, lens[b] - row, end - pos)
            c0 = SR // per
            npc = (SR + lens[b] - 1) // per - c0 + 1
            for r in range(row, row + nrows):
                assert (L, r) not in cover, ("read twice", L, r)
                cover[(L, r)] = c
            if not segs or segs[-1][:2] != (c, L):
                segs.append((c, L, c0, npc, L + c))
            pos += nrows
            row += nrows
            if row == lens[b]:
                row = -pad
                vl += 1
                if vl == VL:
                    vl = 0
                    cum_b += ext[b] * VL
                    nb = next((bb for bb in range(b + 1, len(lens)) if ext[bb] > 0), None)
                    if nb is None:
                        break
                    b = nb
    return cover, segs


def check(lens, VL, G, min_rows, pad):
    cover, segs = walk(lens, VL, G, min_rows, pad)
    for b, n in enumerate(lens):
        for vl in range(VL):
            for r in range(n):
                assert (b * VL + vl, r) in cover, ("never read", b, vl, r)
    holders = {}
    for c, L, _, _, _ in segs:
        holders.setdefault(L, set()).add(c)
    for c, L, c0, npc, _ in segs:
        assert sorted(holders[L]) == list(range(c0, c0 + npc)), (L, holders[L], c0, npc)
    slots = [s[4] for s in segs]
    assert len(slots) == len(set(slots))
    assert max(s[0] for s in segs) < G
    split = {L: c0 for c, L, c0, npc, _ in segs if npc > 1}
    assert len(set(split.values())) == len(split), "two split lanes share a counter"
    assert all(0 <= c0 < G for c0 in split.values())
    per_cta = {}
    for c, L, c0, npc, _ in segs:
        if npc > 1:
            per_cta.setdefault(c, set()).add(L)
    assert all(len(v) <= 2 for v in per_cta.values())


def test_split_plan_random_length_mixes():
    rng = random.Random(7)
    for _ in range(1500):
        B = rng.randint(1, 12)
        lens = [rng.choice([0, rng.randint(1, 40), rng.randint(1, 3000)]) for _ in range(B)]
        if sum(lens) == 0:
            continue
        check(lens, rng.choice([1, 2, 4, 8]), rng.choice([1, 3, 17, 148]),
              rng.choice([1, 64, 256]), rng.choice([0, 1, 7, 128, 256]))


def test_split_plan_workload_shapes():
    check([8001] * 8, 8, 148, 256, 256)                       # the B=8 decode
    rng = random.Random(3)
    check([rng.randint(2, 8193) for _ in range(64)], 1, 148, 256, 128)   # ragged MQA
    check([4096], 8, 148, 256, 128)                           # window-4096 step
