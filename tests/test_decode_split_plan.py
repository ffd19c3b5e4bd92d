"""The split-K decode's row split, modelled on the CPU.

dec::producer (csrc/decode_splitk.cuh) lays the eligible rows of every
(virtual) lane end to end, each non-empty lane preceded by `pad` virtual
rows, and CTA c takes [c*per, (c+1)*per).  This model walks the same way and
checks what the kernel relies on: every real row is read by exactly one CTA,
the (c0, np) a stage header carries are exactly the CTAs holding that lane
(the merge counts arrivals against np), the partial slot lane + CTA is
never shared, and no two split lanes (np > 1) share a first piece c0 (the
arrival counter of a split lane is the workspace word indexed by c0), and
no range holds more than two split lanes (its first and its last segment;
the kernel lists two pending counts per range).  On large calls the last
1/16 of the rows is cut into chunks that CTAs take as they finish; chunk k
is piece G + k, and the same checks hold over the static ranges and the
chunks together (the order in which CTAs take chunks does not matter: a
chunk's rows, slot and counts depend only on k).  The GPU parity tests check the numbers; this checks the plan
over thousands of length mixes that the GPU tests cannot afford.
"""
import random


MAX_TAIL, MAX_GRABS, TAIL_MIN_STAGES = 256, 15, 16


def plan(lens, VL, G, min_rows, pad, tail_div, ROWS=112):
    """The kernel's split (Split in decode_splitk.cuh): static part [0, S)
    in equal CTA ranges, then nch tail chunks of ch rows (pieces G + k)."""
    ext = [n + pad if n > 0 else 0 for n in lens]
    total = sum(e * VL for e in ext)
    S, ch, nch = total, 1, 0
    if tail_div > 0 and total >= G * TAIL_MIN_STAGES * ROWS:
        tail = total // tail_div
        maxch = min(MAX_TAIL, G * MAX_GRABS)
        ch = 2 * ROWS
        if tail > ch * maxch:
            ch = ((tail + maxch - 1) // maxch + ROWS - 1) // ROWS * ROWS
        nch = -(-tail // ch)
        S = total - tail
    per = max(-(-S // G), min_rows)
    return ext, total, S, per, ch, nch


def pieces_of(SR, SE, S, per, G, ch):
    """(c0, np) of a lane's real rows [SR, SE), as Split::pieces."""
    nstat = 0
    if SR < S:
        c0 = SR // per
        nstat = (min(SE, S) - 1) // per - c0 + 1
    else:
        c0 = G + (SR - S) // ch
    ntail = ((SE - 1 - S) // ch - (max(SR, S) - S) // ch + 1) if SE > S else 0
    return c0, nstat + ntail


def walk(lens, VL, G, min_rows, pad, tail_div=0, ROWS=112):
    ext, total, S, per, ch, nch = plan(lens, VL, G, min_rows, pad, tail_div, ROWS)
    assert nch <= min(MAX_TAIL, G * MAX_GRABS)
    ranges = [(c, c * per, min(S, c * per + per)) for c in range(G)]
    ranges += [(G + k, S + k * ch, min(total, S + (k + 1) * ch)) for k in range(nch)]
    cover, segs = {}, []
    for vid, start, end in ranges:
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
            c0, npc = pieces_of(SR, SR + lens[b], S, per, G, ch)
            for r in range(row, row + nrows):
                assert (L, r) not in cover, ("read twice", L, r)
                cover[(L, r)] = vid
            if not segs or segs[-1][:2] != (vid, L):
                segs.append((vid, L, c0, npc, L + vid))
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
    return cover, segs, G + nch


def check(lens, VL, G, min_rows, pad, tail_div=0):
    cover, segs, npieces = walk(lens, VL, G, min_rows, pad, tail_div)
    for b, n in enumerate(lens):
        for vl in range(VL):
            for r in range(n):
                assert (b * VL + vl, r) in cover, ("never read", b, vl, r)
    holders = {}
    for vid, L, _, _, _ in segs:
        holders.setdefault(L, []).append(vid)
    for vid, L, c0, npc, _ in segs:
        assert holders[L][0] == c0 and len(holders[L]) == npc, (L, holders[L], c0, npc)
    slots = [s[4] for s in segs]
    assert len(slots) == len(set(slots))
    assert max(s[0] for s in segs) < npieces <= MAX_TAIL + 1024
    split = {L: c0 for vid, L, c0, npc, _ in segs if npc > 1}
    assert len(set(split.values())) == len(split), "two split lanes share a counter"
    assert all(0 <= c0 < npieces for c0 in split.values())
    per_piece = {}
    for vid, L, c0, npc, _ in segs:
        if npc > 1:
            per_piece.setdefault(vid, set()).add(L)
    assert all(len(v) <= 2 for v in per_piece.values())


def test_split_plan_random_length_mixes():
    rng = random.Random(7)
    for _ in range(1500):
        B = rng.randint(1, 12)
        lens = [rng.choice([0, rng.randint(1, 40), rng.randint(1, 3000)]) for _ in range(B)]
        if sum(lens) == 0:
            continue
        check(lens, rng.choice([1, 2, 4, 8]), rng.choice([1, 3, 17, 148]),
              rng.choice([1, 64, 256]), rng.choice([0, 1, 7, 128, 256]),
              rng.choice([0, 16, 16, 4]))


def test_split_plan_with_a_tail_on_small_grids():
    """Small grids reach the tail with few rows: many chunks, the chunk size
    grown so that at most min(256, 15 G) chunks exist."""
    rng = random.Random(11)
    for _ in range(300):
        B = rng.randint(1, 6)
        lens = [rng.randint(1, 9000) for _ in range(B)]
        check(lens, rng.choice([1, 2, 8]), rng.choice([1, 2, 5]), 64, 0, rng.choice([2, 4, 16]))


def test_split_plan_workload_shapes():
    check([8001] * 8, 8, 148, 256, 256, 16)                   # the B=8 decode
    rng = random.Random(3)
    check([rng.randint(2, 8193) for _ in range(64)], 1, 148, 256, 128, 16)   # ragged MQA
    check([rng.randint(2, 8193) for _ in range(64)], 8, 148, 256, 128, 16)   # ragged MHA
    check([4096], 8, 148, 256, 128, 16)                       # window-4096 step (no tail)
