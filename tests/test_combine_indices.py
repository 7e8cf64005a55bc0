"""Index arithmetic of the split-KV plan and the combine kernel, emulated on
the CPU for every workload (s*H from 16 to 256), several SM counts and
random batches with empty sequences.  The emulation restates the loops of
plan_range, the decode kernel's walk over its range and dec_combine_kernel
(csrc/dec_common.cuh, csrc/tc_decode64.cuh) index for index, and checks
that:
- the ranges partition the tile list, and each CTA finds its first
  sequence;
- the pieces the combine merges are exactly the partials the decode CTAs
  write (same ranges, same slots), and every sequence it does not list is
  finished by one CTA;
- every partial slot and bulk copy lies inside the workspace's partial area,
  every row formed is below s*H, every output element written lies inside
  the output, and every row of every cut sequence is written once.
The GPU tests then check the values."""
import numpy as np
import pytest

import mla_workloads as W

COMBINE_WARPS, BLOCK, SWITCH = 8, 64, 4   # rows per combine block, tile size, kSwitchTiles


class Plan:
    """plan_range's quantities for one batch: real and virtual tile starts,
    the virtual quota and the ranges' real bounds."""

    def __init__(self, seq_lens, max_blocks, ranges):
        L = np.clip(seq_lens.astype(np.int64), 0, max_blocks * BLOCK)
        self.L = L
        self.tiles = (L + BLOCK - 1) // BLOCK
        self.w = np.where(self.tiles > 0, self.tiles + SWITCH, 0)
        self.start = np.concatenate([[0], np.cumsum(self.tiles)])
        self.vstart = np.concatenate([[0], np.cumsum(self.w)])
        self.total, self.vt = int(self.start[-1]), int(self.vstart[-1])
        self.qv = (self.vt + ranges - 1) // ranges if self.vt > 0 else 1
        self.ranges = ranges

    def real(self, v):
        """The real tile a virtual position maps to (the total past the end)."""
        if v >= self.vt:
            return self.total
        b = int(np.nonzero((self.vstart[:-1] <= v) & (v < self.vstart[:-1] + self.w))[0][0])
        return int(self.start[b]) + max(0, v - int(self.vstart[b]) - SWITCH)

    def bounds(self, r):
        v_lo = r * self.qv
        return self.real(v_lo), self.real(min(v_lo + self.qv, self.vt))


def plan_range_lanes(seq_lens, max_blocks, ranges, rng, lanes=32):
    """plan_range for one CTA, lane by lane: (first tile, end tile, the
    sequence holding the first tile and its first tile, or None)."""
    B = len(seq_lens)
    per = (B + lanes - 1) // lanes
    t = [(min(max(int(x), 0), max_blocks * BLOCK) + BLOCK - 1) // BLOCK for x in seq_lens]
    w = [x + SWITCH if x > 0 else 0 for x in t]
    total, vt = sum(t), sum(w)
    qv = (vt + ranges - 1) // ranges if vt > 0 else 1
    v_lo, v_hi = rng * qv, min(rng * qv + qv, vt)
    lo, hi, first = total, total, None
    run_t = run_v = 0
    for l in range(lanes):
        for b in range(min(B, l * per), min(B, l * per + per)):
            if run_v <= v_lo < run_v + w[b]:
                lo, first = run_t + max(0, v_lo - run_v - SWITCH), (b, run_t)
            if run_v <= v_hi < run_v + w[b]:
                hi = run_t + max(0, v_hi - run_v - SWITCH)
            run_t += t[b]
            run_v += w[b]
    return lo, hi, first


def decode_pieces(p, ranges):
    """The decode kernel's walk: for every range, its segments; a segment
    that does not cover its whole sequence writes a partial into slot
    2 r (the range's first segment) or 2 r + 1 (its last).  Returns
    {b: [(r, slot)]} and the set of sequences finished whole by one range."""
    pieces, whole = {}, set()
    for r in range(ranges):
        lo, hi = p.bounds(r)
        pos, seg = lo, 0
        while pos < hi:
            b = int(np.nonzero((p.start[:-1] <= pos) & (pos < p.start[1:]))[0][0])
            a, e = int(p.start[b]), int(p.start[b + 1])
            end = min(hi, e)
            if pos == a and end == e:
                whole.add(b)
            else:
                pieces.setdefault(b, []).append((r, 2 * r + (0 if seg == 0 else 1)))
            pos, seg = end, seg + 1
    return pieces, whole


def combine_list(p):
    """plan_range's list: (b, VA_b, tiles, clamped length) of the sequences
    whose tiles span more than one range, or with no tile."""
    out = []
    for b in range(len(p.tiles)):
        va, t = int(p.vstart[b]), int(p.tiles[b])
        if t == 0 or (va + SWITCH) // p.qv != (va + SWITCH + t - 1) // p.qv:
            out.append((b, va, t, int(p.L[b])))
    return out


def combine_pieces(p, va, t):
    """The combine's ranges and slots of a listed sequence."""
    c0, c1 = (va + SWITCH) // p.qv, (va + SWITCH + t - 1) // p.qv
    slot0 = 2 * c0 + (1 if c0 * p.qv < va else 0)
    return [(c, slot0 if c == c0 else 2 * c) for c in range(c0, c1 + 1)]


def ranges_of(sms, s, H):
    """Ranges per row group, as decode_ranges picks them."""
    groups = (s * H + 63) // 64
    return max(1, min(sms // groups, 148 // groups)), groups


def workspace_slots(s, H):
    """Partial slots the workspace holds (tc_ws: 2 per range of the 64-row plan)."""
    groups = (s * H + 63) // 64
    return 2 * max(1, 148 // groups)


def emulate_combine(B, s, H, p, grid):
    """The combine's loops: CTA c takes blocks c, c + grid, ... of 8 rows of
    the listed sequences; warp w of a block takes row 8 rb + w; thread 0
    bulk-copies rows [8 rb, 8 rb + nr) of each piece's slot."""
    rows = s * H
    nbr = (rows + COMBINE_WARPS - 1) // COMBINE_WARPS
    lst = combine_list(p)
    nblk = len(lst) * nbr
    reads, writes, rows_seen, copies = [], [], set(), []
    # every CTA reads list entry cta // nbr before it knows the list's
    # length: the entry must lie in the list area (B entries)
    assert grid <= B * nbr
    for cta in range(grid):
        assert 0 <= cta // nbr < B
        for blk in range(cta, nblk, grid):
            li, rb = divmod(blk, nbr)
            b, va, t, L = lst[li]
            pcs = combine_pieces(p, va, t) if t > 0 else []
            split = len(pcs) > 1
            rr0 = rb * COMBINE_WARPS
            nr = min(COMBINE_WARPS, rows - rr0)
            if split:
                for _, slot in pcs:
                    copies.append((slot, rr0, rr0 + nr))
            for warp in range(COMBINE_WARPS):
                rr = rr0 + warp
                if warp >= nr:
                    continue
                assert rr < rows
                visible = L - s + rr // H + 1 > 0
                if not split and visible:
                    continue
                orow = b * rows + rr
                rows_seen.add((b, rr))
                writes.append((orow * 512, orow * 512 + 4 * 32 * 4))   # 4 x 32 lanes x 4 columns
                if not split or not visible:
                    continue
                for _, slot in pcs:
                    reads.append((slot, rr))
    return reads, writes, rows_seen, copies


def check_plan(seq_lens, max_blocks, ranges):
    """Ranges partition the list, each CTA finds its first sequence, and the
    combine's pieces are the decode's partials."""
    p = Plan(seq_lens, max_blocks, ranges)
    prev = 0
    for r in range(ranges):
        lo, hi = p.bounds(r)
        assert lo == prev and lo <= hi
        prev = hi
        lo2, hi2, first = plan_range_lanes(seq_lens, max_blocks, ranges, r)
        assert (lo2, hi2) == (lo, hi)
        if lo < hi:
            b, a = first
            assert p.start[b] == a <= lo < p.start[b + 1]
    assert prev == p.total
    pieces, whole = decode_pieces(p, ranges)
    listed = {b for b, _, _, _ in combine_list(p)}
    for b in range(len(seq_lens)):
        if p.tiles[b] == 0:
            assert b in listed and b not in pieces and b not in whole
        elif b in listed:
            va, t = int(p.vstart[b]), int(p.tiles[b])
            assert combine_pieces(p, va, t) == pieces[b] and len(pieces[b]) > 1
            assert all(0 <= slot < 2 * ranges for _, slot in pieces[b])
        else:
            assert b in whole and b not in pieces
    return p


@pytest.mark.parametrize("sms", [148, 132, 8, 1])
@pytest.mark.parametrize("name", ["tiny", "v2lite", "v2", "longctx", "mtp"])
def test_combine_indices_stay_in_bounds(name, sms):
    cfg = W.CONFIGS[name]
    sl = W.seq_lens_of(cfg)
    max_blocks = int((sl.max() + 63) // 64)
    ranges, groups = ranges_of(sms, cfg.s, cfg.H)
    p = check_plan(sl, max_blocks, ranges)
    grid = min(cfg.B * ((cfg.s * cfg.H + COMBINE_WARPS - 1) // COMBINE_WARPS), 3 * sms)
    reads, writes, rows_seen, copies = emulate_combine(cfg.B, cfg.s, cfg.H, p, grid)
    rows = cfg.s * cfg.H
    nslot = workspace_slots(cfg.s, cfg.H)
    for slot, rr in reads:
        assert 0 <= slot < 2 * ranges <= nslot and 0 <= rr < rows
    for slot, r0, r1 in copies:   # bulk copies stay inside the slot's rows
        assert 0 <= slot < 2 * ranges <= nslot and 0 <= r0 < r1 <= rows and r1 - r0 <= COMBINE_WARPS
    for lo, hi in writes:
        assert 0 <= lo and hi <= cfg.B * rows * 512
    # every row of every cut sequence is written exactly by one warp of one item
    pieces, _ = decode_pieces(p, ranges)
    assert rows_seen == {(b, r) for b in pieces for r in range(rows)}
    # the list fits the plan area (plan_list_off(B) + 4 B ints)
    assert len(combine_list(p)) <= cfg.B and ((cfg.B + 9) & ~3) >= 6 + cfg.B


def test_combine_rows_bound_at_sixteen_rows():
    """s*H = 16 (the V2-Lite shape): no row past 15 is formed, and the rows
    of an empty sequence are still written (zeroed)."""
    sl = np.array([4096, 4096, 100, 0], np.int32)
    p = check_plan(sl, 64, 3)
    reads, writes, rows_seen, _ = emulate_combine(4, 1, 16, p, grid=3)
    assert all(rr < 16 for _, rr in reads)
    assert max(r for _, r in rows_seen) == 15
    # the empty sequence's rows are zeroed (written) though it has no partial
    assert {(3, r) for r in range(16)} <= rows_seen


@pytest.mark.parametrize("seed", range(8))
@pytest.mark.parametrize("ranges", [1, 3, 74, 148])
def test_plan_on_random_batches(seed, ranges):
    """Random lengths, a fifth of them empty, many sequences shorter than
    one range's quota: the ranges still partition the list (some empty when
    a range falls inside a sequence's switch weight), every CTA finds its
    first sequence, and the combine's pieces are the decode's partials."""
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 300))
    sl = rng.integers(0, 3000, size=B).astype(np.int32)
    sl[rng.random(B) < 0.2] = 0
    check_plan(sl, 64, ranges)


def test_switch_weight_evens_out_the_ranges():
    """On the V2-shaped batch every range but the last carries the same load:
    its tiles plus the part of each sequence's four-tile switch weight that
    falls inside it (a range that starts two sequences gets fewer tiles)."""
    cfg = W.CONFIGS["v2"]
    sl = W.seq_lens_of(cfg)
    p = Plan(sl, 64, 74)
    tiles = []
    for r in range(73):           # the last range takes what is left
        lo, hi = p.bounds(r)
        v0, v1 = r * p.qv, (r + 1) * p.qv
        weight = sum(max(0, min(v1, int(p.vstart[b]) + SWITCH) - max(v0, int(p.vstart[b])))
                     for b in range(cfg.B) if p.tiles[b] > 0)
        assert (hi - lo) + weight == p.qv
        tiles.append(hi - lo)
    assert min(tiles) == p.qv - 2 * SWITCH and max(tiles) < p.qv
