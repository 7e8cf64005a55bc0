"""Index arithmetic of the split-KV plan and the combine kernel, emulated on
the CPU for every workload (s*H from 16 to 256) and several SM counts: every
partial slot the combine reads lies inside the workspace's partial area,
every row it forms is below s*H, every output element it writes lies inside
the output, and every row of every cut sequence is written once.  The emulation restates the loops of plan_range and
dec_combine_kernel (csrc/dec_common.cuh) index for index; the GPU tests then
check the values."""
import numpy as np
import pytest

import mla_workloads as W

COMBINE_WARPS, BLOCK = 8, 64


def plan(seq_lens, s, max_blocks, ranges, tile=64):
    L = np.clip(seq_lens.astype(np.int64), 0, max_blocks * BLOCK)
    tiles = (L + tile - 1) // tile
    start = np.concatenate([[0], np.cumsum(tiles)])
    total = int(start[-1])
    q = (total + ranges - 1) // ranges if total > 0 else 1
    return q, total, start


def ranges_of(sms, s, H):
    """Ranges per row group, as decode_ranges picks them."""
    groups = (s * H + 63) // 64
    return max(1, min(sms // groups, 148 // groups)), groups


def workspace_slots(s, H):
    """Partial slots the workspace holds (tc_ws: 2 per range of the 64-row plan)."""
    groups = (s * H + 63) // 64
    return 2 * max(1, 148 // groups)


def combine_list(seq_lens, max_blocks, q, start):
    """plan_range's list: sequences cut by a range end or with no tile, as
    (b, first tile, end tile, clamped length)."""
    out = []
    for b in range(len(seq_lens)):
        a0, a1 = int(start[b]), int(start[b + 1])
        if a1 == a0 or a0 // q != (a1 - 1) // q:
            out.append((b, a0, a1, min(max(int(seq_lens[b]), 0), max_blocks * BLOCK)))
    return out


def emulate_combine(B, s, H, seq_lens, max_blocks, q, start, grid):
    """The combine's loops: CTA c takes blocks c, c + grid, ... of 8 rows of
    the listed sequences; warp w of a block takes row 8 rb + w; thread 0
    bulk-copies rows [8 rb, 8 rb + nr) of each piece's slot."""
    rows = s * H
    nbr = (rows + COMBINE_WARPS - 1) // COMBINE_WARPS
    lst = combine_list(seq_lens, max_blocks, q, start)
    nblk = len(lst) * nbr
    reads, writes, rows_seen, copies = [], [], set(), []
    for cta in range(grid):
        for blk in range(cta, nblk, grid):
            li, rb = divmod(blk, nbr)
            b, a0, a1, L = lst[li]
            c0 = a0 // q if a1 > a0 else 0
            c1 = (a1 - 1) // q if a1 > a0 else 0
            split = a1 > a0 and c0 != c1
            rr0 = rb * COMBINE_WARPS
            nr = min(COMBINE_WARPS, rows - rr0)
            if split:
                for c in range(c0, c1 + 1):
                    slot = 2 * c + (1 if (c == c0 and a0 != c * q) else 0)
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
                for c in range(c0, c1 + 1):
                    slot = 2 * c + (1 if (c == c0 and a0 != c * q) else 0)
                    reads.append((slot, rr))
    return reads, writes, rows_seen, copies


@pytest.mark.parametrize("sms", [148, 132, 8, 1])
@pytest.mark.parametrize("name", ["tiny", "v2lite", "v2", "longctx", "mtp"])
def test_combine_indices_stay_in_bounds(name, sms):
    cfg = W.CONFIGS[name]
    sl = W.seq_lens_of(cfg)
    max_blocks = int((sl.max() + 63) // 64)
    ranges, groups = ranges_of(sms, cfg.s, cfg.H)
    q, total, start = plan(sl, cfg.s, max_blocks, ranges)
    assert q * ranges >= total                      # every tile lies in some range
    grid = min(cfg.B * ((cfg.s * cfg.H + COMBINE_WARPS - 1) // COMBINE_WARPS), 3 * sms)
    reads, writes, rows_seen, copies = emulate_combine(cfg.B, cfg.s, cfg.H, sl, max_blocks, q, start, grid)
    rows = cfg.s * cfg.H
    nslot = workspace_slots(cfg.s, cfg.H)
    for slot, rr in reads:
        assert 0 <= slot < 2 * ranges <= nslot and 0 <= rr < rows
    for slot, r0, r1 in copies:   # bulk copies stay inside the slot's rows
        assert 0 <= slot < 2 * ranges <= nslot and 0 <= r0 < r1 <= rows and r1 - r0 <= COMBINE_WARPS
    for lo, hi in writes:
        assert 0 <= lo and hi <= cfg.B * rows * 512
    # every row of every cut sequence is written exactly by one warp of one item
    cut = [b for b in range(cfg.B) if start[b + 1] > start[b] and start[b] // q != (start[b + 1] - 1) // q]
    assert rows_seen == {(b, r) for b in cut for r in range(rows)}
    # the list fits the plan area (plan_list_off(B) + 4 B ints) and every listed
    # sequence is cut or empty
    lst = combine_list(sl, max_blocks, q, start)
    assert len(lst) <= cfg.B and ((cfg.B + 9) & ~3) % 4 == 0 and (cfg.B + 9) & ~3 >= 6 + cfg.B


def test_combine_rows_bound_at_sixteen_rows():
    """s*H = 16 (the V2-Lite shape): no row past 15 is formed, and the rows
    of an empty sequence are still written (zeroed)."""
    sl = np.array([4096, 4096, 100, 0], np.int32)
    q, total, start = plan(sl, 1, 64, ranges=3)
    reads, writes, rows_seen, _ = emulate_combine(4, 1, 16, sl, 64, q, start, grid=3)
    assert all(rr < 16 for _, rr in reads)
    assert max(r for _, r in rows_seen) == 15
    # the empty sequence's rows are zeroed (written) though it has no partial
    assert {(3, r) for r in range(16)} <= rows_seen


def range_start(seq_lens, ranges, rng, max_blocks=64, lanes=32):
    """plan_range for one CTA: lane l sums the tiles of sequences
    [l per, (l+1) per), a scan over lanes gives each lane's first tile, and
    the lane whose chunk holds tile rng*q names the sequence and its start."""
    B = len(seq_lens)
    per = (B + lanes - 1) // lanes
    tiles = [(min(max(int(L), 0), max_blocks * 64) + 63) // 64 for L in seq_lens]
    sums = [sum(tiles[min(B, l * per):min(B, l * per + per)]) for l in range(lanes)]
    total = sum(sums)
    q = (total + ranges - 1) // ranges if total > 0 else 1
    lo, found, run = rng * q, [], 0
    for l in range(lanes):
        for b in range(min(B, l * per), min(B, l * per + per)):
            if run <= lo < run + tiles[b]:
                found.append((b, run))
            run += tiles[b]
    return q, total, found


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("ranges", [1, 3, 74, 148])
def test_range_start_matches_the_search(seed, ranges):
    """Each CTA's first sequence (plan_range) is the largest b with
    start[b] <= lo, empty sequences included; exactly one lane finds it when
    the range has work, none when it has not."""
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 300))
    sl = rng.integers(0, 3000, size=B).astype(np.int32)
    sl[rng.random(B) < 0.2] = 0
    q, total, start = plan(sl, 1, 64, ranges)
    for r in range(ranges):
        q2, total2, found = range_start(sl, ranges, r)
        assert (q2, total2) == (q, total)
        lo = r * q
        if lo >= total:
            assert found == []
            continue
        want = int(np.nonzero(start <= lo)[0].max())   # largest index with start <= lo
        assert found == [(want, int(start[want]))] and start[want] <= lo < start[want + 1]
