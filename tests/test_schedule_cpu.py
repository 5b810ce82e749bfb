"""The forward kernel's work list, checked on the CPU through a step-by-step twin
of its device code (build_varlen_tables and Sched::decode in
csrc/attn_fwd_sm100.cu): for dense and packed batches, every (sequence, head,
128-row sub-tile) is covered by exactly one list position, the list is ordered as
the scheduler intends (groups together in the bulk, a longest-first tail), and
the dense non-causal last-wave split covers the same rows as the unsplit list.

The twin mirrors the integer steps of the device code, so a change there must be
mirrored here; the coverage property is what the kernel relies on (each output
row written once)."""
import math
import random

import pytest

import attn_inputs as ai

BM = 128  # query rows per sub-tile


def ceil_div(a, b):
    return (a + b - 1) // b


def build_varlen_tables(cu, B, H, T, total, tail_items, ishift=8):
    """Twin of build_varlen_tables: returns (order, gstart, tstart, items, gtail, nbulk)
    or None for an invalid cu_seqlens (items of 2^ishift query rows)."""
    if cu[0] != 0 or cu[B] != total:
        return None
    nts = []
    for b in range(B):
        L = cu[b + 1] - cu[b]
        nt = 0 if L < 0 else ceil_div(L, 1 << ishift)
        if L < 0 or nt > T:
            return None
        nts.append(nt)
    hist = [0] * (T + 1)
    for nt in nts:
        hist[nt] += 1
    off = [0] * (T + 1)  # off[n] = #{b : nt_b > n}
    for n in range(T + 1):
        off[n] = sum(hist[n + 1:])
    cnt = list(off)
    order = [0] * B
    for b in range(B):  # stable placement, descending nt
        key = nts[b]
        order[off[key]] = b
        off[key] += 1
    gstart = [0] * (B + 1)
    for i in range(B):
        gstart[i + 1] = gstart[i] + H * nts[order[i]]
    items = gstart[B]
    i0 = h0 = 0
    if items > tail_items:
        i0 = max(i for i in range(B) if gstart[i] <= items - tail_items)
        Ti = (gstart[i0 + 1] - gstart[i0]) // H
        rest = items - gstart[i0 + 1]
        h0 = max(0, H - ceil_div(tail_items - rest, Ti))
    Ti0 = (gstart[i0 + 1] - gstart[i0]) // H
    tstart = [0] * T
    acc = 0
    for t in range(T - 1, -1, -1):
        tstart[t] = acc
        later = cnt[t] - (i0 + 1)
        acc += H * max(later, 0) + (H - h0 if Ti0 > t else 0)
    return order, gstart, tstart, items, i0 * H + h0, gstart[i0] + h0 * Ti0


class Sched:
    """Twin of the kernel's Sched (list parameters and decode)."""

    def __init__(self, B, H, N, grid, cu=None, split_ok=False, pair=False):
        self.B, self.H, self.N, self.cu = B, H, N, cu
        self.ishift = 9 if pair else 8  # CTA pairs: items of 512 rows
        self.T = ceil_div(N, 1 << self.ishift)
        claimers = grid // 2 if pair else grid
        tail_items = 2 * claimers
        grid = claimers
        if cu is None:
            groups = B * H
            k = min(ceil_div(tail_items, self.T), groups)
            self.pairs = groups * self.T
            self.gtail = groups - k
            self.nbulk = self.gtail * self.T
        else:
            r = build_varlen_tables(cu, B, H, self.T, cu[B], tail_items, self.ishift)
            assert r is not None
            self.order, self.gstart, self.tstart, self.pairs, self.gtail, self.nbulk = r
        self.split = 0
        if split_ok and cu is None and not pair:
            rem = self.pairs % grid
            if rem > 0 and 2 * rem <= grid:
                self.split = rem
        self.count = self.pairs + self.split

    def seq(self, i):
        if self.cu is None:
            return i, i * self.N, self.N, self.T
        b = self.order[i]
        L = self.cu[b + 1] - self.cu[b]
        return b, self.cu[b], L, ceil_div(L, 1 << self.ishift)

    def decode(self, idx):
        """(b, h, row_base, two, t) of list position idx."""
        sub = -1
        if self.split and idx >= self.pairs - self.split:
            u = idx - (self.pairs - self.split)
            idx = self.pairs - self.split + (u >> 1)
            sub = u & 1
        H = self.H
        if idx < self.nbulk:
            if self.cu is None:
                g = idx // self.T
                t = self.T - 1 - (idx - g * self.T)
            else:
                lo, hi = 0, self.B - 1
                while lo < hi:
                    mid = (lo + hi + 1) >> 1
                    if self.gstart[mid] <= idx:
                        lo = mid
                    else:
                        hi = mid - 1
                Ti = self.seq(lo)[3]
                r = idx - self.gstart[lo]
                hh = r // Ti
                g = lo * H + hh
                t = Ti - 1 - (r - hh * Ti)
        else:
            u = idx - self.nbulk
            if self.cu is None:
                k = self.B * H - self.gtail
                lev = u // k
                t = self.T - 1 - lev
                g = self.gtail + (u - lev * k)
            else:
                lo, hi = 0, self.T - 1
                while lo < hi:
                    mid = (lo + hi) >> 1
                    if self.tstart[mid] <= u:
                        hi = mid
                    else:
                        lo = mid + 1
                t = lo
                g = self.gtail + (u - self.tstart[lo])
        i = g // H
        h = g - i * H
        b, _, L, _ = self.seq(i)
        row_base = (t << self.ishift) + (BM if (sub > 0) else 0)
        two = sub < 0
        return b, h, row_base, two, t


def _coverage(s, lengths):
    seen = {}
    blocks = (1 << s.ishift) // (2 * BM)  # 128-row blocks of a sub-tile (a pair: one per CTA)
    for idx in range(s.count):
        b, h, row_base, two, _ = s.decode(idx)
        L = lengths[b]
        for st in ((0, 1) if two else (0,)):
            for blk in range(blocks):
                row0 = row_base + (st * blocks + blk) * BM
                if row0 < L:  # rows past the sequence end are not stored
                    key = (b, h, row0)
                    seen[key] = seen.get(key, 0) + 1
    expected = {(b, h, r) for b, L in enumerate(lengths) for h in range(s.H)
                for r in range(0, L, BM)}
    assert set(seen) == expected, (len(set(seen)), len(expected))
    assert all(v == 1 for v in seen.values()), [k for k, v in seen.items() if v != 1][:5]


def _cu(lengths):
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + L)
    return cu


@pytest.mark.parametrize("B,H,N,grid", [(4, 16, 2048, 148), (2, 16, 8192, 148), (1, 1, 256, 1),
                                        (3, 5, 1000, 148), (2, 3, 300, 7), (1, 2, 513, 148),
                                        (7, 1, 129, 3)])
@pytest.mark.parametrize("split_ok", [False, True])
def test_dense_list_covers_every_subtile_once(B, H, N, grid, split_ok):
    s = Sched(B, H, N, grid, split_ok=split_ok)
    _coverage(s, [N] * B)


@pytest.mark.parametrize("grid", [148, 1, 5])
def test_varlen_workload_list_covers_every_subtile_once(grid):
    w = ai.VARLEN
    s = Sched(w.B, w.H, w.N, grid, cu=w.cu_seqlens())
    _coverage(s, w.seq_lengths())


def test_random_varlen_lists_cover_every_subtile_once():
    rng = random.Random(11)
    for _ in range(60):
        B = rng.choice([1, 2, 3, 16, 40, 200])
        lengths = [rng.choice([0, 1, 127, 128, 129, 255, 256, 257]) if rng.random() < 0.3
                   else rng.randint(0, 5000) for _ in range(B)]
        H = rng.choice([1, 2, 3, 16])
        N = max(max(lengths), 1)
        grid = rng.choice([1, 2, 7, 148])
        s = Sched(B, H, N, grid, cu=_cu(lengths))
        _coverage(s, lengths)


def test_list_order_groups_then_longest_first_tail():
    """Bulk positions keep each (sequence, head) together with t descending; the
    tail visits t in non-increasing order; the tail holds >= 2 items per CTA."""
    w = ai.VARLEN
    grid = 148
    s = Sched(w.B, w.H, w.N, grid, cu=w.cu_seqlens())
    dec = [s.decode(i) for i in range(s.count)]
    bulk, tail = dec[:s.nbulk], dec[s.nbulk:]
    assert len(tail) >= 2 * grid
    groups_seen, prev = [], None
    for b, h, _, _, t in bulk:
        if (b, h) != prev:
            assert (b, h) not in groups_seen, "a group's items are split in the bulk"
            groups_seen.append((b, h))
            prev = (b, h)
    ts = [t for *_, t in tail]
    assert all(a >= c for a, c in zip(ts, ts[1:])), "tail not longest-first"
    # sequences appear longest first
    lens = [w.seq_lengths()[b] for b, _ in groups_seen]
    assert [math.ceil(L / 256) for L in lens] == sorted((math.ceil(L / 256) for L in lens),
                                                         reverse=True)


def test_invalid_cu_seqlens_rejected():
    assert build_varlen_tables([0, 5, 3], 2, 1, 1, 3, 4) is None  # negative length
    assert build_varlen_tables([1, 5, 9], 2, 1, 1, 9, 4) is None  # cu[0] != 0
    assert build_varlen_tables([0, 5, 9], 2, 1, 1, 10, 4) is None  # cu[B] != total
    assert build_varlen_tables([0, 600], 1, 1, 2, 600, 4) is None  # longer than T*256


@pytest.mark.parametrize("grid", [148, 144, 2])
def test_pair_lists_cover_every_block_once(grid):
    """CTA pairs (items of 512 rows, claimed by one CTA of each pair): the dense and
    packed benchmark workloads and random packed batches."""
    _coverage(Sched(2, 16, 8192, grid, pair=True), [8192] * 2)
    _coverage(Sched(4, 16, 2048, grid, pair=True), [2048] * 4)
    _coverage(Sched(3, 5, 700, grid, pair=True), [700] * 3)
    w = ai.VARLEN
    _coverage(Sched(w.B, w.H, w.N, grid, cu=w.cu_seqlens(), pair=True), w.seq_lengths())
    rng = random.Random(12)
    for _ in range(20):
        lengths = [rng.randint(0, 3000) for _ in range(rng.choice([1, 4, 30]))]
        _coverage(Sched(len(lengths), 3, max(max(lengths), 1), grid, cu=_cu(lengths), pair=True), lengths)


def bwd_decode(idx, nbh, ntiles, group):
    """Twin of the backward's block order (decode_block in csrc/attn_bwd_sm100.cu):
    blocks dealt in groups of `group` (sequence, head) pairs, by rank inside a group.
    Returns (bh, rank)."""
    G = min(nbh, group)
    grp = idx // (G * ntiles)
    gsize = min(G, nbh - grp * G)
    rem = idx - grp * G * ntiles
    rank = rem // gsize
    return grp * G + (rem - rank * gsize), rank


@pytest.mark.parametrize("nbh,ntiles", [(32, 64), (1, 1), (3, 5), (17, 9), (8, 64), (40, 3)])
@pytest.mark.parametrize("group", [1, 4, 8, 16, 64])
def test_bwd_block_order_is_a_bijection(nbh, ntiles, group):
    """Every (sequence-head pair, tile rank) is dealt to exactly one block of the
    nbh * ntiles grid; inside a group ranks do not decrease (longest work first);
    the blocks running together span at most `group` pairs per rank sweep."""
    seen = {}
    prev = None
    for idx in range(nbh * ntiles):
        bh, rank = bwd_decode(idx, nbh, ntiles, group)
        assert 0 <= bh < nbh and 0 <= rank < ntiles
        seen[(bh, rank)] = seen.get((bh, rank), 0) + 1
        grp = bh // min(nbh, group)
        if prev is not None and prev[0] == grp:
            assert rank >= prev[1]
        prev = (grp, rank)
    assert len(seen) == nbh * ntiles and all(v == 1 for v in seen.values())
