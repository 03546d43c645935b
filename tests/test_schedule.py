"""The backward kernel's work-item numbering, replayed on the host.

The fused backward kernel numbers its items -- (key tile, head) pairs of a
key window [kt_lo, kt_hi) -- so that heads come in groups of hg, key tiles
ascend within a group and the group's heads interleave (the decode at the top
of ``bwd_kernel`` in io_aware_exact_25_b200/csrc/bwd_sm100.cuh).  CTAs take
item numbers 0 .. n_items-1 from a counter (or by block index), so the
decode must be a bijection onto the window's (key tile, head) pairs for
every problem shape, window and SM count, or a key tile's dK, dV would be
computed twice or never.  This test restates the decode from that rule and
checks the bijection and the order it promises over a wide sweep.
"""
import itertools


def decode_all(BH, nT, kt_lo, kt_hi, n_sm, causal):
    kt_hi = min(kt_hi, nT)
    kt_lo = min(kt_lo, kt_hi)
    nTr = kt_hi - kt_lo
    n_items = BH * nTr
    avg_len = max(1, nT - (kt_lo + kt_hi - 1) // 2 if causal else nT)
    hg = min(BH, max(1, (n_sm + avg_len - 1) // avg_len))
    n_groups = max(1, BH // hg)
    out = []
    for w in range(n_items):
        grp = min(w // (hg * nTr), n_groups - 1)
        h0 = grp * hg
        nh = BH - h0 if grp == n_groups - 1 else hg
        r = w - h0 * nTr
        jl = r // nh
        out.append((kt_lo + jl, h0 + (r - jl * nh), grp))
    return out, hg


def test_decode_is_a_bijection_onto_the_window():
    for BH, nT, n_sm, causal in itertools.product((1, 2, 3, 7, 16, 32, 37, 128), (1, 2, 3, 16, 64, 65, 512),
                                                  (1, 8, 132, 148), (False, True)):
        windows = {(0, nT), (0, 1 << 30)}
        for a in (0, 1, nT // 3, nT - 1):
            for b in (a + 1, nT // 2 + 1, nT):
                if 0 <= a < b <= nT:
                    windows.add((a, b))
        for kt_lo, kt_hi in windows:
            items, _ = decode_all(BH, nT, kt_lo, kt_hi, n_sm, causal)
            hi = min(kt_hi, nT)
            want = {(j, h) for j in range(kt_lo, hi) for h in range(BH)}
            got = [(j, h) for j, h, _ in items]
            assert len(got) == len(want) and set(got) == want, (BH, nT, n_sm, causal, kt_lo, kt_hi)


def test_order_groups_heads_and_ascends_key_tiles():
    BH, nT, n_sm = 32, 64, 148
    items, hg = decode_all(BH, nT, 0, nT, n_sm, True)
    assert hg == 5  # ceil(148 / average causal length 32.5 query tiles)
    for (j0, h0, g0), (j1, h1, g1) in zip(items, items[1:]):
        assert g1 >= g0  # groups one after another
        if g1 == g0:
            assert j1 >= j0  # key tiles ascend within a group: longest causal items first
    # every group's heads are consecutive, and the last one takes the rest
    groups = {}
    for j, h, g in items:
        groups.setdefault(g, set()).add(h)
    sizes = [len(groups[g]) for g in sorted(groups)]
    assert all(s == hg for s in sizes[:-1]) and sizes[-1] == BH - hg * (len(sizes) - 1) >= hg
