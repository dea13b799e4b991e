"""The stream-K partition of the decode kernels, modelled in plain Python.

fa_decode_fwd cuts the list of (batch entry, head, 64-key tile) units into G
equal contiguous chunks, one per CTA; a CTA writes a segment it holds whole
directly and a shared segment's pieces as partial records in one of two
slots (its first piece in slot 0, its last in slot 1); the merge kernel
finds the records of a shared segment from the segment's unit range alone.
This model restates those rules and checks, over many random length mixes
and grid sizes, that every tile is covered exactly once, that whole pieces
are exactly the segments one CTA holds, that no CTA writes a slot twice and
that the records the merge reads are exactly the records written."""
import random

import pytest


def tiles(L):
    return (L + 63) // 64


def partition(lengths, H, G):
    """Pieces per CTA, as the stream kernel walks them: (g, b, h, t0, n, whole, slot)."""
    prefix = [0]
    for L in lengths:
        prefix.append(prefix[-1] + H * tiles(L))
    U = prefix[-1]
    chunk = -(-U // G) if U else 0
    pieces = []
    for g in range(G):
        u0, u1 = g * chunk, min(U, (g + 1) * chunk)
        if u0 >= u1:
            continue
        b = max(i for i in range(len(lengths)) if prefix[i] <= u0)
        while prefix[b + 1] == prefix[b]:
            b += 1
        T = tiles(lengths[b])
        rel = u0 - prefix[b]
        h, tp = rel // T, rel % T
        u = u0
        while u < u1:
            n = min(T - tp, u1 - u)
            pieces.append((g, b, h, tp, n, tp == 0 and n == T, 0 if u == u0 else 1))
            u += n
            tp += n
            if tp == T and u < u1:
                tp = 0
                h += 1
                if h == H:
                    h = 0
                    b += 1
                    while prefix[b + 1] == prefix[b]:
                        b += 1
                    T = tiles(lengths[b])
    return prefix, U, chunk, pieces


def merge_reads(lengths, H, G, prefix, chunk):
    """(b, h) -> list of (g, slot) records the merge combines; None for a
    segment written whole by one CTA; [] for a segment without keys."""
    out = {}
    for b, L in enumerate(lengths):
        T = tiles(L)
        for h in range(H):
            if T == 0:
                out[(b, h)] = []
                continue
            s0 = prefix[b] + h * T
            s1 = s0 + T
            g0, g1 = s0 // chunk, (s1 - 1) // chunk
            if g0 == g1:
                out[(b, h)] = None
                continue
            out[(b, h)] = [(g0 + k, 1 if (k == 0 and g0 * chunk < s0) else 0) for k in range(g1 - g0 + 1)]
    return out


def check(lengths, H, G):
    prefix, U, chunk, pieces = partition(lengths, H, G)
    covered = {}
    written_slots = set()
    whole = set()
    records = {}
    for g, b, h, t0, n, is_whole, slot in pieces:
        for t in range(t0, t0 + n):
            assert (b, h, t) not in covered
            covered[(b, h, t)] = g
        if is_whole:
            whole.add((b, h))
        else:
            assert (g, slot) not in written_slots, "a CTA wrote one slot twice"
            written_slots.add((g, slot))
            records.setdefault((b, h), []).append((g, slot))
    # every tile exactly once
    for b, L in enumerate(lengths):
        for h in range(H):
            for t in range(tiles(L)):
                assert (b, h, t) in covered
    assert len(covered) == U
    # at most two records per CTA
    per_cta = {}
    for g, _ in written_slots:
        per_cta[g] = per_cta.get(g, 0) + 1
    assert all(c <= 2 for c in per_cta.values())
    # the merge reads exactly what was written
    reads = merge_reads(lengths, H, G, prefix, chunk)
    for key, r in reads.items():
        if r is None:
            assert key in whole and key not in records
        elif r == []:
            assert key not in whole and key not in records
        else:
            assert key not in whole
            assert sorted(r) == sorted(records[key]), (key, r, records.get(key))


@pytest.mark.parametrize("seed", range(200))
def test_partition_covers_every_tile_once_and_merge_reads_what_was_written(seed):
    rnd = random.Random(seed)
    B = rnd.randint(1, 40)
    H = rnd.randint(1, 8)
    mode = seed % 4
    if mode == 0:  # serving-style ragged
        lengths = [rnd.randint(0, 5000) for _ in range(B)]
    elif mode == 1:  # many empty and tiny sequences
        lengths = [rnd.choice([0, 0, 1, 63, 64, 65, rnd.randint(0, 300)]) for _ in range(B)]
    elif mode == 2:  # all full
        L = rnd.randint(1, 20000)
        lengths = [L] * B
    else:  # one long, the rest short
        lengths = [rnd.randint(0, 200) for _ in range(B)]
        lengths[rnd.randrange(B)] = rnd.randint(5000, 60000)
    if sum(lengths) == 0:
        lengths[0] = 1
    for G in (1, 3, 7, 296, rnd.randint(1, 1000)):
        check(lengths, H, G)


def test_empty_batch_entries_at_the_ends():
    check([0, 0, 100, 0, 0], 3, 296)
    check([0, 5000, 0], 2, 5)
