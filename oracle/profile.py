"""Expert profile file (STRP v1) and the slot-budget hit rate, restated from
the "Coder benchmark record" page: section "expert profile file" (magic STRP,
version 1, a header of five 32-bit fields - version, layers, experts, ranked
pairs, entries - the ranked (layer, expert) pairs as two 16-bit fields each in
rank order, and one inverse table per layer of n_expert entries, -1 for an
unranked pair) and section "why a 72% hit rate proves the mapping" (with S
cache slots filled in rank order, the share of expert reads that find their
expert resident).

TEST INFRASTRUCTURE ONLY, like the rest of oracle/: only the tests may call it.
Readings where the page is silent or garbled: every field is little-endian;
the header's "ranked pairs" counts the body and "entries" the inverse tables
(L * E); an inverse entry is a signed 32-bit rank.
"""
from __future__ import annotations

import struct

import numpy as np


def profile_bytes(pairs, L: int, E: int) -> bytes:
    """The file for `pairs` [(layer, expert), ...] in rank order."""
    pairs = [(int(l), int(e)) for l, e in pairs]
    rank = {}
    for r, p in enumerate(pairs):
        assert p not in rank and 0 <= p[0] < L and 0 <= p[1] < E
        rank[p] = r
    out = [b"STRP", struct.pack("<5I", 1, L, E, len(pairs), L * E)]
    for l, e in pairs:
        out.append(struct.pack("<HH", l, e))
    for l in range(L):
        for e in range(E):
            out.append(struct.pack("<i", rank.get((l, e), -1)))
    return b"".join(out)


def parse_profile(data: bytes):
    """(L, E, pairs [(layer, expert)], inverse [[rank]]) of a file."""
    assert data[:4] == b"STRP"
    version, L, E, n, entries = struct.unpack_from("<5I", data, 4)
    assert version == 1 and entries == L * E
    pos = 24
    pairs = []
    for _ in range(n):
        pairs.append(struct.unpack_from("<HH", data, pos))
        pos += 4
    inverse = []
    for _ in range(L):
        inverse.append(list(struct.unpack_from(f"<{E}i", data, pos)))
        pos += 4 * E
    assert pos == len(data)
    return L, E, pairs, inverse


def hit_rate(pairs, slots: int, hist) -> float:
    """Share of the reads counted in hist [L][E] whose (layer, expert) is among
    the first `slots` ranked pairs."""
    hist = np.asarray(hist)
    resident = set((int(l), int(e)) for l, e in list(pairs)[:slots])
    total = int(hist.sum())
    hit = sum(int(hist[l, e]) for l, e in resident)
    return hit / total if total else 0.0
