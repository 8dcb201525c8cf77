"""CPU statement of the split-KV work partition the library uses (host logic
for the bit-exact plan test).

Sequence n has tiles_n = ceil(L_n / 128) tiles of 128 tokens, or none when
L_n < 1 or L_n > max_pages_per_seq * page_size.  The concatenation of all
tiles is cut into num_ctas contiguous ranges of ceil(total / num_ctas) tiles.
"""
from __future__ import annotations

TILE = 128


def seq_tiles(L, page_size, max_pages):
    if L < 1 or L > max_pages * page_size:
        return 0
    return -(-L // TILE)


def plan(seqlens, page_size, max_pages, num_ctas):
    """Returns the flat int list the library's plan dump writes."""
    tiles = [seq_tiles(int(L), page_size, max_pages) for L in seqlens]
    total = sum(tiles)
    chunk = -(-total // num_ctas) if total > 0 else 0
    firsts, acc = [], 0
    for t in tiles:
        firsts.append(acc)
        acc += t

    def seq_of(g):
        for n, (f, t) in enumerate(zip(firsts, tiles)):
            if t > 0 and f <= g < f + t:
                return n
        return -1

    out = []
    for c in range(num_ctas):
        g0, g1 = c * chunk, min(c * chunk + chunk, total)
        if g0 < g1:
            out += [g0, g1, seq_of(g0), seq_of(g1 - 1)]
        else:
            out += [min(g0, total), max(g1, min(g0, total)), -1, -1]
    for f, t in zip(firsts, tiles):
        if t == 0:
            out += [0, -1]
        else:
            out += [(f + t - 1) // chunk - f // chunk + 1, f // chunk]
    return out
