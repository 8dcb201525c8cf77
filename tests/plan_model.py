"""CPU statement of the split-KV work partition the library uses (host logic
for the bit-exact plan test).

Sequence n has tiles_n = ceil(L_n / 128) tiles of 128 tokens, or none when
L_n < 1 or L_n > max_pages_per_seq * page_size.  Each tile costs TILE_COST
units and each valid sequence SEQ_COST more, placed after its last tile, so a
CTA whose range enters a new sequence is given less token work.  Tile t of
sequence n starts at cum_n + TILE_COST * t; with
chunk = TILE_COST * max(ceil(total / (num_ctas * TILE_COST)), 1) (a whole
number of tiles), CTA c owns the tiles that start in
[c * chunk, (c + 1) * chunk).
"""
from __future__ import annotations

TILE = 128
TILE_COST = 8
SEQ_COST = 4


def seq_tiles(L, page_size, max_pages):
    if L < 1 or L > max_pages * page_size:
        return 0
    return -(-L // TILE)


def owners(seqlens, page_size, max_pages, num_ctas):
    """Owner CTA of every tile, as a list of (sequence, tile, cta)."""
    tiles = [seq_tiles(int(L), page_size, max_pages) for L in seqlens]
    total = sum(TILE_COST * t + SEQ_COST for t in tiles if t)
    chunk = TILE_COST * max(-(-total // (num_ctas * TILE_COST)), 1)
    out, cum = [], 0
    for n, t in enumerate(tiles):
        if not t:
            continue
        for i in range(t):
            out.append((n, i, (cum + TILE_COST * i) // chunk))
        cum += TILE_COST * t + SEQ_COST
    return out


def plan(seqlens, page_size, max_pages, num_ctas):
    """Returns the flat int list the library's plan dump writes."""
    own = owners(seqlens, page_size, max_pages, num_ctas)
    per_cta = [[0, 0, -1, -1] for _ in range(num_ctas)]
    for g, (n, _, c) in enumerate(own):
        p = per_cta[c]
        if p[2] < 0:
            p[0], p[2] = g, n
        p[1], p[3] = g + 1, n
    out = [v for p in per_cta for v in p]
    for n in range(len(seqlens)):
        cs = sorted({c for m, _, c in own if m == n})
        out += [len(cs), cs[0]] if cs else [0, -1]
    return out
