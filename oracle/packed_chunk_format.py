"""Reference codec of a packed rank-chunk format at 2.5 bytes per slot.

TEST INFRASTRUCTURE ONLY, under the same rules as ``effort_oracle``: nothing
on the product path may import or call it, and it shares nothing with the
CUDA library.  It defines a storage format; the method's results do not
change with the format (the format is lossless), so their oracle stays
``effort_oracle``.

Source: [SHOW-HN] Hacker News thread "Show HN: Speeding up LLM inference 2x
times (possibly)", item 40067677: the author's exchange on embedding
position bits in the weight word (the bits a weight loses to its position
against the bits it gains from belonging to a known bucket: a bucket's
weights span a smaller range than the whole row's), and the post's note
that the format stores each row sorted, so only a leading part of it is
read.

Reading (the pages give no fp16 bit layout):

* A chunk is what the rank-chunk layout stores: a run of consecutive ranks
  of one (row, panel) list, ordered by column, in 64 slots.  Its first rank
  is its largest magnitude H (binary16 magnitude bits, kept beside the chunk
  as its head, which the dispatch reads anyway).
* Every slot is 20 bits: the value's sign, a 12-bit offset d = H - m of its
  magnitude bits m below the head, and a 7-bit column gap (from column -1
  of the panel for the first slot, else from the previous slot).  Offset
  4095 stands for magnitude 0 whatever H is (the sign is kept, so -0 stays
  -0).  Binary16 magnitudes order like their bit patterns, so m = H - d is
  exact.  A chunk's cut keeps every entry's offset at most 4094 (or its
  magnitude 0); a gap above 127 is bridged by filler slots (+0, gap 127);
  pads after the last entry are (+0, gap 0).  The format is lossless: every
  stored value's bits and column come back exactly.
* Storage, for aligned per-lane loads (8 lanes x 8 slots): plane A holds one
  16-bit word per slot, (sign << 15) | (d << 3) | (gap >> 4); plane B holds
  the low 4 gap bits, 8 slots per 32-bit word (slot k of the word in bits
  4k .. 4k + 3).  64 x 2 + 8 x 4 = 160 bytes per chunk: 2.5 bytes per slot.
"""
from __future__ import annotations

import numpy as np

SLOTS = 64
GAP_MAX = 127
D_ZERO = 4095          # offset code of magnitude 0
D_MAX = 4094           # largest offset of a nonzero magnitude
BYTES_PER_CHUNK = SLOTS * 2 + (SLOTS // 8) * 4


def _fits(head_mag: int, mag: int) -> bool:
    return mag == 0 or 0 <= head_mag - mag <= D_MAX


def slots_needed(cols_sorted) -> int:
    """Slots of a chunk whose entries lie at these panel-local columns
    (ascending): one per entry plus the fillers its gaps need."""
    prev, n = -1, 0
    for c in cols_sorted:
        g = c - prev
        n += 1 + (g - 1) // GAP_MAX
        prev = c
    return n


def cut_list(entries):
    """Greedy cut of one list into chunks.

    entries: [(column, binary16 bits)] in rank order (|w| descending, ties
    to the lower column), columns panel-local.  Each chunk takes as many
    next ranks as fit in 64 slots with every offset encodable.  Returns the
    chunks as lists of (column, bits) in rank order.
    """
    chunks, q = [], 0
    while q < len(entries):
        head = entries[q][1] & 0x7FFF
        t = 0
        while q + t < len(entries):
            col, bits = entries[q + t]
            if not _fits(head, bits & 0x7FFF):
                break
            if slots_needed(sorted(c for c, _ in entries[q:q + t + 1])) > SLOTS:
                break
            t += 1
        if t == 0:
            raise ValueError("an entry that cannot start a chunk")  # unreachable: d = 0 for the head
        chunks.append(entries[q:q + t])
        q += t
    return chunks


def encode_chunk(chunk):
    """(head magnitude bits, plane A uint16[64], plane B uint32[8]) of one
    chunk given as [(column, bits)] (any order; stored by column)."""
    head = max(b & 0x7FFF for _, b in chunk)
    slots = []  # (sign, d, gap)
    prev = -1
    for col, bits in sorted(chunk):
        g = col - prev
        while g > GAP_MAX:
            slots.append((0, D_ZERO, GAP_MAX))
            g -= GAP_MAX
        m = bits & 0x7FFF
        if not _fits(head, m):
            raise ValueError("magnitude out of the chunk's range")
        slots.append((bits >> 15, D_ZERO if m == 0 else head - m, g))
        prev = col
    if len(slots) > SLOTS:
        raise ValueError("chunk over 64 slots")
    slots += [(0, D_ZERO, 0)] * (SLOTS - len(slots))
    a = np.zeros(SLOTS, np.uint16)
    b = np.zeros(SLOTS // 8, np.uint32)
    for k, (s, d, g) in enumerate(slots):
        a[k] = (s << 15) | (d << 3) | (g >> 4)
        b[k // 8] |= np.uint32((g & 15) << (4 * (k % 8)))
    return head, a, b


def decode_chunk(head, a, b):
    """[(column, binary16 bits, kind)] of the 64 slots; kind is 'value' for
    a slot with a nonzero magnitude, 'zero' for magnitude 0 (an entry of
    magnitude 0, a filler or a pad)."""
    out, col = [], -1
    for k in range(SLOTS):
        w = int(a[k])
        g = ((w & 7) << 4) | ((int(b[k // 8]) >> (4 * (k % 8))) & 15)
        d = (w >> 3) & 0xFFF
        col += g
        m = 0 if d == D_ZERO else head - d
        out.append((col, ((w >> 15) << 15) | m, "zero" if m == 0 else "value"))
    return out


def encode_list(entries):
    """All chunks of one list: [(head, plane A, plane B, entries of the chunk)]."""
    return [(*encode_chunk(c), c) for c in cut_list(entries)]
