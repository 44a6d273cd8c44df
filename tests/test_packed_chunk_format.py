"""Pins of the packed 2.5-byte-per-slot chunk codec (oracle/packed_chunk_format).

* Round trip: every chunk decodes slot by slot to the list the layout rule
  gives, built here independently (entries by column, a filler for every
  127 columns of a longer gap, pads after the last entry).
* The cut: runs of consecutive ranks, at most 64 slots, every offset
  encodable, and greedy (the next rank would break one of the two limits).
* Edge cases: zeros of both signs, subnormals, ties, gaps up to the panel
  width, a magnitude range wider than the 12-bit offset.
* Size: 160 bytes per chunk; bytes per stored entry against the 3-byte slot
  layout on fp16 N(0, 0.02^2) rows.
"""
import numpy as np
import pytest

from oracle import packed_chunk_format as PF


def expected_slots(chunk):
    """(column, bits) of the 64 slots by the layout rule."""
    out, prev = [], -1
    for col, bits in sorted(chunk):
        g = col - prev
        while g > PF.GAP_MAX:
            prev += PF.GAP_MAX
            out.append((prev, 0))
            g -= PF.GAP_MAX
        out.append((col, bits))
        prev = col
    last = out[-1][0]
    return out + [(last, 0)] * (PF.SLOTS - len(out))


def rank_order(cols, bits):
    """(column, bits) in rank order: |w| descending, ties to the lower column."""
    return sorted(zip(cols, bits), key=lambda e: (-(e[1] & 0x7FFF), e[0]))


def check_list(entries):
    chunks = PF.encode_list(entries)
    got = []
    for head, a, b, chunk in chunks:
        assert a.nbytes + b.nbytes == PF.BYTES_PER_CHUNK == 160
        assert head == chunk[0][1] & 0x7FFF
        dec = PF.decode_chunk(head, a, b)
        assert [(c, bits) for c, bits, _ in dec] == expected_slots(chunk)
        got.extend(chunk)
    assert got == entries  # consecutive ranks, in order, nothing lost
    # greedy: the rank after each chunk would break the offset or the slot limit
    q = 0
    for _, _, _, chunk in chunks:
        q += len(chunk)
        if q < len(entries):
            head = chunk[0][1] & 0x7FFF
            m = entries[q][1] & 0x7FFF
            grown = sorted(c for c, _ in chunk + [entries[q]])
            assert not (m == 0 or head - m <= PF.D_MAX) or PF.slots_needed(grown) > PF.SLOTS
    return chunks


def gaussian_panel_list(rng, width=2048, keep=1.0, stored=3 / 8):
    w = (rng.standard_normal(width) * 0.02).astype(np.float16)
    bits = w.view(np.uint16).astype(np.int64)
    order = rank_order(range(width), bits)
    n = int(np.floor(keep * width + 0.5))
    return order[:max(1, -(-int(n * stored * 8) // 8))]


@pytest.mark.parametrize("seed", range(6))
def test_round_trip_gaussian_lists(seed):
    rng = np.random.default_rng(seed)
    check_list(gaussian_panel_list(rng, stored=3 / 8))
    check_list(gaussian_panel_list(rng, stored=1.0))   # a whole list, down to the smallest magnitudes
    check_list(gaussian_panel_list(rng, width=300, keep=0.6))


def test_zeros_signs_subnormals_and_ties():
    e = rank_order([5, 9, 12, 40, 41, 300, 301, 2047],
                   [0x3C00, 0xBC00, 0x0001, 0x8001, 0x0000, 0x8000, 0x3C00, 0x0000])
    chunks = check_list(e)
    dec = [(c, b) for head, a, bb, _ in chunks for c, b, _ in PF.decode_chunk(head, a, bb)]
    assert (300, 0x8000) in dec and (41, 0x0000) in dec  # -0 stays -0
    assert (12, 0x0001) in dec and (40, 0x8001) in dec   # subnormals exact


def test_gaps_up_to_the_panel_width():
    e = rank_order([0, 2047], [0x2000, 0x2001])
    (head, a, b, chunk), = check_list(e)
    assert PF.slots_needed([0, 2047]) == 2 + (2047 - 1) // 127


def test_magnitude_range_wider_than_the_offset_starts_a_new_chunk():
    # 0x7000 down to 0x6000 spans 4096 patterns: the last one cannot share the head's chunk
    e = [(0, 0x7000), (1, 0x7000 - 4094), (2, 0x6000), (3, 0x0000)]
    chunks = check_list(e)
    assert [len(c) for *_, c in chunks] == [2, 2]


def test_slot_limit_cuts_a_dense_run():
    e = rank_order(list(range(200)), [0x3000] * 200)  # ties: column order
    chunks = check_list(e)
    # the third chunk starts 129 columns after column -1: one filler, 63 entries
    assert [len(c) for *_, c in chunks] == [64, 64, 63, 9]


def test_bytes_per_stored_entry_against_three_byte_slots():
    # stored parts (3/8) of fp16 N(0, 0.02^2) panel lists: 2.5 B per slot,
    # 2.71 B per stored entry (fillers for gaps above 127 and each list's
    # partial last chunk) against 3.06 B for the 3-byte layout's chunks
    rng = np.random.default_rng(77)
    packed, entries3, n_entries = 0, 0, 0
    for _ in range(40):
        lst = gaussian_panel_list(rng)
        packed += len(PF.cut_list(lst)) * PF.BYTES_PER_CHUNK
        n_entries += len(lst)
        # the 3-byte layout: 64-slot chunks, 8-bit gaps (fillers per 255 columns), no range limit
        q = 0
        while q < len(lst):
            t = 0
            while q + t < len(lst):
                cols = sorted(c for c, _ in lst[q:q + t + 1])
                prev, s = -1, 0
                for c in cols:
                    s += 1 + (c - prev - 1) // 255
                    prev = c
                if s > 64:
                    break
                t += 1
            entries3 += 64 * 3
            q += t
    assert packed / n_entries <= 2.75
    assert packed <= 0.9 * entries3
