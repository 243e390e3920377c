"""CPU model of the append kernel's shared-memory tile layout.

The append stages a kind's rows of a tile as [part][row][64 elements] with 16-byte
chunk c of a part row stored at chunk c ^ (row & 7).  Two producers fill it: the
tensor-copy unit with its 128-byte swizzle (16-byte chunk bits 4-6 of the offset xor
the 128-byte row bits 7-9, inside a 1024-byte aligned box), and lane-wise cp.async
copies through the kernel's own address formula.  One consumer reads it: lane
(row, part) loads chunk c at (part row address | (row & 7) << 4) ^ (c << 4).  This
test checks, for every head dim and head count the kernel serves, that both producers
put every element where the consumer looks for it.
"""
import pytest


def _geom(d, esize):
    tpr = d // 64                      # lanes per row
    rows = 32 // tpr                   # rows per tile
    pb = 64 * esize                    # bytes of one lane's part of a row
    return tpr, rows, pb


def _tile_at(r, b, rows, pb):
    """cp.async producer: byte b of input row r."""
    return (b // pb) * (rows * pb) + r * pb + ((((b % pb) >> 4) ^ (r & 7)) << 4) + (b & 15)


def _tensor_copy(part, h_local, t_local, e, hb, rows, pb):
    """Tensor-copy producer: element e (0..63) of box (part; head h_local, token t_local)."""
    linear = (t_local * hb + h_local) * 128 + e * 2
    swz = linear ^ (((linear >> 7) & 7) << 4)
    return part * rows * pb + swz


def _consumer(rl, part, c, rows, pb):
    row = (part * rows + rl) * pb + ((rl & 7) << 4)
    return row ^ (c << 4)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("esize", [2, 4])
def test_cp_async_layout_matches_consumer(d, esize):
    tpr, rows, pb = _geom(d, esize)
    for rl in range(rows):
        for part in range(tpr):
            for c in range(pb // 16):
                addr = _consumer(rl, part, c, rows, pb)
                # chunk c of this lane's part holds input bytes part*pb + 16c .. +15
                b = part * pb + 16 * c
                assert _tile_at(rl, b, rows, pb) == addr
    # the layout is a permutation of the buffer
    seen = {_tile_at(r, b, rows, pb) for r in range(rows) for b in range(0, d * esize)}
    assert seen == set(range(rows * d * esize))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("h_kv", [1, 2, 4, 8, 16, 32])
def test_tensor_copy_layout_matches_cp_async(d, h_kv):
    tpr, rows, pb = _geom(d, 2)
    if h_kv <= rows and rows % h_kv == 0:
        hb = h_kv
    elif h_kv % rows == 0:
        hb = rows
    else:
        pytest.skip("tile is not a box of the input")
    tb = rows // hb
    for part in range(tpr):
        for t_local in range(tb):
            for h_local in range(hb):
                r = t_local * hb + h_local          # pair index within the tile
                for e in range(64):
                    b = (part * 64 + e) * 2        # byte of the input row
                    assert _tensor_copy(part, h_local, t_local, e, hb, rows, pb) == \
                        _tile_at(r, b, rows, pb)
