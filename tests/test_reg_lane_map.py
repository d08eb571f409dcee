"""The register-streamed decode kernel's lane arithmetic, checked on the CPU.

A 32-lane model of one warp working on one chunk (2 KB of K: 8 tokens at
head_dim 128, 16 at head_dim 64, at most one block), with the index
formulas of decode_reg.cuh written out: which 16-byte piece of which row each
lane loads, the transposing butterfly that turns the lanes' partial dot
products into whole logits, the lane each row's probability is read from for
PV, and the sum over row groups at the end.  Every pool byte of a chunk must
be loaded exactly once, every logit must land on the lanes the kernel reads
it from, and the result must equal the dot products computed directly
("PagedAttention Explained", section "How PagedAttention works", item 5: each
token's key is dotted with the query, then its value weighted).
"""
import numpy as np
import pytest


def chunk_rows(D, BS):
    return min(BS, 2048 // (2 * D))


def cfg(D, rows):
    cpr = D // 8        # 16-byte pieces (8 bf16) per row
    rpi = 32 // cpr     # rows one warp-wide load covers
    rpl = rows // rpi   # rows per lane per chunk
    return cpr, rpi, rpl


def transpose_reduce(x, n, m):
    """The butterfly as the kernel runs it: x[lane] holds n values; at each
    xor step over mask m a lane keeps half (the upper half when its mask bit
    is set) and adds the partner's copy of that half."""
    if m == 0:
        return x
    lanes = np.arange(32)
    if n > 1:
        half = n // 2
        new = np.empty((32, half))
        for lane in lanes:
            upper = (lane & m) != 0
            partner = lane ^ m
            p_upper = (partner & m) != 0
            for i in range(half):
                keep = x[lane, i + half] if upper else x[lane, i]
                sent = x[partner, i] if p_upper else x[partner, i + half]  # what the partner sends
                new[lane, i] = keep + sent
        return transpose_reduce(new, half, m // 2)
    new = x.copy()
    for lane in lanes:
        new[lane, 0] = x[lane, 0] + x[lane ^ m, 0]
    return transpose_reduce(new, 1, m // 2)


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("BS", [8, 16, 32])
def test_chunk_loads_cover_each_byte_once(D, BS):
    rows = chunk_rows(D, BS)
    cpr, rpi, rpl = cfg(D, rows)
    rowb = D * 2
    slice_bytes = BS * rowb
    assert BS % rows == 0 and rows * rowb <= 2048
    for q in range(BS // rows):  # every chunk of one block
        seen = np.zeros(slice_bytes, dtype=int)
        for lane in range(32):
            c, r0 = lane % cpr, lane // cpr
            lane_off = r0 * rowb + c * 16  # within the (block, kv head) slice
            for k in range(rpl):
                off = lane_off + (q % (BS // rows)) * rows * rowb + k * rpi * rowb
                assert 0 <= off and off + 16 <= slice_bytes
                seen[off:off + 16] += 1
        chunk = slice(q * rows * rowb, (q + 1) * rows * rowb)
        assert (seen[chunk] == 1).all() and seen.sum() == rows * rowb


@pytest.mark.parametrize("D,rows", [(128, 8), (64, 8), (64, 16)])
def test_butterfly_logits_and_pv_sources(D, rows):
    cpr, rpi, rpl = cfg(D, rows)
    spread = cpr // rpl  # lanes that end up holding one logit
    rng = np.random.default_rng(D)
    qv = rng.standard_normal(D)
    K = rng.standard_normal((rows, D))
    V = rng.standard_normal((rows, D))
    logits = K @ qv

    # partial dot products: lane (c, r0) over dims [8c, 8c + 8) of rows r0 + rpi k
    sc = np.empty((32, rpl))
    for lane in range(32):
        c, r0 = lane % cpr, lane // cpr
        for k in range(rpl):
            sc[lane, k] = K[r0 + rpi * k, 8 * c:8 * c + 8] @ qv[8 * c:8 * c + 8]
    red = transpose_reduce(sc, rpl, cpr // 2)[:, 0]
    for lane in range(32):
        c, r0 = lane % cpr, lane // cpr
        vi = c // spread
        assert np.isclose(red[lane], logits[r0 + rpi * vi], rtol=0, atol=1e-12)

    # the chunk maximum: xor masks spread .. 16 visit every row's logit
    for lane in range(32):
        seen = {lane}
        m = spread
        while m < 32:
            seen |= {x ^ m for x in seen}
            m <<= 1
        assert np.isclose(max(red[x] for x in seen), logits.max(), rtol=0, atol=1e-12)

    # PV: row r0 + rpi k's probability comes from lane (lane & ~(cpr - 1)) | (k spread)
    p = np.exp(red - logits.max())
    o = np.zeros((32, 8))
    for lane in range(32):
        c, r0 = lane % cpr, lane // cpr
        for k in range(rpl):
            src = (lane & ~(cpr - 1)) | (k * spread)
            assert src // cpr == r0  # same row group
            row = r0 + rpi * k
            assert np.isclose(p[src], np.exp(logits[row] - logits.max()), rtol=0, atol=1e-12)
            o[lane] += p[src] * V[row, 8 * c:8 * c + 8]
    # sum over the row groups (xor masks cpr .. 16), then lane c of row group 0 holds dims [8c, 8c + 8)
    m = cpr
    while m < 32:
        o = o + o[np.arange(32) ^ m]
        m <<= 1
    want = np.exp(logits - logits.max()) @ V
    for c in range(cpr):
        assert np.allclose(o[c], want[8 * c:8 * c + 8], rtol=0, atol=1e-12)

    # the running sum: one owner lane per logit, summed over all 32 lanes
    owners = [lane for lane in range(32) if (lane % cpr) % spread == 0]
    assert len(owners) == rows
    assert np.isclose(sum(p[x] for x in owners), np.exp(logits - logits.max()).sum(), rtol=0, atol=1e-12)
