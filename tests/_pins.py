"""Independent restatements used to pin the oracle (CPU only).

These are deliberately written differently from the oracle: eq. 4 is transcribed
literally with floating-point log2 / floor / ceil and real division, as printed;
the 3D window and the sliding window are vectorised numpy enumerations over
grid coordinates; tile reduction is a numpy reshape-sum.
"""
import numpy as np

TILE = 128


def radial_mask_literal(f: int, s: int) -> np.ndarray:
    """eq. 4 of "Radial Attention ..." (sec. 3), literally, in float arithmetic.
    Returns the n x n kept mask (True = M is 0), token index = frame*s + position."""
    n = f * s
    q = np.arange(n)[:, None]
    key = np.arange(n)[None, :]
    i, k = q // s, q % s
    j, l = key // s, key % s
    dist = np.abs(i - j).astype(np.float64)
    p2 = 2.0 ** np.floor(np.log2(np.maximum(dist, 1.0)))
    first = (p2 <= s) & (np.abs(k - l) + 1 <= s / p2)
    second = (np.mod(dist, np.ceil(p2 / s)) == 0) & (k == l)
    return first | second


def window3d_mask_grid(T: int, H: int, W: int, r_t: int, r_s: int) -> np.ndarray:
    """Cube neighbourhood on the (t, h, w) grid, out-of-grid neighbours absent."""
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    t, h, w = t.ravel(), h.ravel(), w.ravel()
    return ((np.abs(t[:, None] - t[None, :]) <= r_t) & (np.abs(h[:, None] - h[None, :]) <= r_s)
            & (np.abs(w[:, None] - w[None, :]) <= r_s))


def swc_mask_frames(f: int, s: int, W: int) -> np.ndarray:
    """Query frame i sees key frames max(0, i-W+1) .. i (prose of the Vera page)."""
    fr = np.repeat(np.arange(f), s)
    lo = np.maximum(0, fr - W + 1)
    return (fr[None, :] >= lo[:, None]) & (fr[None, :] <= fr[:, None])


def tile_reduce(mask: np.ndarray) -> np.ndarray:
    """Kept pairs per 128x128 tile of an n x n mask (zero padded at the tail)."""
    n = mask.shape[0]
    nb = -(-n // TILE)
    pad = np.zeros((nb * TILE, nb * TILE), dtype=np.int64)
    pad[:n, :n] = mask
    return pad.reshape(nb, TILE, nb, TILE).sum(axis=(1, 3))


def radial_closed_form_total(f: int, s: int) -> int:
    """Kept pairs of eq. 4 summed over frame distances.

    For frame distance D (w = 2^floor(log2 max(D,1))): if w <= s a frame pair
    keeps the diagonal band |k-l| <= m with m = floor(s/w) - 1, i.e.
    s(2m+1) - m(m+1) pairs; otherwise it keeps the s diagonal pairs when
    D mod ceil(w/s) == 0 and nothing else.  Distance 0 occurs f times, distance
    D > 0 occurs 2(f-D) times."""
    total = 0
    for D in range(f):
        w = 1 << (max(D, 1).bit_length() - 1)
        if w <= s:
            m = s // w - 1
            per = s * (2 * m + 1) - m * (m + 1)
        else:
            per = s if D % (-(-w // s)) == 0 else 0
        total += (f if D == 0 else 2 * (f - D)) * per
    return total


def csr_from_tiles(counts: np.ndarray):
    kept = counts > 0
    row_ptr = np.concatenate([[0], np.cumsum(kept.sum(axis=1))]).astype(np.int32)
    qb, kb = np.nonzero(kept)
    col_idx = kb.astype(np.int32)
    count = counts[qb, kb].astype(np.int32)
    flag = (count == TILE * TILE).astype(np.uint8)
    return row_ptr, col_idx, count, flag


def block_mask_from_tiles(counts: np.ndarray, n: int) -> np.ndarray:
    """Element mask of block mode: every valid pair of every kept tile."""
    kept = counts > 0
    return np.kron(kept, np.ones((TILE, TILE), dtype=bool))[:n, :n]


def radial_tile_stats_intervals(f: int, s: int):
    """Tile statistics of eq. 4 at the 128 x 128 granularity, from the key
    interval of each (query frame segment, key frame) pair instead of pairs.

    Only for shapes where every frame distance keeps a diagonal band (w <= s for
    D <= f - 1).  A query tile covers one or two frame segments of consecutive
    positions [ka, kb]; in key frame j at distance D it keeps the positions
    [ka - m, kb + m] (m = floor(s / w) - 1), so its kept key tiles are those that
    interval touches.  A kept tile is FULL iff every (query segment, key segment)
    pair inside it is within the band: max(kb - la, lb - ka) <= m for the key
    segment [la, lb] of frame j, and the tile has no tail rows or keys.
    Returns, per query tile, the sorted kept key tiles and the FULL ones."""
    n = f * s
    nb = -(-n // TILE)
    assert 1 << (max(f - 1, 1).bit_length() - 1) <= s, "a frame distance with w > s"
    m_of = np.empty(f, dtype=np.int64)
    for D in range(f):
        w = 1 << (max(D, 1).bit_length() - 1)
        m_of[D] = s // w - 1
    rows, fulls = [], []
    frames = np.arange(f)
    for qb in range(nb):
        r0, r1 = qb * TILE, min(n, qb * TILE + TILE) - 1
        segs = [(i, max(r0, i * s) - i * s, min(r1, i * s + s - 1) - i * s) for i in range(r0 // s, r1 // s + 1)]
        kept = set()
        for i, ka, kbp in segs:
            m = m_of[np.abs(i - frames)]
            lo = np.maximum(0, ka - m) + frames * s
            hi = np.minimum(s - 1, kbp + m) + frames * s
            for a, b in zip(lo // TILE, hi // TILE):
                kept.update(range(int(a), int(b) + 1))
        kept = np.array(sorted(kept), dtype=np.int64)
        rows.append(kept)
        full = []
        fulls.append(full)
        if r1 - r0 + 1 < TILE:
            continue
        for kb in kept:
            c0, c1 = kb * TILE, min(n, kb * TILE + TILE) - 1
            if c1 - c0 + 1 < TILE:
                continue
            ok = True
            for i, ka, kbp in segs:
                for j in range(c0 // s, c1 // s + 1):
                    la, lb = max(c0, j * s) - j * s, min(c1, j * s + s - 1) - j * s
                    if max(kbp - la, lb - ka) > m_of[abs(i - j)]:
                        ok = False
                        break
                if not ok:
                    break
            if ok:
                full.append(int(kb))
    return rows, fulls
