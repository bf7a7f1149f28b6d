"""The 16-head MQA attention's shared-memory plan and tile loads, modelled on the CPU: the tile
loads (ids first, then the row copies) cover every (key row, 16-byte chunk) of the K and V tiles
once; P, written into the current stage's K tile, stays inside it; and the block's footprint
lets six CTAs share an SM's 228 KB (each also holding the 1 KB the driver reserves)."""

HG, D_QK, D_V, KT, STAGES, NWV = 16, 128, 128, 32, 2, 2
THREADS = (HG // 16) * NWV * 32
QCH, VCH = D_QK // 8, D_V // 8
Q_BYTES = HG * D_QK * 2
K_TILE, V_TILE = KT * D_QK * 2, KT * D_V * 2
P_BYTES = HG * KT * 2


def swz(r, c, chunks):
    return (r * chunks + (c ^ (r & 7))) * 16


def pswz(r, c):
    return (r * 4 + (c ^ ((r >> 1) & 3))) * 16


def test_tile_loads_cover_every_row_chunk_once():
    for chunks in (QCH, VCH):
        n_it = (KT * chunks + THREADS - 1) // THREADS
        seen = {}
        for tid in range(THREADS):
            for u in range(n_it):
                i = tid + u * THREADS
                if i < KT * chunks:
                    rc = (i // chunks, i % chunks)
                    seen[rc] = seen.get(rc, 0) + 1
        assert set(seen) == {(r, c) for r in range(KT) for c in range(chunks)}
        assert all(v == 1 for v in seen.values())
        offs = sorted(swz(r, c, chunks) for r, c in seen)
        assert offs[0] == 0 and offs[-1] + 16 == KT * chunks * 16 and len(set(offs)) == len(offs)


def test_p_fits_in_the_k_tile_and_six_ctas_fit_an_sm():
    p_offs = [pswz(r, c) + b for r in range(HG) for c in range(KT // 8) for b in range(16)]
    assert min(p_offs) == 0 and max(p_offs) < P_BYTES <= K_TILE and len(set(p_offs)) == P_BYTES
    off_p = Q_BYTES + STAGES * K_TILE + STAGES * V_TILE
    off_idx = off_p + 0                    # P lives in the K tile: no buffer of its own
    smem = off_idx + STAGES * KT * 4 + 2 * NWV * HG * 4
    assert smem == 37376
    assert 6 * (smem + 1024) <= 228 * 1024 < 7 * (smem + 1024)
    assert 5 * (smem + P_BYTES + 1024) <= 228 * 1024 < 6 * (smem + P_BYTES + 1024)   # with its own P: five
