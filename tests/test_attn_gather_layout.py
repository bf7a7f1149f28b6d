"""The MLA attention's gather, its index arithmetic modelled on the CPU: for both CTAs of the
pair, the three gather warps' requests (the first 32 chunks of 16 bytes of each row, one
request per row; the remaining 4 or 8 chunks of 8 or 4 rows per request) write every (row,
chunk) of the CTA's column range exactly once, each to its own 16-byte slot of the 128-byte
swizzled K-major tile, inside the 40 KB stage, and every request keeps all 32 lanes busy."""

NK, K_BLK, STAGE = 64, 8192, 40960


def requests(half):
    ch_lo, ch_hi = (0, 36) if half == 0 else (32, 72)
    blk0 = 0 if half == 0 else 4
    out = []   # (warp, [(row, chunk, dst) per lane])
    for gw in range(3):
        for r in range(gw, NK, 3):
            out.append((gw, [(r, ch_lo + lane) for lane in range(32)]))
        rc_sh = 2 if half == 0 else 3
        rpg = 32 >> rc_sh
        for grp in range(gw, NK // rpg, 3):
            r0 = grp * rpg
            lanes = []
            for lane in range(32):
                src_lane = (r0 & 31) + (lane >> rc_sh)
                assert src_lane < 32                          # the shuffle reads a real lane
                assert (r0 < 32) == (r0 + (lane >> rc_sh) < 32)   # one id register per request
                lanes.append((r0 + (lane >> rc_sh), ch_lo + 32 + (lane & ((1 << rc_sh) - 1))))
            out.append((gw, lanes))
    return ch_lo, ch_hi, blk0, out


def dst(r, c, blk0):
    return ((c >> 3) - blk0) * K_BLK + r * 128 + (((c & 7) ^ (r & 7)) << 4)


def test_gather_requests_cover_each_row_chunk_once_in_the_swizzled_stage():
    for half in (0, 1):
        ch_lo, ch_hi, blk0, reqs = requests(half)
        seen = {}
        for _, lanes in reqs:
            assert len(lanes) == 32
            for r, c in lanes:
                seen[(r, c)] = seen.get((r, c), 0) + 1
        assert set(seen) == {(r, c) for r in range(NK) for c in range(ch_lo, ch_hi)}
        assert all(v == 1 for v in seen.values())
        offs = [dst(r, c, blk0) for r, c in seen]
        assert min(offs) >= 0 and max(offs) + 16 <= STAGE and len(set(offs)) == len(offs)


def test_gather_work_is_balanced_over_the_three_warps():
    for half in (0, 1):
        _, _, _, reqs = requests(half)
        per_warp = [sum(1 for w, _ in reqs if w == gw) for gw in range(3)]
        assert max(per_warp) - min(per_warp) <= 2, per_warp
