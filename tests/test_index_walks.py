"""Host-side checks of the index arithmetic the elementwise and spectral kernels use (mirrors of
the device code, no GPU): the strided row walk of the momentum and apply passes, the shared-memory
layout of v in the streaming spectral passes, the row coverage of the column-slab pass, the
block / stage split of the power pass and where its warps' z meet at the end of an iteration.
Each mirror is compared with the plain definition (division, a dense loop) it replaces."""
import pytest


# ---------------------------------------------------------------- strided row walk (rowpos.cuh)
def rowpos_at(v, per_row):
    i = v // per_row
    return [i, v - i * per_row]


def rowstep_of(stride, per_row):
    return stride // per_row, stride % per_row


def rowpos_add(p, step, per_row):
    i, j = p[0] + step[0], p[1] + step[1]
    if j >= per_row:
        j -= per_row
        i += 1
    return [i, j]


@pytest.mark.parametrize("per_row", [1, 7, 96, 192, 384, 419, 1000, 4096])
@pytest.mark.parametrize("stride", [1, 7, 256, 512])
def test_row_walk_matches_division(per_row, stride):
    """Walking a flattened index in fixed strides by one division at the start and an add with at
    most one wrap per step gives the same (row, position) as dividing at every step."""
    step = rowstep_of(stride, per_row)
    for start in (0, 1, per_row - 1, 3 * per_row + 5, 123457):
        p = rowpos_at(start, per_row)
        v = start
        for _ in range(200):
            assert p == [v // per_row, v % per_row]
            v += stride
            p = rowpos_add(p, step, per_row)


# ---------------------------------------------------------------- v in shared memory (vs_index)
def vs_index(c):
    return (c & ~255) | ((c & 4) << 5) | (((c & 255) >> 3) << 2) | (c & 3)


@pytest.mark.parametrize("cols", [8, 256, 520, 768, 1536, 2048])
def test_split_layout_is_a_bijection_with_conflict_free_lane_reads(cols):
    """The split layout maps the columns of every 256-column chunk one to one onto that chunk's
    256 slots; lane k's 16-byte reads at 4k and 128 + 4k of chunk i hold columns 8k..8k+3 and
    8k+4..8k+7, and the eight lanes of a quarter warp start their 16-byte reads in eight distinct
    groups of four banks (no bank conflict)."""
    span = (cols + 255) & ~255
    pos = [vs_index(c) for c in range(span)]
    assert sorted(pos) == list(range(span))
    for i in range(span // 256):
        for k in range(32):
            lo = [pos.index(256 * i + 4 * k + t) for t in range(4)]
            hi = [pos.index(256 * i + 128 + 4 * k + t) for t in range(4)]
            assert lo == [256 * i + 8 * k + t for t in range(4)]
            assert hi == [256 * i + 8 * k + 4 + t for t in range(4)]
        for q in range(4):  # quarter warps
            for base in (0, 128):
                # first of the four 4-byte banks each 16-byte read covers
                slots = {(256 * i + base + 4 * k) % 32 // 4 for k in range(8 * q, 8 * q + 8)}
                assert len(slots) == 8


# ---------------------------------------------------------------- column-slab phase 1 rows
@pytest.mark.parametrize("S", [64, 128, 256])
@pytest.mark.parametrize("rows", [1, 3, 31, 64, 130, 768, 1000])
def test_column_slab_rows_each_read_once(S, rows):
    """Phase 1 of the column-slab pass: warp w and row group g of its lanes start at row
    w * RPW + g and step by (warps x RPW) rows, kSlabUnroll rows per pass of the loop; every row
    of the slab is read by exactly one (warp, row group)."""
    warps, unroll = 8, 8
    lpr = S // 8
    rpw = 32 // lpr
    rstride = warps * rpw
    seen = [0] * rows
    for w in range(warps):
        for g in range(rpw):
            r0 = w * rpw + g
            while r0 < rows:
                for u in range(unroll):
                    r = r0 + u * rstride
                    if r < rows:
                        seen[r] += 1
                r0 += rstride * unroll
    assert seen == [1] * rows


@pytest.mark.parametrize("S", [64, 128, 256])
@pytest.mark.parametrize("unroll", [4, 8])
@pytest.mark.parametrize("rows", [1, 3, 31, 64, 130, 768, 1000])
def test_column_slab_phase2_rows_each_written_once(S, unroll, rows):
    """Phase 2 of the column-slab pass walks the rows warp-uniformly: warp w starts at w * RPW,
    steps by (warps x RPW x unroll), and row group g takes row start + g + u * (warps x RPW) for
    u < unroll when it is below `rows`; every row's partial is written by exactly one lane."""
    warps = 8
    lpr = S // 8
    rpw = 32 // lpr
    rstride = warps * rpw
    seen = [0] * rows
    for w in range(warps):
        rb = w * rpw
        while rb < rows:
            for lane in range(32):
                g, k = lane // lpr, lane % lpr
                for u in range(unroll):
                    r = rb + g + u * rstride
                    if k == 0 and r < rows:
                        seen[r] += 1
            rb += rstride * unroll
    assert seen == [1] * rows


# ---------------------------------------------------------------- power pass blocks and stages
def power_blocks(rows, want):
    rpb = ((rows + want - 1) // want + 7) // 8 * 8
    return (rows + rpb - 1) // rpb, rpb


@pytest.mark.parametrize("rows", [1, 8, 9, 77, 300, 768, 3352, 4000, 32768])
@pytest.mark.parametrize("want", [1, 2, 12, 37, 64])
def test_power_pass_blocks_cover_rows_in_whole_stages(rows, want):
    """The row split of the streaming power pass: every block but the last holds a multiple of
    eight rows (whole stages), no block is empty, the blocks cover the rows exactly once, and there
    are never more blocks than asked for (the per-matrix partial count the launch sizes)."""
    nblk, rpb = power_blocks(rows, want)
    assert 1 <= nblk <= max(1, want) and rpb % 8 == 0
    covered = []
    for b in range(nblk):
        beg, end = b * rpb, min(rows, b * rpb + rpb)
        assert end > beg
        nst = (end - beg + 7) // 8  # stages of eight rows
        assert nst * 8 >= end - beg > (nst - 1) * 8
        covered.extend(range(beg, end))
    assert covered == list(range(rows))


# ---------------------------------------------------------------- power pass: warps' z in held stages
def held_step(nst, f32):
    """First stage of the final step when that step holds the eight warps' z, else -1."""
    jl = (nst - 1) & ~1
    return jl if (jl + 1 < nst or f32) else -1


@pytest.mark.parametrize("f32", [False, True])
@pytest.mark.parametrize("C", [8, 48, 256, 768, 1536, 2048])
@pytest.mark.parametrize("nst", [1, 2, 3, 8, 35, 36])
@pytest.mark.parametrize("stages", [2, 3, 7, 8])
def test_power_pass_held_stages_take_every_warps_z(f32, C, nst, stages):
    """At the end of an iteration of the streaming power pass, warp w writes its z (C floats,
    eight columns per lane step) to slot w % wps of stage held_j + w / wps of the ring: the slots
    are disjoint, lie inside their stage, the held stages are distinct ring slots, and the
    consumer threads' eight-column reads cover every column of every warp exactly once."""
    warps = 8
    stage_bytes = warps * C * (4 if f32 else 2)
    hj = held_step(nst, f32)
    if hj < 0:
        assert not f32 and nst % 2 == 1  # odd bf16 steps add the warps' z one after another
        return
    wps = warps if f32 else warps // 2
    assert wps * C * 4 <= stage_bytes
    for gbase in (0, 5 * nst, 17 * nst):
        gl = gbase + hj
        held = {gl % stages} | ({(gl + 1) % stages} if hj + 1 < nst else set())
        assert len(held) == (2 if hj + 1 < nst else 1)
        written = {}
        for w in range(warps):
            sw = (gl if w < wps else gl + 1) % stages
            assert sw in held
            for lane in range(32):
                for i in range((C + 255) // 256):
                    c = 8 * lane + 256 * i
                    if c < C:
                        for k in range(8):
                            byte = (w % wps) * C * 4 + 4 * (c + k)
                            assert byte + 4 <= stage_bytes
                            key = (sw, byte)
                            assert key not in written
                            written[key] = (w, c + k)
        assert len(written) == warps * C
        reads = []
        for t in range(256):
            for c in range(8 * t, C, 8 * 256):
                for w in range(warps):
                    sw = (gl if w < wps else gl + 1) % stages
                    for k in range(8):
                        reads.append(written[(sw, (w % wps) * C * 4 + 4 * (c + k))])
        assert sorted(reads) == sorted(written.values())
