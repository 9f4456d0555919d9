"""Host-side checks of the streaming GEMV kernel's work partition (CPU only).

The kernel cuts each CTA's rows into per-team superblock ranges, the ranges into
row segments and the segments into ring stages of at most 4 segments. This
replays that index arithmetic (as the kernel states it) for the launch
configuration the library plans, and checks: every superblock is streamed by
exactly one team; each stage is one contiguous copy that fits its ring slot
and is a multiple of 16 bytes; every row is written exactly once, either by
the team holding a whole row segment or, for a row cut between teams, by the
team holding its first superblock, which adds the following teams' partials;
every lane's superblock index stays inside its stage; shared memory fits.
"""
import pytest

import gguf_quant_dequant_q4k_b200 as q4k
import q4k_synth

SEG = 4
SM_COUNT = 148
SMEM_OPTIN = 232448


def team_range(cluster_id, gteam, n, nsb, clusters, cluster, teams):
    """Superblock range of cluster-global team gteam (= cta_rank*teams + team)."""
    base, extra = n // clusters, n % clusters
    rows = base + (1 if cluster_id < extra else 0)
    row_begin = cluster_id * base + min(cluster_id, extra)
    S0, L = row_begin * nsb, rows * nsb
    nt = cluster * teams
    s0 = S0 + (L * gteam) // nt
    s1 = S0 + (L * (gteam + 1)) // nt
    if s1 > s0:
        row0 = s0 // nsb
        nseg = (s1 - 1) // nsb - row0 + 1
    else:
        row0, nseg = 0, 0
    return s0, s1, row0, nseg


def stream_regs(m, slices):
    """Registers per thread the kernel is compiled for (80 for one vector and
    one slice, else 128)."""
    threads = 640 if (m == 1 and slices == 1) else 480
    return 16384 // (((threads // 32 + 1 + 3) // 4) * 32) // 8 * 8


def lane_geometry(slices):
    """(quant bytes per lane and row, lanes per superblock, positions per
    warp): slices (1 or 2) 16-byte quant slices per lane."""
    lb = 16 * slices
    return lb, 128 // lb, 32 // (128 // lb)


def kernel_vectors(m):
    """Vectors one streaming launch carries: 1 or 2 (the streaming kernel runs
    m <= 2 for q4k_gemv, and pairs for the fused SwiGLU)."""
    return min(m, 2)


def max_nsb(mk, slices):
    threads = 640 if (mk == 1 and slices == 1) else 480
    return min((threads // 32) * lane_geometry(slices)[2], 80 * slices)


def k_chunk_nsbs(m, k):
    """Superblocks of each K-chunk the library launches for the first vector
    group: the fewest equal chunks one team covers (the last may be shorter)."""
    mk = kernel_vectors(m)
    nsb = k // 256
    top = max_nsb(mk, 2 if mk == 1 else 1)
    if nsb <= top:
        return [nsb]
    count = -(-nsb // top)
    per = -(-nsb // count)
    return [min(per, nsb - i * per) for i in range(count)]


def expected_launch(m, n, k, fused):
    """The launch policy the planner states: compact CTAs (at most 32768
    registers and 112 KiB of shared memory, two per SM) unless the matrix is
    very tall (512 or more rows per SM); two quant slices per lane for one
    vector on very tall matrices, for K beyond one-slice teams, or where a
    compact one-slice team would not fit. Returns (compact, slices, max compute
    warps, CTAs per SM, shared-memory cap)."""
    nsb = k // 256
    mi = kernel_vectors(m)
    tall = -(-n // SM_COUNT) >= 512
    cw = lambda regs: 32768 // (regs * 32) - 1
    compact_s1 = (not tall) and -(-nsb * 8 // 32) <= cw(stream_regs(mi, 1))
    compact_s2 = (not tall) and mi == 1 and not fused and -(-nsb * 4 // 32) <= cw(stream_regs(1, 2))
    compact = compact_s1 or compact_s2
    wide = mi == 1 and not fused and (tall or nsb > 80 or (compact and not compact_s1))
    sl = 2 if wide else 1
    maxw = cw(stream_regs(mi, sl)) if compact else (640 if (mi == 1 and sl == 1) else 480) // 32
    return compact, sl, maxw, (2 if compact else 1), (112 if compact else 220) * 1024


def seg_bounds(s0, s1, row0, i, nsb):
    return max(s0, (row0 + i) * nsb), min(s1, (row0 + i + 1) * nsb)


def check_plan(m, n, k):
    p = q4k.q4k_gemv_plan_for(m, n, k, SM_COUNT)
    if p["kernel"] != q4k.Q4K_KERNEL_STREAM:
        return p
    chunks = k_chunk_nsbs(m, k)
    mk0 = kernel_vectors(m)
    groups = -(-m // mk0)
    assert p["launches"] == groups * len(chunks)
    assert sum(chunks) == k // 256 and max(chunks) <= max_nsb(mk0, p["slices"])
    m = mk0
    if len(chunks) > 1:
        # every K-chunk is a launch on rows of chunk length (the partition below
        # is the first chunk's; the last chunk's is checked as its own plan)
        if chunks[-1] != chunks[0]:
            check_plan(m, n, chunks[-1] * 256)
        k = chunks[0] * 256
    nsb = k // 256
    ctas, teams, depth, cluster = p["grid"], p["teams"], p["depth"], p["cluster"]
    assert cluster in (1, 2) and ctas % cluster == 0
    clusters = ctas // cluster
    assert clusters <= n
    slices = p["slices"]                     # 16-byte quant slices per lane (0: one 8-byte half)
    compact, exp_slices, maxw, per_sm, smem_cap = expected_launch(m, n, k, False)
    assert slices == exp_slices
    assert clusters <= per_sm * SM_COUNT
    lb, lanes_sb, pos = lane_geometry(slices)
    team_warps = -(-nsb * lanes_sb // 32)
    assert team_warps * pos >= nsb            # a team's lanes cover every superblock position
    assert p["block"] == teams * team_warps * 32 + 32      # + one producer warp
    assert p["block"] <= maxw * 32 + 32
    mk = m
    if compact:   # a compact CTA leaves room for one of the next kernel beside it
        assert p["block"] * stream_regs(mk, slices) <= 32768
    assert 2 <= depth <= 8 and 1 <= teams <= 20
    stage_bytes = -(-SEG * nsb * 144 // 128) * 128
    # [seg][positions][4 groups] float4 coefficients + float2 rounding errors
    coef_per_warp = SEG * pos * 4 * (16 + 8)
    need = (teams * depth * stage_bytes + teams * team_warps * coef_per_warp
            + teams * depth * 2 * team_warps * SEG * mk * 4 + teams * 2 * mk * 4)
    need = -(-need // 16) * 16 + cluster * teams * 32 + teams * 2 * depth * 8
    assert p["smem_bytes"] == need and need <= smem_cap - 1024
    covered = [0] * (n * nsb)
    writes = [0] * n
    for q in range(clusters):
        # every team of the cluster, in cluster-global order (rank-major)
        ranges = [team_range(q, g, n, nsb, clusters, cluster, teams)
                  for g in range(cluster * teams)]
        for t, (s0, s1, row0, nseg) in enumerate(ranges):
            for sb in range(s0, s1):
                covered[sb] += 1
            nstages = -(-nseg // SEG)
            for s in range(nstages):
                i0 = s * SEG
                nseg_s = min(SEG, nseg - i0)
                b, _ = seg_bounds(s0, s1, row0, i0, nsb)
                _, e = seg_bounds(s0, s1, row0, i0 + nseg_s - 1, nsb)
                nbytes = (e - b) * 144
                assert 0 < nbytes <= stage_bytes and nbytes % 16 == 0
                # every lane's superblock in each segment lies inside the stage
                for u in range(nseg_s):
                    sb_b, sb_e = seg_bounds(s0, s1, row0, i0 + u, nsb)
                    assert b <= sb_b < sb_e <= e
            for i in range(nseg):
                row = row0 + i
                sb_b, sb_e = seg_bounds(s0, s1, row0, i, nsb)
                rb, re = sb_b - row * nsb, sb_e - row * nsb
                if rb == 0 and re == nsb:
                    writes[row] += 1
                elif rb > 0:
                    assert i == 0, "a contributor partial must be the team's first segment"
                else:
                    assert i == nseg - 1, "an owner partial must be the team's last segment"
            # finishing a row cut between teams
            if nseg:
                last = row0 + nseg - 1
                lb, le = seg_bounds(s0, s1, row0, nseg - 1, nsb)
                lb, le = lb - last * nsb, le - last * nsb
                if lb == 0 and le < nsb:
                    got = le
                    for t2 in range(t + 1, cluster * teams):
                        o0, o1, _, _ = ranges[t2]
                        if o0 >= (last + 1) * nsb:
                            break
                        if o1 <= o0:
                            continue
                        assert o0 == last * nsb + got, "contributors must be contiguous"
                        got = min(o1, (last + 1) * nsb) - last * nsb
                    assert got == nsb, "a cut row's partials must cover the whole row"
                    writes[last] += 1
    assert all(c == 1 for c in covered), "every superblock streamed exactly once"
    assert all(w == 1 for w in writes), "every row written exactly once"
    return p


SHAPES = (q4k_synth.SHAPES_TINY + q4k_synth.SHAPES_1P5B + q4k_synth.SHAPES_7B
          + [(4096, 14336), (1024, 4096), (14336, 4096), (128256, 4096), (75776, 4096),
             (75628, 4096), (151936, 1536), (100000, 20480), (1000, 28672), (64, 30720),
             (8192, 28672), (2, 30720), (7, 20736), (150, 23040)]
          + [(1, 256), (2, 256), (5, 512), (7, 768), (31, 1280), (33, 2304), (37, 8960),
             (129, 256), (1, 14336), (3, 11008), (97, 4352), (300, 3840), (149, 1024),
             (147, 20480), (1000, 20480), (77, 1536), (40, 4096), (200, 1792), (3, 20480),
             (150, 15360), (1, 4096), (8, 14336), (16, 8960), (63, 11008), (2, 1536)])


@pytest.mark.parametrize("n,k", SHAPES)
@pytest.mark.parametrize("m", [1, 2])
def test_stream_partition(m, n, k):
    check_plan(m, n, k)


def check_tc_plan(m, n, k):
    """m >= 3: the tensor-core kernel. One persistent CTA per SM at most, over
    128-row tiles; a digits launch and a GEMV launch per group of up to 16
    vectors; the stage ring (digit image of N x 256 fp16, 128 x 144 bytes of
    weights, 80 bytes of block metadata per vector) fits shared memory."""
    p = q4k.q4k_gemv_plan_for(m, n, k, SM_COUNT)
    assert p["kernel"] == q4k.Q4K_KERNEL_TC
    tiles, nsb = -(-n // 128), k // 256
    items = tiles * nsb                          # (128-row tile, superblock column)
    assert p["grid"] == min(items, SM_COUNT) and p["block"] == 480 and p["cluster"] == 1
    assert p["launches"] == 2 * -(-m // 16)
    mp = 8 if min(m, 16) <= 8 else 16
    n_mma = -(-5 * mp // 16) * 16
    wstages = 4 if mp == 8 else 3              # weight ring
    bstages = min(6, (212 * 1024 - wstages * 128 * 144 - 16 * mp * 80) // (n_mma * 512))   # digit images
    assert p["depth"] == wstages and bstages >= 3
    assert p["smem_bytes"] == (1024 + bstages * n_mma * 512 + 16 * mp * 80 + wstages * 128 * 144
                               + (2 * (bstages + 16 + wstages) + 11) * 8 + 16)
    assert p["smem_bytes"] <= 232448
    assert p["units"] == items and p["units_per_cta_max"] == -(-items // p["grid"])
    # equal contiguous ranges: every item owned once, counts differ by at most one
    ranges = [(items * c // p["grid"], items * (c + 1) // p["grid"]) for c in range(p["grid"])]
    assert ranges[0][0] == 0 and ranges[-1][1] == items
    assert all(r1 == s2 for (_, r1), (s2, _) in zip(ranges, ranges[1:]))
    assert max(b - a for a, b in ranges) - min(b - a for a, b in ranges) <= 1
    return p


def test_tc_balanced_items():
    """The tile x superblock items are shared out evenly over up to 148 CTAs:
    14336 x 4096 (1792 items) gives 12 or 13 per CTA, 1536 x 1536 (72 items)
    one per CTA."""
    p = q4k.q4k_gemv_plan_for(8, 14336, 4096, SM_COUNT)
    assert p["grid"] == SM_COUNT and p["units_per_cta_max"] == 13
    p = q4k.q4k_gemv_plan_for(8, 1536, 1536, SM_COUNT)
    assert p["grid"] == 72 and p["units_per_cta_max"] == 1


@pytest.mark.parametrize("n,k", SHAPES)
@pytest.mark.parametrize("m", [3, 4, 8, 9, 16, 17, 64])
def test_tc_plan(m, n, k):
    """Three or more vectors: the tensor-core kernel, except three or four on a
    shape the integer kernel takes."""
    if i8_expected(m, n, k):
        check_i8_plan(n, k, m)
    else:
        check_tc_plan(m, n, k)


def i8_whole(tiles):
    busiest = -(-tiles // SM_COUNT)
    return tiles >= SM_COUNT and busiest * SM_COUNT * 8 <= tiles * 9


def i8_config(n, k, m=1):
    """The integer kernel's launch for m <= 4 vectors of an n x k matrix (m = 3
    as four), or None: whole tiles per CTA (at least one 128-row tile per SM,
    the busiest CTA at most 1/8 above the mean) or at least 5 superblock
    columns per CTA on average; items of two superblock columns (padded at the
    end of a tile for an odd K/256 >= 9; never for four vectors, whose
    accumulators leave tensor memory for one) where four two-column weight
    stages fit beside the CTA's digit-image slots (an image of N x 256 bytes,
    N = 8 for one vector and 4 per vector otherwise, + 80 B of metadata per
    vector and column; 8 x 2 KB of header ring), else one column with 8, 6 or
    4 stages."""
    if not 1 <= m <= 4:
        return None
    mv = 1 if m == 1 else 2 if m == 2 else 4
    image, meta = (8 if mv == 1 else 4 * mv) * 256, 80 * mv
    tiles, nsb = -(-n // 128), k // 256
    whole = i8_whole(tiles)
    if not whole and tiles * nsb < 5 * SM_COUNT:
        return None
    # fewer tiles than SMs: one whole tile per CTA where that adds at most
    # 7 / 5 / 3 superblock columns (one / two / four vectors) to the busiest CTA
    if not whole and tiles < SM_COUNT and nsb * (SM_COUNT - tiles) <= {1: 7, 2: 5, 4: 3}[mv] * SM_COUNT:
        whole = True
    barriers = 2 * 8 + 4 + 2 * 4 + 2 * 8 + 1
    for cpi in ([2, 1] if mv < 4 and (nsb % 2 == 0 or nsb >= 9) else [1]):
        npi = -(-nsb // cpi)
        items = tiles * npi
        ctas = min(tiles, SM_COUNT) if whole else min(items, SM_COUNT)
        per = -(-tiles // ctas) * npi if whole else -(-items // ctas)
        ncols = min(per * cpi, npi * cpi)
        off = -(-(ncols * (image + meta) + 8 * 2048) // 1024) * 1024
        fit = (220 * 1024 - 1024 - off - barriers * 8 - 16) // (cpi * 128 * 144)
        if fit < 4:
            continue
        ws = 4 if cpi == 2 else 8 if fit >= 8 else 6 if fit >= 6 else 4
        smem = 1024 + off + ws * cpi * 128 * 144 + barriers * 8 + 16
        return dict(cpi=cpi, npi=npi, items=items, ctas=ctas, per=per, ncols=ncols, ws=ws, smem=smem,
                    whole=whole)
    return None


def i8_expected(m, n, k):
    return i8_config(n, k, m) is not None


def check_i8_plan(n, k, m=1):
    """One persistent CTA per SM at most over equal contiguous ranges of whole
    tiles or of items; 18 warps; the plan's smem, stages and per-CTA share as
    the launch rule above gives them."""
    p = q4k.q4k_gemv_plan_for(m, n, k, SM_COUNT)
    assert p["kernel"] == q4k.Q4K_KERNEL_I8, p
    c = i8_config(n, k, m)
    tiles, nsb = -(-n // 128), k // 256
    assert p["grid"] == c["ctas"] and p["block"] == 18 * 32 and p["cluster"] == 1 and p["launches"] == 1
    assert p["slices"] == c["cpi"] and p["depth"] == c["ws"] and p["smem_bytes"] == c["smem"] <= 220 * 1024
    assert p["units"] == tiles * nsb and p["units_per_cta_max"] == c["per"] * c["cpi"]
    npi, items = c["npi"], c["items"]
    if c["whole"]:
        ranges = [(tiles * q // p["grid"] * npi, tiles * (q + 1) // p["grid"] * npi) for q in range(p["grid"])]
        assert all(a % npi == 0 and b % npi == 0 for a, b in ranges)   # no tile is cut
    else:
        ranges = [(items * q // p["grid"], items * (q + 1) // p["grid"]) for q in range(p["grid"])]
        assert max(b - a for a, b in ranges) - min(b - a for a, b in ranges) <= 1
    assert ranges[0][0] == 0 and ranges[-1][1] == items
    assert all(r1 == s2 for (_, r1), (s2, _) in zip(ranges, ranges[1:]))
    # a CTA's digit-image slots cover every (padded) column of its range
    assert all(min((b - a) * c["cpi"], npi * c["cpi"]) <= c["ncols"] for a, b in ranges)
    return p


@pytest.mark.parametrize("n,k", SHAPES + [(148 * 128, 256), (296 * 128 - 51, 512), (1184 * 128 + 1, 4096),
                                          (160 * 128, 4096), (128256, 15872), (128256, 16128),
                                          (3000, 15872), (4096 + 77, 8192), (2048, 8192), (4096, 28672),
                                          (5000, 11008), (151553, 256), (8192, 28672), (18944, 15872)])
@pytest.mark.parametrize("m", [1, 2, 3, 4, 5])
def test_i8_choice(m, n, k):
    """Up to four vectors run on the integer tensor-core kernel where it pays;
    any other shape (or m) keeps its streaming / batched plan."""
    p = q4k.q4k_gemv_plan_for(m, n, k, SM_COUNT)
    if i8_expected(m, n, k):
        check_i8_plan(n, k, m)
    else:
        assert p["kernel"] != q4k.Q4K_KERNEL_I8, (m, n, k, p)


def test_i8_few_tiles_whole():
    """The 8B/7B FFN up projections (112 / 86 tiles): one whole tile per CTA on
    112 / 86 CTAs for one vector; two vectors keep it for 112 tiles only, four
    for neither (their columns cost more than the cut tiles' publication)."""
    for m, n, whole_ctas in [(1, 14336, 112), (1, 11008, 86), (2, 14336, 112), (2, 11008, None),
                             (4, 14336, None), (4, 11008, None)]:
        p = check_i8_plan(n, 4096, m)
        if whole_ctas:
            assert p["grid"] == whole_ctas and p["units_per_cta_max"] == 16, (m, n, p)
        else:
            assert p["grid"] == SM_COUNT, (m, n, p)


def test_i8_sweep_choice():
    """The decode sweep: the LM head (whole tiles) and the 7B/8B FFN
    projections (cut tiles) on the integer kernel, the smaller projections on
    the streaming kernel."""
    want = {(8960, 1536): 2, (1536, 8960): 2, (1536, 1536): 2, (11008, 4096): 4, (4096, 11008): 4,
            (4096, 4096): 2, (4096, 14336): 4, (128256, 4096): 4}
    for (n, k), kern in want.items():
        assert q4k.q4k_gemv_plan_for(1, n, k, SM_COUNT)["kernel"] == kern, (n, k)


def test_lm_head_partition():
    """The LM head (1002 tiles): 7 tiles on 114 CTAs, 6 on the other 34."""
    p = check_i8_plan(128256, 4096)
    assert p["units_per_cta_max"] == 7 * 16 and p["depth"] == 4 and p["slices"] == 2   # four stages of two columns
    # two vectors: the same items; four: one column per item, six stages beside a 70 KB image
    p = check_i8_plan(128256, 4096, 2)
    assert p["depth"] == 4 and p["slices"] == 2
    p = check_i8_plan(128256, 4096, 4)
    assert p["units_per_cta_max"] == 7 * 16 and p["depth"] == 6 and p["slices"] == 1
    # beyond the digit image's K the tall matrix streams with two-slice lanes
    p = check_plan(1, 128256, 20480)
    assert p["kernel"] == q4k.Q4K_KERNEL_STREAM and p["slices"] == 2


@pytest.mark.parametrize("n,k,cluster", [(1, 14336, 2), (7, 8192, 2), (1, 256, 1), (40, 4096, 1),
                                         (16, 8960, 1), (8, 14336, 1), (1, 7936, 1),
                                         (1536, 8960, 1), (4096, 4096, 1), (128256, 20480, 1)])
def test_cluster_choice(n, k, cluster):
    """N < 8 with K >= 8192 splits rows across the two CTAs of a cluster (split-K)."""
    p = check_plan(1, n, k)
    assert p["cluster"] == cluster, p


def test_kernel_choice():
    assert q4k.q4k_gemv_plan_for(1, 4096, 4096, SM_COUNT)["kernel"] == q4k.Q4K_KERNEL_STREAM
    assert q4k.q4k_gemv_plan_for(2, 4096, 4096, SM_COUNT)["kernel"] == q4k.Q4K_KERNEL_STREAM
    # two to four vectors on the larger projections: the integer kernel (W read once)
    for m in (2, 3, 4):
        assert q4k.q4k_gemv_plan_for(m, 4096, 14336, SM_COUNT)["kernel"] == q4k.Q4K_KERNEL_I8, m
    # three or more vectors: the tensor-core kernel (digits + GEMV per 16 vectors)
    for m, n, k in [(3, 4096, 4096), (8, 4096, 14336), (8, 14336, 4096), (5, 4096, 4096),
                    (16, 128256, 4096), (3, 64, 61696)]:
        p = q4k.q4k_gemv_plan_for(m, n, k, SM_COUNT)
        assert p["kernel"] == q4k.Q4K_KERNEL_TC and p["launches"] == 2, (m, n, k, p)
    assert q4k.q4k_gemv_plan_for(1, 64, 20480, SM_COUNT)["kernel"] == q4k.Q4K_KERNEL_STREAM
    # one vector, K beyond one-slice teams: two-slice teams up to K = 30720
    p = q4k.q4k_gemv_plan_for(1, 64, 20736, SM_COUNT)
    assert p["kernel"] == q4k.Q4K_KERNEL_STREAM and p["slices"] == 2 and p["launches"] == 1
    assert q4k.q4k_gemv_plan_for(1, 64, 30720, SM_COUNT)["launches"] == 1
    # beyond one team: K-chunks on the streaming kernel, never the general one
    for m, k, launches in [(1, 30976, 2), (1, 61440, 2), (1, 61696, 3), (2, 15360, 1),
                           (2, 15616, 2)]:
        p = q4k.q4k_gemv_plan_for(m, 64, k, SM_COUNT)
        assert p["kernel"] == q4k.Q4K_KERNEL_STREAM and p["launches"] == launches, (m, k, p)
    # the fused SwiGLU beyond the streaming range stays on the general kernel
    assert (q4k.q4k_gemv_swiglu_plan_for(1, 64, 20736, SM_COUNT)["kernel"]
            == q4k.Q4K_KERNEL_WARP_ROWS)


def test_batches_beyond_eight_vectors():
    """m > 16 runs as vector groups of 16 on the tensor-core kernel (the
    realizar page tiles batches); m > 64 is refused."""
    assert q4k.q4k_gemv_plan_for(16, 14336, 4096, SM_COUNT)["launches"] == 2
    assert q4k.q4k_gemv_plan_for(33, 4096, 4096, SM_COUNT)["launches"] == 6
    assert q4k.q4k_gemv_plan_for(64, 4096, 4096, SM_COUNT)["launches"] == 8
    p = q4k.q4k_gemv_plan_for(20, 64, 30976, SM_COUNT)
    assert p["kernel"] == q4k.Q4K_KERNEL_TC and p["launches"] == 4
    with pytest.raises(q4k.Q4KError):
        q4k.q4k_gemv_plan_for(65, 4096, 4096, SM_COUNT)


def check_fused_plan(m, n, k):
    """Fused gate/up SwiGLU: each CTA's gate rows followed by the same up rows
    form a virtual range of 2*rows rows that its teams cut; a stage crossing
    from gate into up rows is two copies. Checks: every virtual superblock is
    streamed once, every copy stays inside the CTA's rows of its matrix and is
    a multiple of 16 bytes, every virtual row is finished exactly once, and
    shared memory (with the row-total buffer) fits."""
    p = q4k.q4k_gemv_swiglu_plan_for(m, n, k, SM_COUNT)
    if p["kernel"] != q4k.Q4K_KERNEL_STREAM:
        return p
    nsb = k // 256
    ctas, teams, depth = p["grid"], p["teams"], p["depth"]
    compact, _, maxw, per_sm, smem_cap = expected_launch(m, n, k, True)
    assert p["cluster"] == 1 and ctas == min(n, per_sm * SM_COUNT)
    team_warps = -(-nsb * 8 // 32)
    assert teams * team_warps <= maxw
    assert p["block"] == teams * team_warps * 32 + 32
    stage_bytes = -(-SEG * nsb * 144 // 128) * 128
    rows_cap = -(-n // ctas)
    mi = min(m, 2)
    need = (teams * depth * stage_bytes + teams * team_warps * SEG * 4 * 4 * (16 + 8)
            + teams * depth * 2 * team_warps * SEG * mi * 4 + teams * 2 * mi * 4)
    need = -(-need // 16) * 16 + teams * 32 + teams * 2 * depth * 8
    need += -(-(mi * 2 * rows_cap * 4) // 16) * 16
    assert p["smem_bytes"] == need and need <= smem_cap - 1024
    base, extra = n // ctas, n % ctas
    gate_seen = [0] * (n * nsb)
    up_seen = [0] * (n * nsb)
    for q in range(ctas):
        rows = base + (1 if q < extra else 0)
        row0 = q * base + min(q, extra)
        L = 2 * rows * nsb
        bound = rows * nsb
        writes = [0] * (2 * rows)
        ranges = []
        for t in range(teams):
            s0, s1 = L * t // teams, L * (t + 1) // teams
            ranges.append((s0, s1))
        for t, (s0, s1) in enumerate(ranges):
            if s1 <= s0:
                continue
            rbase = s0 // nsb
            nseg = (s1 - 1) // nsb - rbase + 1
            for st in range(-(-nseg // SEG)):
                vs = max(s0, (rbase + st * SEG) * nsb)
                ve = min(s1, (rbase + st * SEG + SEG) * nsb)
                assert 0 < (ve - vs) * 144 <= stage_bytes
                pieces = []
                if vs < bound:
                    pieces.append(("gate", vs, min(ve, bound)))
                if ve > bound:
                    pieces.append(("up", max(vs, bound) - bound, ve - bound))
                for which, a, b in pieces:
                    assert 0 <= a < b <= rows * nsb and ((b - a) * 144) % 16 == 0
                    seen = gate_seen if which == "gate" else up_seen
                    for sb in range(a, b):
                        seen[row0 * nsb + sb] += 1
            for i in range(nseg):
                v = rbase + i
                b_, e_ = max(s0, v * nsb) - v * nsb, min(s1, (v + 1) * nsb) - v * nsb
                if b_ == 0 and e_ == nsb:
                    writes[v] += 1
                elif b_ == 0:          # this team holds the row's first superblock
                    writes[v] += 1
        assert all(w == 1 for w in writes), (q, writes)
    assert all(c == 1 for c in gate_seen) and all(c == 1 for c in up_seen)
    return p


@pytest.mark.parametrize("n,k", [(14336, 4096), (11008, 4096), (8960, 1536), (1, 256), (3, 4096),
                                 (149, 1024), (300, 3840), (1000, 20480), (7, 14336)])
@pytest.mark.parametrize("m", [1, 2, 3])
def test_fused_partition(m, n, k):
    check_fused_plan(m, n, k)


def test_fused_falls_back_beyond_the_stream_range():
    assert q4k.q4k_gemv_swiglu_plan_for(1, 64, 20736, SM_COUNT)["kernel"] == q4k.Q4K_KERNEL_WARP_ROWS
    assert q4k.q4k_gemv_swiglu_plan_for(1, 64, 20480, SM_COUNT)["kernel"] == q4k.Q4K_KERNEL_STREAM
    assert q4k.q4k_gemv_swiglu_plan_for(1, 7, 14336, SM_COUNT)["cluster"] == 1
