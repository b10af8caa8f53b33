"""CPU models of the kernels' index arithmetic (no GPU).

Each test restates, in Python, the address formulas and constants of a kernel
(ks_fma32.cu, ks_tc.cu) and checks the properties the kernel relies on:
every output owned or written exactly once, copies that cover a stage exactly
once, and shared-memory accesses that stay within one wavefront (fp32
operands) or reach eight distinct bank groups per quarter-warp (16-byte
accesses of the tcgen05 transposer).  They were run before each kernel's
first GPU run; kept here so a change to the formulas must change them too.
"""
import collections
import math
import os
import re

import pytest

# --------------------------------------------------------------- ks_fma32.cu
KJT = 8
THREADS = 256
FMA32_TILES = [(8, 2, 4, 16), (8, 4, 2, 16), (8, 2, 4, 12), (8, 4, 2, 12), (4, 2, 4, 16), (4, 1, 8, 16),
               (4, 4, 2, 16), (4, 2, 4, 12), (4, 1, 8, 12), (2, 2, 4, 16), (2, 4, 2, 16), (2, 8, 1, 16),
               (2, 2, 4, 12), (2, 4, 2, 12), (1, 4, 2, 16), (1, 8, 1, 16), (1, 2, 4, 16), (1, 4, 2, 12),
               (1, 8, 1, 12)]


def fma32_geometry(dl, wm, wk, tn):
    kq = 2 if dl == 2 else 4 if dl == 1 else 1
    rg = 32 // (dl * kq)
    ra = {8: 72, 4: 36, 2: 20, 1: 12}[dl]
    bm, kw = 8 * rg * wm, kq * tn
    bkl = kw * wk
    bkp = bkl + 4
    psb = KJT * bkp + (8 if dl == 2 else 4)
    return dict(kq=kq, rg=rg, ra=ra, bm=bm, kw=kw, bkl=bkl, bkp=bkp, psb=psb, a_words=bm * ra)


def wavefronts(addrs, width):
    """Shared-memory wavefronts one warp access needs (distinct word addresses,
    `width` consecutive words each; identical addresses are broadcast)."""
    banks = collections.defaultdict(set)
    for a in set(addrs):
        for w in range(width):
            banks[(a + w) % 32].add((a + w) // 32)
    return max(len(v) for v in banks.values())


@pytest.mark.parametrize("tile", FMA32_TILES)
def test_fma32_lanes_own_each_output_once_and_loads_are_one_wavefront(tile):
    dl, wm, wk, tn = tile
    g = fma32_geometry(*tile)
    owned = collections.Counter()
    for warp in range(8):
        w_m, w_k = warp // wk, warp % wk
        roles = []
        for lane in range(32):
            c_kq, c_l, c_rg = lane % g["kq"], (lane // g["kq"]) % dl, lane // (g["kq"] * dl)
            a_row, b_col = w_m * 8 * g["rg"] + c_rg, w_k * g["kw"] + 4 * c_kq
            roles.append((a_row, b_col, c_l))
            for m in range(8):
                for q in range(tn // 4):
                    for e in range(4):
                        owned[(a_row + g["rg"] * m, b_col + 4 * g["kq"] * q + e, c_l)] += 1
        for jj in range(KJT):
            for m in range(8):  # one scalar X load per (jj, m): As[row][jj * DL + l]
                xs = [(r + g["rg"] * m) * g["ra"] + jj * dl + l for (r, _, l) in roles]
                assert wavefronts(xs, 1) == 1
            for q in range(tn // 4):  # one 16-byte values load per (jj, q): Bs[l][jj][k..k+3]
                vs = [g["a_words"] + l * g["psb"] + c + jj * g["bkp"] + 4 * g["kq"] * q for (_, c, l) in roles]
                assert wavefronts(vs, 4) == 1
    assert len(owned) == g["bm"] * g["bkl"] * dl and set(owned.values()) == {1}


@pytest.mark.parametrize("tile", FMA32_TILES)
def test_fma32_copies_cover_a_stage_once(tile):
    dl, wm, wk, tn = tile
    g = fma32_geometry(*tile)
    bm, bkl, ra, bkp, psb, a_words = g["bm"], g["bkl"], g["ra"], g["bkp"], g["psb"], g["a_words"]
    ca = 2 * dl
    nxc, xr = (bm * ca + THREADS - 1) // THREADS, THREADS // ca
    nv = (dl * bkl * KJT + THREADS - 1) // THREADS
    k4 = bkl // 4
    nvt = (dl * KJT * k4 + THREADS - 1) // THREADS
    vk = THREADS // 8
    xs, vs, vts = collections.Counter(), collections.Counter(), collections.Counter()
    for tid in range(THREADS):
        xn, xf = tid // ca, 4 * (tid % ca)
        for t in range(nxc):
            if nxc * THREADS == bm * ca or xn + t * xr < bm:
                for e in range(4):
                    xs[(xn + t * xr) * ra + xf + e] += 1
        vj, kq = tid % 8, tid >> 3
        for t in range(nv):  # 4-byte values copies, transposing [k][j] -> [j][k]
            if bkl % vk == 0:
                kc, l = (vk * t) % bkl, (vk * t) // bkl
            else:
                e8 = kq + vk * t
                l, kc = e8 // bkl, e8 % bkl - kq
            if bkl % vk == 0 or nv * THREADS == dl * bkl * KJT or kq + vk * t < dl * bkl:
                vs[a_words + vj * bkp + kq + l * psb + kc] += 1
        for t in range(nvt):  # 16-byte copies from the transposed values
            e = tid + t * THREADS
            if nvt * THREADS == dl * KJT * k4 or e < dl * KJT * k4:
                kk4, jl = e % k4, e // k4
                j, l = jl % KJT, jl // KJT
                for q in range(4):
                    vts[a_words + l * psb + j * bkp + 4 * kk4 + q] += 1
    x_expect = {r * ra + c for r in range(bm) for c in range(KJT * dl)}
    v_expect = {a_words + l * psb + j * bkp + k for l in range(dl) for j in range(KJT) for k in range(bkl)}
    assert set(xs) == x_expect and set(xs.values()) == {1}
    assert set(vs) == v_expect and set(vs.values()) == {1}
    assert set(vts) == v_expect and set(vts.values()) == {1}


def fma32_source():
    path = os.path.join(os.path.dirname(__file__), "..", "kronecker_sparse_matrix_b200", "csrc", "ks_fma32.cu")
    with open(path) as f:
        return f.read()


def test_fma32_copy_warpgroup_roles_barriers_and_register_split():
    """The copy warpgroup's threads take each of a stage's 256 copy roles once,
    the barrier counts match the arrivals, and the setmaxnreg split fits the
    registers the block is launched with (a split above it would wait forever)."""
    src = fma32_source()
    threads = int(re.search(r"constexpr int kThreads = (\d+);", src).group(1))
    roles = int(re.search(r"constexpr int kCopyRoles = (\d+);", src).group(1))
    assert roles == THREADS and threads % 128 == 0
    compute = 256  # warps 0-7 compute, warps 8.. issue copies
    copy = threads - compute
    # copy thread pt plays roles pt + copy * v, v < roles / copy
    got = collections.Counter(pt + copy * v for pt in range(copy) for v in range(roles // copy))
    assert roles % copy == 0 and set(got) == set(range(roles)) and set(got.values()) == {1}
    # every copy thread makes one .noinc arrival per stage; every compute warp one arrival
    full = int(re.search(r"mbar_init\(&full_bar\[s\], (\d+)\)", src).group(1))
    empty = int(re.search(r"mbar_init\(&empty_bar\[s\], (\d+)\)", src).group(1))
    assert full == copy and empty == compute // 32
    dec = int(re.search(r"setmaxnreg\.dec\.sync\.aligned\.u32 (\d+)", src).group(1))
    inc = int(re.search(r"setmaxnreg\.inc\.sync\.aligned\.u32 (\d+)", src).group(1))
    # registers per thread at launch: 64K per SM over the launch bound, in units of 8
    launch = (65536 // threads) // 8 * 8
    assert dec % 8 == 0 and inc % 8 == 0 and 24 <= dec <= 256 and 24 <= inc <= 256
    assert copy * dec + compute * inc <= threads * launch


# ------------------------------------------------------------------ ks_tc.cu
# es = element bytes: 2 (bf16, kind::f16) or 4 (fp32 read as TF32, kind::tf32).
def chunk_j(dls, es=2):
    return 16 if dls == 16 else (32 if dls == 8 else 128 // dls) // es


def tc_dls(p, es):
    """l per tile: 16 for bf16 with d % 64 == 0 and c <= 96, or d = 16 and b %
    32 != 0; 8 for d % 8 == 0; else d."""
    a, b, c, d = p
    if es == 2 and d % 16 == 0 and ((d % 64 == 0 and c <= 96) or (d == 16 and b % 32)):
        return 16
    return 8 if d % 8 == 0 else d


def group_stride(es):
    return 144 if es == 2 else 256


def octet_stride(es):
    return 16 * 144 if es == 2 else 128 * 32


def plane_stride(dls, es):
    return (chunk_j(dls, es) // 8) * octet_stride(es)


def slot_bytes(dls, es):
    raw = 128 * chunk_j(dls, es) * dls * es
    return (raw if dls in (1, 16) else dls * plane_stride(dls, es) + 1023) // 1024 * 1024


def tc_task_unit(dls, task, units):
    """bf16 transposer: task -> (raw unit q, group g of 8 rows)."""
    if dls == 8:
        return task % units, task // units
    q = task & 7
    return q, ((task >> 3) + (q >> (1 if dls == 2 else 2))) & 15


def bf16_transposer_writes(dls):
    """(q, g, e) -> plane address of output unit e of a bf16 task."""
    es, ctj = 2, chunk_j(dls, 2)
    out = {}
    for q in range(ctj * dls * es // 16):
        for g in range(16):
            for e in range(8):
                f = 8 * q + e
                j, l = f // dls, f % dls
                out[(q, g, e)] = l * plane_stride(dls, es) + (j >> 3) * octet_stride(es) + g * group_stride(es) + \
                    (j & 7) * 16
    return out


@pytest.mark.parametrize("dls", [2, 4, 8])
def test_tc_bf16_transposer_quarter_warps_reach_eight_bank_groups(dls):
    es, ctj = 2, chunk_j(dls, 2)
    units = ctj * dls * es // 16
    tasks = 16 * units // 128
    slot = slot_bytes(dls, es)
    assert slot >= 128 * ctj * dls * es  # the in-place planes cover the raw chunk
    wr = bf16_transposer_writes(dls)
    written, mapped = set(), set()
    for k in range(tasks):
        for t0 in range(0, 128, 8):  # one quarter-warp: 8 consecutive lanes
            qg = [tc_task_unit(dls, t + 128 * k, units) for t in range(t0, t0 + 8)]
            for r in range(8):  # reads of the raw chunk
                groups = {((g * 8 + r) * units + q) % 8 for q, g in qg}
                assert len(groups) == 8
            for e in range(8):  # writes of the padded planes
                addrs = []
                for q, g in qg:
                    a = wr[(q, g, e)]
                    assert 0 <= a and a + 16 <= slot and a not in written
                    written.add(a)
                    addrs.append(a)
                assert len({(a // 16) % 8 for a in addrs}) == 8
            mapped.update(qg)
    assert len(mapped) == tasks * 128 and all(0 <= q < units and 0 <= g < 16 for q, g in mapped)


@pytest.mark.parametrize("dls", [2, 4, 8])
def test_tc_bf16_mma_descriptor_reads_what_the_transposer_wrote(dls):
    """bf16 A operand of one MMA (plane l, K step s): the canonical MN-major
    no-swizzle layout, element (row m, k) at start + (m // 8) * SBO +
    (k // 8) * LBO + (k % 8) * 16 + (m % 8) * 2, start = l * PS + 2 s OS,
    LBO = OS, SBO = GS; it must land on X[row m][j = 16 s + k][l]."""
    es, ctj = 2, chunk_j(dls, 2)
    wr = bf16_transposer_writes(dls)
    where = {}
    for (q, g, e), a in wr.items():
        f = 8 * q + e
        j, l = f // dls, f % dls
        for r in range(8):
            where[(g * 8 + r, j, l)] = a + r * es
    assert len(where) == 128 * ctj * dls and len(set(where.values())) == len(where)
    os_, gs, ps = octet_stride(es), group_stride(es), plane_stride(dls, es)
    for l in range(dls):
        for s in range(ctj // 16):
            start = l * ps + 2 * s * os_
            for m in range(128):
                for k in range(16):
                    addr = start + (m // 8) * gs + (k // 8) * os_ + (k % 8) * 16 + (m % 8) * es
                    assert addr == where[(m, 16 * s + k, l)]


def dls16_transposer():
    """bf16 with 16 l: warp tw, group g = 4 it + tw; lane -> raw unit q =
    (j, l half h); reads rows r of unit q, writes line (l = 8 h + e, j) of the
    group's planes.  Returns per group the lanes' (read addresses per r,
    write addresses per e, j, h), addresses relative to the slot."""
    g16 = 4096
    out = {}
    for tw in range(4):
        for it in range(4):
            g = 4 * it + tw
            lanes = []
            for lane in range(32):
                quarter, idx = lane >> 3, lane & 7
                h = (idx >> 2) ^ (quarter & 1)
                j = 8 * (quarter >> 1) + idx
                q = 2 * j + h
                reads = [g * g16 + r * 512 + q * 16 for r in range(8)]
                writes = [g * g16 + (2 * (8 * h + e) + (j >> 3)) * 128 + (j & 7) * 16 for e in range(8)]
                lanes.append((reads, writes, j, h, q))
            out[g] = lanes
    return out


def test_tc_bf16_dls16_transposer_is_in_place_and_conflict_free():
    """Each warp's group: the lanes' units cover the 8 rows' 4 KB once, the
    writes land inside the same 4 KB, once each, and every quarter-warp's
    16-byte reads and writes reach eight distinct bank groups."""
    slot = slot_bytes(16, 2)
    assert slot == 128 * 512 == 128 * chunk_j(16, 2) * 16 * 2
    tr = dls16_transposer()
    assert sorted(tr) == list(range(16))
    for g, lanes in tr.items():
        assert sorted(q for *_, q in lanes) == list(range(32))
        lo, hi = g * 4096, g * 4096 + 4096
        reads = [a for rd, *_ in lanes for a in rd]
        writes = [a for _, wr, *_ in lanes for a in wr]
        assert sorted(reads) == list(range(lo, hi, 16)) and sorted(writes) == list(range(lo, hi, 16))
        for q0 in range(0, 32, 8):
            quarter = lanes[q0:q0 + 8]
            for r in range(8):
                assert len({(rd[r] // 16) % 8 for rd, *_ in quarter}) == 8
            for e in range(8):
                assert len({(wr[e] // 16) % 8 for _, wr, *_ in quarter}) == 8


def test_tc_bf16_dls16_mma_descriptor_reads_what_the_transposer_wrote():
    """Plane l's A operand for the chunk's one K step: MN-major no swizzle,
    element (row m, k) at l * 256 + (m // 8) * SBO + (k // 8) * LBO + (k % 8) *
    16 + (m % 8) * 2 with LBO = 128, SBO = 4096; it must hold X[row m][j = k][l]."""
    where = {}
    for g, lanes in dls16_transposer().items():
        for reads, writes, j, h, q in lanes:
            for e in range(8):
                for r in range(8):  # line e holds element e of unit q for rows 0..7
                    where[(8 * g + r, j, 8 * h + e)] = writes[e] + 2 * r
    assert len(where) == 128 * 16 * 16 and len(set(where.values())) == len(where)
    for l in range(16):
        for m in range(128):
            for k in range(16):
                addr = l * 256 + (m // 8) * 4096 + (k // 8) * 128 + (k % 8) * 16 + (m % 8) * 2
                assert addr == where[(m, k, l)]
    # the raw row is [j][l], 16 l per j: unit q = 2 j + h holds l = 8 h .. 8 h + 7
    for g, lanes in dls16_transposer().items():
        for reads, writes, j, h, q in lanes:
            assert q * 16 == (j * 16 + 8 * h) * 2


# ------------------------------------------------------------- ks_dv_tc.cu
def dv_tc_transposer(mn_rows):
    """The bf16 dV kernel's transposer for one operand of a stage (16 rows n):
    raw [n][mn][8 l] (16-byte unit = 8 l) -> per-l K-major planes with the
    32-byte swizzle, row mn = 32 bytes (16 n), half h of row mn at
    h ^ bit 2 of mn.  Task = (mn, row half nh) for tasks t < 2 * mn_rows
    (A: t = thread + 128 nh, mn = thread; B: mn = t % c, nh = t // c).
    Returns per task its raw read addresses (8 units) and its 8 writes (l)."""
    plane = mn_rows * 32
    out = {}
    for t in range(2 * mn_rows):
        mn, nh = (t % 128, t // 128) if mn_rows == 128 else (t % mn_rows, t // mn_rows)
        reads = [((8 * nh + r) * mn_rows + mn) * 16 for r in range(8)]
        writes = [e * plane + mn * 32 + ((nh ^ ((mn >> 2) & 1)) << 4) for e in range(8)]
        out[t] = (mn, nh, reads, writes)
    return out


@pytest.mark.parametrize("mn_rows", [128, 64, 48, 32, 16])
def test_dv_tc_transposer_is_in_place_and_matches_the_k_major_descriptor(mn_rows):
    """Both operands of the dV kernel: every raw unit read once, every plane
    unit written once inside the raw stage, quarter-warps reach eight bank
    groups on reads (and on writes except where a quarter-warp straddles the
    row halves of a narrow operand), and the K-major 32-byte-swizzle
    descriptor (SBO = 256 bytes) reads X[n][mn][l] at element (mn, n)."""
    tr = dv_tc_transposer(mn_rows)
    raw = 16 * mn_rows * 16
    reads = sorted(a for v in tr.values() for a in v[2])
    writes = sorted(a for v in tr.values() for a in v[3])
    assert reads == list(range(0, raw, 16)) and writes == list(range(0, raw, 16))
    for t0 in range(0, len(tr), 8):
        q = [tr[t] for t in range(t0, min(t0 + 8, len(tr)))]
        for r in range(8):
            assert len({(v[2][r] // 16) % 8 for v in q}) == len(q)
        if all(v[1] == q[0][1] for v in q):
            for e in range(8):
                assert len({(v[3][e] // 16) % 8 for v in q}) == len(q)
    where = {}
    for mn, nh, rd, wr in tr.values():
        for e in range(8):
            for h in range(8):
                where[(mn, 8 * nh + h, e)] = wr[e] + 2 * h
    for l in range(8):
        for mn in range(mn_rows):
            for k in range(16):
                a = mn * 32 + (k // 8) * 16 + (k % 8) * 2
                a ^= ((a >> 7) & 1) << 4  # the 32-byte swizzle: bit 4 ^= bit 7
                assert l * mn_rows * 32 + a == where[(mn, k, l)]


def tf32_tasks(dls):
    """The fp32 transposer of ks_tc.cu, modelled per thread t (0..127) and task
    k: the raw addresses it reads (one list per load instruction) and, per
    output unit, the plane address and the (row, j, l) of its four words."""
    ctj = chunk_j(dls, 4)
    jqn, lqn = ctj // 4, (2 if dls == 8 else 1)
    tpr = jqn * lqn
    rb = ctj * dls * 4
    ps, os_ = plane_stride(dls, 4), octet_stride(4)
    out = {}
    for t in range(128):
        for k in range(tpr):
            task = t + 128 * k
            lq, jq, n = task % lqn, (task // lqn) % jqn, task // tpr
            reads, units = [], []
            if dls == 2:
                sw = n & 1
                reads = [n * rb + (2 * jq + sw) * 16, n * rb + (2 * jq + 1 - sw) * 16]
                words = {0: [(n, 4 * jq + w, 0) for w in range(4)], 1: [(n, 4 * jq + w, 1) for w in range(4)]}
                les = [0, 1]
            else:
                rot = ((jq + 2 * (n & 1)) & 3) if dls == 8 else (n & 3)
                for i in range(4):
                    j = 4 * jq + ((i + rot) & 3)
                    reads.append(n * rb + (j * (dls // 4) + lq) * 16)
                words = {e: [(n, 4 * jq + w, 4 * lq + e) for w in range(4)] for e in range(4)}
                les = [0, 1, 2, 3]
            half = (jq & 1) ^ ((n >> 2) & 1)
            for e in les:
                addr = (jq >> 1) * os_ + n * 32 + half * 16 + (4 * lq + e) * ps
                units.append((addr, words[e]))
            out[(t, k)] = (reads, units)
    return out, tpr


@pytest.mark.parametrize("dls", [2, 4, 8])
def test_tc_tf32_transposer_covers_the_planes_and_spreads_bank_groups(dls):
    """Every element of the raw chunk lands once in the planes, which fit the
    slot; each quarter-warp's reads reach eight bank groups, its writes at
    least four (a 16-byte store of eight lanes in at most two wavefronts)."""
    ctj = chunk_j(dls, 4)
    tasks, tpr = tf32_tasks(dls)
    slot = slot_bytes(dls, 4)
    placed = {}
    for (t, k), (reads, units) in tasks.items():
        for addr, words in units:
            assert 0 <= addr and addr + 16 <= slot
            for w, elem in enumerate(words):
                assert elem not in placed
                placed[elem] = addr + 4 * w
    assert len(placed) == 128 * ctj * dls and len(set(placed.values())) == len(placed)
    for k in range(tpr):
        for t0 in range(0, 128, 8):
            lanes = [tasks[(t, k)] for t in range(t0, t0 + 8)]
            for i in range(len(lanes[0][0])):
                assert len({(r[0][i] // 16) % 8 for r in lanes}) == 8
            for u in range(len(lanes[0][1])):
                groups = [(r[1][u][0] // 16) % 8 for r in lanes]
                assert max(groups.count(g) for g in groups) <= 2


def test_tc_tf32_raw_reads_pick_the_right_elements():
    """The raw chunk holds row n's (j, l) at n * rb + (j * dls + l) * 4; the
    words the model assigns to each output unit are the ones the reads fetch."""
    for dls in (2, 4, 8):
        ctj = chunk_j(dls, 4)
        rb = ctj * dls * 4
        tasks, _ = tf32_tasks(dls)
        for (t, k), (reads, units) in tasks.items():
            fetched = set()
            for r in reads:
                n, off = divmod(r, rb)
                for w in range(4):
                    f = off // 4 + w
                    fetched.add((n, f // dls, f % dls))
            assert fetched == {elem for _, words in units for elem in words}


@pytest.mark.parametrize("dls", [2, 4, 8])
def test_tc_tf32_mma_descriptor_reads_what_the_transposer_wrote(dls):
    """TF32 A operand of one MMA (plane l, K step s): the canonical K-major
    layout with the 32-byte swizzle, element (row m, k) at start + (m // 8) *
    SBO + (m % 8) * 32 + k * 4 with address bit 4 flipped by bit 7 (within
    the 256-byte atom), start = l * PS + s * OS (256-byte aligned), SBO = 256.
    It must land on X[row m][j = 8 s + k][l]."""
    ctj = chunk_j(dls, 4)
    tasks, _ = tf32_tasks(dls)
    placed = {}
    for reads, units in tasks.values():
        for addr, words in units:
            for w, elem in enumerate(words):
                placed[elem] = addr + 4 * w
    ps, os_ = plane_stride(dls, 4), octet_stride(4)
    for l in range(dls):
        for s in range(ctj // 8):
            start = l * ps + s * os_
            assert start % 256 == 0
            for m in range(128):
                for k in range(8):
                    addr = start + (m // 8) * 256 + (m % 8) * 32 + k * 4
                    addr ^= ((addr >> 7) & 1) << 4
                    assert addr == placed[(m, 8 * s + k, l)]


def tc_bp(dls, b):
    for bp in range(min(256, 512 // dls), 15, -16):
        if b % bp == 0:
            return bp
    return 0


def tc_kc(dls, bp, es=2):
    ce = 128 // es
    kcm = ce // dls
    lw = min(8, kcm)
    for kc in range(min(bp, kcm) // lw * lw, lw - 1, -lw):
        if bp % kc == 0 and dls * kc == ce:
            return kc
    for kc in range(min(bp, kcm) // lw * lw, lw - 1, -lw):
        if bp % kc == 0:
            return kc
    return 0


@pytest.mark.parametrize("es", [2, 4])
@pytest.mark.parametrize("p", [(2, 48, 48, 2), (1, 48, 48, 4), (2, 64, 64, 16), (1, 192, 48, 8), (3, 32, 16, 4),
                               (1, 256, 256, 2), (2, 48, 48, 1), (1, 16, 16, 1), (1, 96, 96, 4), (1, 80, 16, 2),
                               (1, 48, 8, 1), (2, 256, 64, 16), (1, 48, 48, 32), (2, 96, 64, 64), (1, 48, 32, 16),
                               (1, 48, 48, 64), (1, 192, 48, 64)])
def test_tc_epilogue_writes_each_output_once(p, es):
    """The output boxes of a tile: 32 rows x (DLS * kc) elements per warp and
    chunk, either one tensor store of a contiguous box (d == DLS), one 4-D
    tensor store of a [k][row][l] box (32-byte l runs, d > DLS) or 16-byte stores of its
    units; N = 300 leaves a ragged last row block."""
    a, b, c, d = p
    dls = tc_dls(p, es)
    bp = tc_bp(dls, b)
    kc = tc_kc(dls, bp, es)
    assert kc > 0 and bp % kc == 0 and dls * kc * es <= 128
    rpu = 16 // es
    n, out_f = 300, a * b * d
    units = dls * kc * es // 16
    written = collections.Counter()
    for i in range(a):
        for gl in range(d // dls):
            l0 = gl * dls
            for ps in range(b // bp):
                for oc in range(bp // kc):
                    kq = ps * bp + oc * kc
                    ybase = i * b * d + l0
                    for rb in range(math.ceil(n / 128)):
                        for quad in range(4):
                            row0 = rb * 128 + 32 * quad
                            if d == dls:  # one box: rows row0.., columns ybase + kq*d ..
                                if row0 >= n:
                                    continue
                                x = ybase + kq * d
                                assert (x * es) % 16 == 0
                                for r in range(min(32, n - row0)):
                                    for e in range(dls * kc):
                                        written[(row0 + r, x + e)] += 1
                            elif dls * es == 32:  # one 4-D box [k][row][l] of Y viewed as (d, N, b, a)
                                if row0 >= n:
                                    continue
                                assert (l0 * es) % 16 == 0 and kq + kc <= b
                                for k in range(kc):
                                    for r in range(min(32, n - row0)):
                                        for l in range(dls):
                                            written[(row0 + r, i * b * d + (kq + k) * d + l0 + l)] += 1
                            else:
                                for lane in range(32):
                                    u = lane & 7
                                    if u >= units:
                                        continue
                                    col = ybase + (kq + rpu * u // dls) * d + (rpu * u) % dls
                                    for r in range(lane >> 3, min(32, n - row0), 4):
                                        for e in range(rpu):
                                            written[(row0 + r, col + e)] += 1
    assert all(0 <= r < n and 0 <= col < out_f for r, col in written)
    assert len(written) == n * out_f and set(written.values()) == {1}


@pytest.mark.parametrize("dls,es", [(1, 2), (2, 2), (4, 2), (8, 2), (16, 2), (1, 4), (2, 4), (4, 4), (8, 4)])
def test_tc_shared_memory_offsets_keep_their_alignment(dls, es):
    """Every X ring slot is a TMA destination (128-byte aligned at least, 1 KiB
    for the 128-byte swizzle of d = 1), and the values ring that follows the X
    ring holds swizzle atoms of 8 rows x the row width, which must sit at
    multiples of their size: slot sizes and values planes keep 1 KiB / atom
    alignment for every ring depth and pass width."""
    ctj = chunk_j(dls, es)
    slot = slot_bytes(dls, es)
    assert slot % 1024 == 0
    row = ctj * es  # values row bytes: the swizzle width
    assert row in (32, 64, 128)
    atom = 8 * row
    for bp in range(16, min(256, 512 // dls) + 1, 16):
        plane = bp * ctj * es
        vstage = plane * dls
        for stages in range(2, 9):
            off_v = stages * slot
            for vs in range(4):
                for l in range(dls):
                    assert (off_v + vs * vstage + l * plane) % atom == 0


@pytest.mark.parametrize("dls,es", [(8, 4), (16, 2), (8, 2)])
def test_tc_4d_store_staging_is_the_box_in_order(dls, es):
    """32-byte l runs (fp32 with DLS = 8, bf16 with DLS = 16) and d > DLS: the epilogue writes unit u of row `lane` at
    ((RPU u) / DLS) * 32 DLS es + lane * DLS es + ((RPU u) % DLS) es, which must
    be exactly the box (DLS l, 32 rows, kc k) in its shared order (l fastest,
    then row, then k), every byte once, within the 4 KB staging; eight lanes of
    one 16-byte store reach at least four bank groups.  (The bf16 form of this
    layout with DLS = 8 is modelled too although it keeps 16-byte stores.)"""
    rpu = 16 // es
    kc = (128 // es) // dls
    units = dls * kc * es // 16
    seen = set()
    for lane in range(32):
        for u in range(units):
            off = ((rpu * u) // dls) * (32 * dls * es) + lane * (dls * es) + ((rpu * u) % dls) * es
            for h in range(rpu):
                f = rpu * u + h
                k, l = f // dls, f % dls
                box = ((k * 32 + lane) * dls + l) * es
                assert off + h * es == box and box not in seen
                seen.add(box)
    assert len(seen) == kc * 32 * dls and max(seen) + es <= 4096
    for u in range(units):
        for q0 in range(0, 32, 8):
            g = [(((rpu * u) // dls) * (32 * dls * es) + lane * (dls * es) + ((rpu * u) % dls) * es) // 16 % 8
                 for lane in range(q0, q0 + 8)]
            assert max(g.count(x) for x in g) <= 2


@pytest.mark.parametrize("es", [2, 4])
def test_tc_fused_bias_units_are_aligned_and_cover_the_chunk(es):
    """The tensor-core epilogue reads a chunk's bias as 16-byte units of RPU
    consecutive (k, l) outputs at bias + ybase + (kq + e0) * d + lu: every unit
    is 16-byte aligned (for a 16-byte-aligned bias) and the units cover the
    chunk's kc x DLS columns exactly once, on sweep and test patterns; the
    tile's copy of them in shared memory puts each at the index the chunks
    read."""
    from kronecker_sparse_matrix_b200 import inputs
    pats = inputs.sweep_patterns()[::5] + [(1, 192, 48, 8), (1, 256, 64, 16), (2, 64, 64, 2), (4, 64, 32, 1),
                                           (2, 48, 24, 2), (1, 32, 40, 4), (1, 16, 56, 8), (3, 32, 16, 4),
                                           (2, 64, 64, 32), (1, 48, 48, 1), (1, 64, 8, 1)]
    rpu = 16 // es
    for (a, b, c, d) in pats:
        if c % (32 // es):
            continue
        dls = tc_dls((a, b, c, d), es)
        bp = tc_bp(dls, b)
        kc = tc_kc(dls, bp, es) if bp else 0
        if not kc:
            continue
        units = dls * kc * es // 16
        for i in range(min(a, 2)):
            for l0 in range(0, d, dls):
                ybase = i * b * d + l0
                for kq in range(0, b, kc):
                    cols = []
                    for u in range(units):
                        e0, lu = (rpu * u) // dls, (rpu * u) % dls
                        off = ybase + (kq + e0) * d + lu
                        assert (off * es) % 16 == 0
                        cols += [off + h for h in range(rpu)]
                        assert all(off + h == ybase + (kq + (rpu * u + h) // dls) * d + (rpu * u + h) % dls
                                   for h in range(rpu))
                    assert sorted(cols) == sorted(ybase + (kq + e) * d + l for e in range(kc) for l in range(dls))
            # the tile's copy into shared memory: thread et < bp * DLS / RPU takes
            # unit et = (k, l) element RPU * et of the tile, which is unit u of
            # chunk oc for et = oc * units + u, and stays inside the bias
            nu = bp * dls // rpu
            assert nu <= 128 and nu * 16 <= 2048
            for ps in range(b // bp):
                ybase = i * b * d
                for l0 in range(0, d, dls):
                    for et in range(nu):
                        f = rpu * et
                        off = ybase + l0 + (ps * bp + f // dls) * d + f % dls
                        oc, u = divmod(et, units)
                        e0, lu = (rpu * u) // dls, (rpu * u) % dls
                        assert off == ybase + l0 + (ps * bp + oc * kc + e0) * d + lu
                        assert (off * es) % 16 == 0 and off + rpu <= a * b * d


# ------------------------------------------------------------ ks_butterfly.cu
def bfly_swz(e):
    A, B, C = e >> 8, (e >> 4) & 15, e & 15
    return (A << 8) | (((B ^ A) & 15) << 4) | (C ^ ((B >> 1) | ((A & 1) << 3)))


def test_butterfly_row_order_is_a_bijection_and_every_pass_is_conflict_free():
    assert sorted(bfly_swz(e) for e in range(4096)) == list(range(4096))
    for t in range(256):
        u1, u2, u3 = bfly_swz(t), bfly_swz(((t >> 4) << 8) | (t & 15)), bfly_swz(t << 4)
        for D in range(16):
            # the kernel's per-pass shortcuts equal the order of the entry each thread holds
            assert (D << 8) | (u1 ^ ((D << 4) | ((D & 1) << 3))) == bfly_swz((D << 8) | t)
            assert u2 ^ ((D << 4) | (D >> 1)) == bfly_swz(((t >> 4) << 8) | (D << 4) | (t & 15))
            assert u3 ^ D == bfly_swz((t << 4) | D)
    for w in range(8):
        lanes = range(32 * w, 32 * w + 32)
        for D in range(16):
            for pas in ((lambda t: (D << 8) | t), (lambda t: ((t >> 4) << 8) | (D << 4) | (t & 15)),
                        (lambda t: (t << 4) | D)):
                assert wavefronts([bfly_swz(pas(t)) for t in lanes], 1) == 1


def test_butterfly_resident_pass3_weights_cover_each_pair_and_are_conflict_free():
    slot_words = 4                         # one float4 (a pair's 2 x 2 weights in fp32)
    rot = lambda line: line & 7
    rows = 6
    assert rows * 4096 * 4 + 4 * 2048 * 4 * slot_words <= 232448
    for f in range(4):
        where = {}
        for i in range(8):
            for w in range(8):
                addrs = []
                for t in range(32 * w, 32 * w + 32):
                    g = t + 256 * i
                    idx = f * 2048 + (g >> 3) * 8 + ((g & 7) ^ rot(g >> 3))
                    assert idx not in where.values()
                    where[g] = idx
                    addrs.append(idx * slot_words)
                assert wavefronts(addrs, slot_words) == slot_words   # 512 or 256 bytes: optimal
        assert sorted(where) == list(range(2048))
        # pass 3: thread t's k-th pair (q = 8t + k) is read at slot k ^ rot(t) of line t
        for k in range(8):
            for w in range(8):
                addrs = []
                for t in range(32 * w, 32 * w + 32):
                    idx = f * 2048 + t * 8 + (k ^ rot(t))
                    assert where[8 * t + k] == idx
                    addrs.append(idx * slot_words)
                assert wavefronts(addrs, slot_words) == slot_words
