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


# ------------------------------------------------------------------ ks_tc.cu
def chunk_j(dls):
    return 16 if dls == 8 else 64 // dls


def tc_task_unit(dls, task, units):
    if dls == 8:
        return task % units, task // units
    q = task & 7
    return q, ((task >> 3) + (q >> (1 if dls == 2 else 2))) & 15


@pytest.mark.parametrize("dls", [2, 4, 8])
def test_tc_transposer_quarter_warps_reach_eight_bank_groups(dls):
    ctj = chunk_j(dls)
    units = ctj * dls // 8
    tasks = 16 * units // 128
    group_stride, octet_stride = 144, 16 * 144
    slot = dls * (ctj // 8) * octet_stride
    written, mapped = set(), set()
    for k in range(tasks):
        for t0 in range(0, 128, 8):  # one quarter-warp: 8 consecutive lanes
            qg = [tc_task_unit(dls, t + 128 * k, units) for t in range(t0, t0 + 8)]
            for r in range(8):  # reads of the raw chunk
                groups = {((g8 * 8 + r) * units + q) % 8 for q, g8 in qg}
                assert len(groups) == 8
            for e in range(8):  # writes of the padded planes
                addrs = []
                for q, g8 in qg:
                    f = 8 * q + e
                    j, l = f // dls, f % dls
                    a = (l * (ctj // 8) + (j >> 3)) * octet_stride + g8 * group_stride + (j & 7) * 16
                    assert 0 <= a and a + 16 <= slot and a not in written
                    written.add(a)
                    addrs.append(a)
                assert len({(a // 16) % 8 for a in addrs}) == 8
            mapped.update(qg)
    assert len(mapped) == tasks * 128 and all(0 <= q < units and 0 <= g < 16 for q, g in mapped)


def tc_bp(dls, b):
    for bp in range(min(256, 512 // dls), 15, -16):
        if b % bp == 0:
            return bp
    return 0


def tc_kc(dls, bp):
    for kc in range(min(bp, 64 // dls), 7, -8):
        if bp % kc == 0 and dls * kc == 64:
            return kc
    for kc in range(min(bp, 64 // dls), 7, -8):
        if bp % kc == 0:
            return kc
    return 0


@pytest.mark.parametrize("p", [(2, 48, 48, 2), (1, 48, 48, 4), (2, 64, 64, 16), (1, 192, 48, 8), (3, 32, 16, 4),
                               (1, 256, 256, 2), (2, 48, 48, 1), (1, 16, 16, 1), (1, 96, 96, 4), (1, 80, 16, 2)])
def test_tc_epilogue_writes_each_output_once(p):
    """The output boxes of a tile: 32 rows x (DLS * kc) elements per warp and
    chunk, either one tensor store of a contiguous box (d == DLS) or 16-byte
    stores of its units; N = 300 leaves a ragged last row block."""
    a, b, c, d = p
    dls = 8 if d % 8 == 0 else d
    bp = tc_bp(dls, b)
    kc = tc_kc(dls, bp)
    n, out_f = 300, a * b * d
    units = dls * kc // 8
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
                                assert (x * 2) % 16 == 0
                                for r in range(min(32, n - row0)):
                                    for e in range(dls * kc):
                                        written[(row0 + r, x + e)] += 1
                            else:
                                for lane in range(32):
                                    u = lane & 7
                                    if u >= units:
                                        continue
                                    col = ybase + (kq + 8 * u // dls) * d + (8 * u) % dls
                                    for r in range(lane >> 3, min(32, n - row0), 4):
                                        for e in range(8):
                                            written[(row0 + r, col + e)] += 1
    assert all(0 <= r < n and 0 <= col < out_f for r, col in written)
    assert len(written) == n * out_f and set(written.values()) == {1}
