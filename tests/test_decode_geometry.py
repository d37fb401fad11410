"""CPU: the decode kernel's work split and memory geometry, mirrored on the host.

The decode kernel (csrc/decode.cu) cuts a call into segments (one 128-row tile of one
block x one chunk group, chunk-group-major), gives each CTA a contiguous run, builds
the activation sets of its chunk groups in two shared-memory slots, streams each
segment's sign tiles into shared-memory stages, hands units to teams of four warps and
to the issuer warps in turn, and reduces each row tile in the CTA that adds its last
partial.  This test restates that arithmetic and checks, for the shapes the tests and
the bench use, that
  * every unit (row tile, block, chunk) is covered exactly once, by exactly one team
    and one issuer;
  * every bulk copy (sign stage) and every V / U row read lies inside its source area;
  * a CTA touches consecutive chunk groups only;
  * the activation-set bytes the builders write land exactly where the MMA descriptors
    read them, and tile each chunk exactly;
  * shared memory, tensor-memory columns and threads fit, and two decode CTAs never
    share an SM;
  * the per-segment barrier arrivals add up to the counts the barriers are set to;
  * the reduction reads stay inside the workspace that bs_workspace_bytes reports.
A change to the kernels' split or layout that breaks one of these fails here, on the
CPU, before anything runs on a GPU."""
import numpy as np
import pytest

import residual_block_decomp_b200 as R

SM_SMEM = 228 * 1024
RESERVED = 1024
BLOCK_LIMIT = 227 * 1024
SMS = 148


class Cfg:
    def __init__(self, b):
        self.B = b
        self.NB = 32 * b
        self.NCOL = 16 * b
        self.C = 4 if b == 1 else 2
        self.ZB = self.NB * 256
        self.SET = self.C * self.ZB
        self.T = 3 if b <= 2 else 2
        self.NI = 3 if b <= 2 else 2
        self.NACC = 4 if b == 1 else 2
        self.ACOL0 = self.NACC * self.NB
        self.THREADS = 32 * (4 * self.T + self.NI + 5)
        self.ZTHREADS = self.THREADS - 32
        self.STAGE = self.C * 4096
        stg = b * self.C * 256 * 2 + self.C * 256 * 4          # first group's x rows and 1/s
        self.STG_AL = -(-stg // 1024) * 1024
        fixed = 2 * self.SET + 8192 + self.STG_AL
        self.NS = min(16, (BLOCK_LIMIT - fixed) // self.STAGE)
        self.SMEM = self.NS * self.STAGE + fixed


def cta_range(cta, grid, n, NCB, RT):
    """Mirror of the kernel's cta_range: group-aligned runs when the chunk groups are no
    more than the CTAs, contiguous runs otherwise."""
    NG, segs = n * NCB, RT * n * NCB
    if NG <= grid:
        base, extra = divmod(grid, NG)
        if cta < extra * (base + 1):
            g, w = divmod(cta, base + 1)
            k = base + 1
        else:
            c2 = cta - extra * (base + 1)
            g = extra + c2 // base
            w = c2 - (g - extra) * base
            k = base
        return g * RT + (w * RT) // k, g * RT + ((w + 1) * RT) // k
    return cta * segs // grid, (cta + 1) * segs // grid


def geometry(m, d, n, b):
    K = Cfg(b)
    RT, KG = m // 128, d // 256
    NCB = -(-KG // K.C)
    segs = RT * n * NCB
    grid = min(SMS - 4, segs)
    return K, RT, KG, NCB, segs, grid


SHAPES = [(128, 256, 1), (256, 512, 3), (384, 768, 2), (640, 1280, 4), (1024, 4096, 5), (512, 2560, 7),
          (4096, 4096, 8), (14336, 4096, 12), (4096, 14336, 10), (128, 65536, 64), (65536, 256, 2)]


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_shared_tensor_memory_and_threads_fit(b):
    K = Cfg(b)
    assert K.NS >= 4 and K.SMEM <= BLOCK_LIMIT
    # two decode CTAs (each allocating all 512 tensor-memory columns) never share an SM
    assert 2 * (K.SMEM + RESERVED) > SM_SMEM
    assert K.ACOL0 + K.T * 2 * 64 <= 512
    assert K.THREADS <= 1024
    # the epilogue warps start at 4T + NI: with the issuers in between, their indices
    # modulo 4 still cover the four tensor-memory lane quadrants once each
    wepi = 4 * K.T + K.NI
    assert sorted(w % 4 for w in range(wepi, wepi + 4)) == [0, 1, 2, 3]
    # the row-tile reduction's scratch (4 tiles x slices x batch x 128 fp32, then the
    # completed row-tile list) fits the drained sign stages
    assert 4 * (K.THREADS // 128) * b * 128 * 4 + K.THREADS * 4 <= K.NS * K.STAGE
    # the activation sets sit at the start of shared memory: descriptor addresses fit
    # their 14-bit field (16-byte units)
    assert (2 * K.SET) >> 4 < (1 << 14)
    # the first group's V rows (32 bytes per input column) are staged in the second set
    # slot, its x rows and 1/s in the staging area
    assert K.C * 256 * 32 <= K.SET
    assert b * K.C * 256 * 2 + K.C * 256 * 4 <= K.STG_AL


@pytest.mark.parametrize("m,d,n", SHAPES)
@pytest.mark.parametrize("b", [1, 4])
def test_segments_cover_units_once_and_stay_in_bounds(m, d, n, b):
    K, RT, KG, NCB, segs, grid = geometry(m, d, n, b)
    sign_bytes = m * d // 8
    seen = set()
    groups = n * NCB
    for cta in range(grid):
        s0, s1 = cta_range(cta, grid, n, NCB, RT)
        assert s1 > s0
        if groups <= grid:
            assert s0 // RT == (s1 - 1) // RT       # inside one chunk group
        cgs = []
        u = 0
        for s in range(s0, s1):
            cg, rt = divmod(s, RT)
            i, cgi = divmod(cg, NCB)
            kgA = cgi * K.C
            ln = min(K.C, KG - kgA)
            assert 0 <= i < n and 1 <= ln <= K.C
            # sign stage: ln contiguous 4 KiB tiles of row tile rt, inside block i's signs
            assert (rt * KG + kgA) * 4096 + ln * 4096 <= sign_bytes and ln * 4096 <= K.STAGE
            # the group's V rows and the row tile's U rows inside the factor areas
            assert (kgA * 256 + ln * 256) * 32 <= d * 32
            assert (rt * 128 + 127) * 32 + 32 <= m * 32
            for kg in range(kgA, kgA + ln):
                key = (rt, i, kg)
                assert key not in seen
                seen.add((rt, i, kg))
                # unit u: team u mod T, slot (u // T) mod 2, issuer u mod NI
                assert 0 <= u % K.T < K.T and 0 <= u % K.NI < K.NI
                u += 1
            cgs.append(cg)
        assert sorted(set(cgs)) == list(range(cgs[0], cgs[-1] + 1))
    assert len(seen) == RT * n * KG


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_set_bytes_land_where_the_mma_reads(b):
    """The set builders write the byte of operand column n (hi plane n = 16 b + j, lo
    plane NCOL + n) and group column c at chunk c >> 8, K-step t = (c & 255) >> 5,
    K-half kc = (c >> 4) & 1, byte c & 15 of the 16-byte row of core matrix (n >> 3,
    kc), row n & 7.  The decode kernel's descriptor for K-step t (no swizzle, K-major,
    LBO 128 = next core matrix in K, SBO 256 = next core matrix in N) reads that core
    matrix row at t*(NB/8)*256 + (n>>3)*256 + kc*128 + (n&7)*16.  Both must agree, and
    the writes must tile every chunk exactly once."""
    K = Cfg(b)
    hits = np.zeros(K.SET, dtype=np.int32)
    for c in range(K.C * 256):
        cc, cl = c >> 8, c & 255
        t, kc, byte = cl >> 5, (cl >> 4) & 1, cl & 15
        for n in range(K.NB):
            written = cc * K.ZB + (t * (K.NB // 8) * 2 + kc) * 128 + byte + (n >> 3) * 256 + (n & 7) * 16
            read = cc * K.ZB + t * (K.NB // 8) * 256 + (n >> 3) * 256 + kc * 128 + (n & 7) * 16 + byte
            assert written == read
            hits[written] += 1
    assert hits.min() == 1 and hits.max() == 1


@pytest.mark.parametrize("m,d,n", SHAPES)
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_barrier_arrivals_match_counts(m, d, n, b):
    """Per segment the issuer of each unit commits once into the segment's accumulator
    barrier, and the issuer of a short segment's last unit adds C - len plain
    arrivals; each of the four warps of a unit's team arrives once on the sign stage,
    and adds C - len after the segment's last unit.  Every phase therefore receives the
    count its barrier is set to (C and 4 C), short segments included."""
    K, RT, KG, NCB, segs, grid = geometry(m, d, n, b)
    for cgi in range(NCB):
        ln = min(K.C, KG - cgi * K.C)
        assert ln + (K.C - ln) == K.C
        assert 4 * ln + 4 * (K.C - ln) == 4 * K.C


@pytest.mark.parametrize("m,d,n", SHAPES)
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_workspace_layout_and_reduction_reads(m, d, n, b):
    K, RT, KG, NCB, segs, grid = geometry(m, d, n, b)
    NC = n * NCB
    cnt_bytes = -(-RT * 4 // 256) * 256
    part_floats = segs * b * 128
    ws = R.bs_workspace_bytes(m, d, 16, n, b)
    assert ws == cnt_bytes + -(-part_floats * 4 // 256) * 256
    # the last partial the reducer of the last row tile reads
    last = (RT - 1) * b * 128 + 127 + (NC - 1) * RT * b * 128 + (b - 1) * 128
    assert last < part_floats


def test_expansion_rule_reads_columns_in_order():
    """The decode expanders read, for row r of a tile, 16 bytes at r*16 and 16 at
    2048 + r*16 (eight 32-bit words w[0..7]), and K-step t takes byte q of
    (w[pw] >> t) & 0x01010101 as A[r, 32 t + 4 pw + q].  Applied to the library's own
    host packer, that rule must give the signs in natural column order."""
    gen = np.random.default_rng(11)
    m, d = 256, 512
    neg = gen.random((m, d)) < 0.5
    bits = np.packbits(neg, axis=1, bitorder="little")                  # canonical order
    U = np.zeros((m, 16), np.float16)
    V = np.zeros((d, 16), np.float16)
    rec = R.bs_pack_record(m, d, 16, bits, U, V)
    KG = d // 256
    for rt in range(m // 128):
        for kg in range(KG):
            tile = rec[(rt * KG + kg) * 4096:(rt * KG + kg + 1) * 4096]
            for r in range(128):
                w = np.concatenate([tile[r * 16:r * 16 + 16], tile[2048 + r * 16:2048 + r * 16 + 16]]).view("<u4")
                for t in range(8):
                    a = ((w >> t) & 0x01010101).astype("<u4").view(np.uint8)   # bytes (pw, q)
                    cols = kg * 256 + 32 * t + np.arange(32)
                    assert np.array_equal(a.astype(bool), neg[rt * 128 + r, cols])


# ------------------------------------------------------------ grouped launches -----
class Lin:
    def __init__(self, m, d, n, b, seg0, cg0):
        K = Cfg(b)
        self.m, self.d, self.n = m, d, n
        self.RT, self.KG = m // 128, d // 256
        self.NCB = -(-self.KG // K.C)
        self.seg0, self.cg0 = seg0, cg0
        self.segs = self.RT * n * self.NCB


def group_table(shapes, b):
    """The host's table: linears with blocks, segments and chunk groups numbered one
    linear after another (bs_linear_group)."""
    tab, seg, cg = [], 0, 0
    for (m, d, n) in shapes:
        if n == 0:
            continue
        L = Lin(m, d, n, b, seg, cg)
        tab.append(L)
        seg += L.segs
        cg += n * L.NCB
    return tab, seg


def seg_of(tab, s, C):
    """Mirror of the kernel's seg_of: the last linear whose first segment is <= s."""
    lo, hi = 0, len(tab) - 1
    while lo < hi:
        mid = (lo + hi + 1) >> 1
        if tab[mid].seg0 <= s:
            lo = mid
        else:
            hi = mid - 1
    L = tab[lo]
    sl = s - L.seg0
    cg, rt = divmod(sl, L.RT)
    i, cgb = divmod(cg, L.NCB)
    return dict(l=lo, sl=sl, cg=cg, rt=rt, i=i, cgb=cgb, kgA=cgb * C, len=min(C, L.KG - cgb * C))


def seg_next(tab, g, C):
    """Mirror of the kernel's seg_next (no divisions, linears one after another)."""
    g = dict(g)
    g["sl"] += 1
    L = tab[min(g["l"], len(tab) - 1)]
    g["rt"] += 1
    if g["rt"] == L.RT:
        g["rt"] = 0
        g["cg"] += 1
        g["cgb"] += 1
        if g["cgb"] == L.NCB:
            g["cgb"] = 0
            g["i"] += 1
            if g["i"] == L.n:
                g["l"] += 1
                g["i"] = g["cg"] = g["sl"] = 0
        g["kgA"] = g["cgb"] * C
        g["len"] = min(C, tab[min(g["l"], len(tab) - 1)].KG - g["kgA"])
    return g


def group_next(tab, l, cg):
    L = tab[min(l, len(tab) - 1)]
    cg += 1
    if cg == L.n * L.NCB:
        return l + 1, 0
    return l, cg


def _model(counts, layers=2):
    from workloads import LLAMA3_8B_LINEARS
    shapes = [(m, d) for _ in range(layers) for (_, m, d) in LLAMA3_8B_LINEARS]
    return [(m, d, counts[j % len(counts)]) for j, (m, d) in enumerate(shapes)]


GROUPS = [_model([3, 0, 1, 5, 2, 16, 4]), _model([1]), _model([16, 2, 0, 0, 9, 1, 3], layers=4),
          [(128, 256, 1), (256, 512, 2), (128, 256, 0), (1024, 4096, 3)]]


@pytest.mark.parametrize("gi", range(len(GROUPS)))
@pytest.mark.parametrize("b", [1, 3])
def test_grouped_walk_covers_every_linear_once_and_stays_in_bounds(gi, b):
    """A grouped launch: every unit of every linear with blocks is covered exactly once;
    the walk (seg_next) agrees with a fresh lookup (seg_of) at every step; each sign
    copy, V and U read and partial write lies inside its own linear's areas; a CTA's
    chunk groups are consecutive in the launch's numbering, and the background set
    builds (group_next) name exactly the groups the walk reaches."""
    K = Cfg(b)
    shapes = GROUPS[gi]
    tab, segs = group_table(shapes, b)
    grid = min(SMS - 4, segs)
    seen = set()
    for cta in range(grid):
        s0, s1 = cta * segs // grid, (cta + 1) * segs // grid
        assert s1 > s0
        g = seg_of(tab, s0, K.C)
        gids = []
        for s in range(s0, s1):
            f = seg_of(tab, s, K.C)
            assert g == f, (cta, s, g, f)
            L = tab[g["l"]]
            assert 0 <= g["i"] < L.n and 1 <= g["len"] <= K.C and g["sl"] == s - L.seg0
            assert (g["rt"] * L.KG + g["kgA"]) * 4096 + g["len"] * 4096 <= L.m * L.d // 8
            assert (g["kgA"] * 256 + g["len"] * 256) * 32 <= L.d * 32
            assert (g["rt"] * 128 + 128) * 32 <= L.m * 32
            assert (g["sl"] + 1) * b * 128 <= L.segs * b * 128
            for kg in range(g["kgA"], g["kgA"] + g["len"]):
                key = (g["l"], g["rt"], g["i"], kg)
                assert key not in seen
                seen.add(key)
            gids.append(L.cg0 + g["cg"])
            g = seg_next(tab, g, K.C)
        assert sorted(set(gids)) == list(range(gids[0], gids[-1] + 1))
        # the groups after the first, as the epilogue names them
        first = seg_of(tab, s0, K.C)
        l, cg = first["l"], first["cg"]
        for gid in sorted(set(gids))[1:]:
            l, cg = group_next(tab, l, cg)
            assert tab[l].cg0 + cg == gid
    assert len(seen) == sum(L.RT * L.n * L.KG for L in tab)


def group_ws_bytes(shapes, b):
    """Mirror of bs_group_workspace_bytes: all row-tile counters first (their places
    depend on the shapes only), then each linear's partials, 256-byte aligned."""
    C = 4 if b == 1 else 2
    off = -(-sum(m // 128 for (m, d, n) in shapes) * 4 // 256) * 256
    for (m, d, n) in shapes:
        segs = (m // 128) * n * -(-(d // 256) // C)
        off = -(-(off + segs * b * 128 * 4) // 256) * 256
    return off


@pytest.mark.parametrize("m,d,n", SHAPES)
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_bulk_copies_are_16_byte_units(m, d, n, b):
    """Every 1-D bulk copy the decode kernel issues starts on a 16-byte boundary and
    moves a multiple of 16 bytes (the rule of cp.async.bulk): sign stages, the first
    group's V rows, 1/s and x rows, from a 256-byte aligned stack, 16-byte aligned 1/s
    and x, into shared-memory regions at 1024-byte offsets."""
    K, RT, KG, NCB, segs, grid = geometry(m, d, n, b)
    block = m * d // 8 + 32 * (m + d)
    assert block % 16 == 0 and (m * d // 8) % 16 == 0 and (m * d // 8 + 32 * m) % 16 == 0
    for cg in range(n * NCB):
        i, cgb = divmod(cg, NCB)
        kgA = cgb * K.C
        ln = min(K.C, KG - kgA)
        gcols = ln * 256
        col0 = kgA * 256
        for rt in range(RT):
            src = i * block + (rt * KG + kgA) * 4096
            assert src % 16 == 0 and (ln * 4096) % 16 == 0
        v_src = i * block + m * d // 8 + 32 * m + col0 * 32
        assert v_src % 16 == 0 and (gcols * 32) % 16 == 0
        assert (col0 * 4) % 16 == 0 and (gcols * 4) % 16 == 0            # 1/s
        for lane in range(b):
            assert (lane * d * 2 + col0 * 2) % 16 == 0 and (gcols * 2) % 16 == 0   # x row
    # shared-memory destinations: sets, stages, control block, staging
    assert (2 * K.SET) % 1024 == 0 and K.STAGE % 1024 == 0 and (2 * K.SET + K.NS * K.STAGE + 8192) % 1024 == 0


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_every_a_slot_has_one_issuer(b):
    """Unit u goes to team u % T, A slot (u // T) % 2 of that team, and issuer u % NI.
    The issuer waits on the slot's ready barrier by phase parity, so it must see every
    use of the slot in turn: all uses of one slot go to one issuer."""
    K = Cfg(b)
    owner = {}
    for u in range(10000):
        slot = (u % K.T, (u // K.T) % 2)
        assert owner.setdefault(slot, u % K.NI) == u % K.NI, (b, slot)
    assert len(owner) == 2 * K.T and len(set(owner.values())) == K.NI
