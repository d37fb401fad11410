"""CPU: the decode kernel's work split and memory geometry, mirrored on the host.

The decode kernel (csrc/decode.cu) cuts a call into segments (one 128-row tile of one
block x C chunks of 256 columns, chunk-group-major) and gives each CTA a contiguous run.
This test restates that arithmetic and checks, for the shapes the tests and the bench
use, that
  * every unit (row tile, block, chunk) is covered exactly once;
  * every bulk copy (sign stage, V rows, U tile) lies inside its block's area;
  * a CTA touches consecutive chunk groups only;
  * the per-CTA shared memory fits 227 KB and the tensor-memory columns fit 512;
  * the reduction reads stay inside the workspace that bs_workspace_bytes reports.
A change to the kernel's split or layout that breaks one of these fails here, on the
CPU, before anything runs on a GPU."""
import pytest

import residual_block_decomp_b200 as R

SMEM_LIMIT = 227 * 1024
SMS = 148


def chunks_per_segment(b):
    return 4 if b == 1 else 2


def shared_memory(b):
    """Bytes of dynamic shared memory per CTA: sign stages + two chunk-group sets +
    V rows + x rows and 1/s + x (.) 1/s + U ring + control block."""
    nb, C = 32 * b, chunks_per_segment(b)
    cols = C * 256
    fixed = 2 * (512 + C * nb * 256) + cols * 32 + (cols * b * 2 + cols * 4) + cols * b * 4 + 4 * 4096 + 1024
    stage = C * 4096
    ns = min(16, (SMEM_LIMIT - fixed) // stage)
    return ns, ns * stage + fixed


def tmem_columns(b):
    nb = 32 * b
    pairs = (512 - 2 * nb) // 128
    return pairs, 2 * nb + 128 * pairs


def geometry(m, d, n, b):
    C = chunks_per_segment(b)
    RT, KG = m // 128, d // 256
    NCB = -(-KG // C)
    segs = RT * n * NCB
    grid = min(SMS, segs)
    return C, RT, KG, NCB, segs, grid


SHAPES = [(128, 256, 1), (256, 512, 3), (384, 768, 2), (640, 1280, 4), (1024, 4096, 5), (512, 2560, 7),
          (4096, 4096, 8), (14336, 4096, 12), (4096, 14336, 10), (128, 65536, 64), (65536, 256, 2)]


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_shared_and_tensor_memory_fit(b):
    ns, smem = shared_memory(b)
    assert ns >= 2 and smem <= SMEM_LIMIT
    pairs, cols = tmem_columns(b)
    assert 2 <= pairs <= 3 and cols <= 512


@pytest.mark.parametrize("m,d,n", SHAPES)
@pytest.mark.parametrize("b", [1, 4])
def test_segments_cover_units_once_and_stay_in_bounds(m, d, n, b):
    C, RT, KG, NCB, segs, grid = geometry(m, d, n, b)
    sign_bytes = m * d // 8
    seen = set()
    for cta in range(grid):
        s0, s1 = cta * segs // grid, (cta + 1) * segs // grid
        assert s1 > s0
        cgs = []
        for s in range(s0, s1):
            cg, rt = divmod(s, RT)
            i, cgi = divmod(cg, NCB)
            kgA = cgi * C
            ln = min(C, KG - kgA)
            assert 0 <= i < n and 1 <= ln <= C
            # sign stage: ln contiguous 4 KiB tiles of row tile rt, inside block i's signs
            assert (rt * KG + kgA) * 4096 + ln * 4096 <= sign_bytes
            # V rows of the group and the row tile's U rows, inside the factor areas
            assert (kgA * 256 + ln * 256) * 32 <= d * 32 and rt * 128 * 32 + 4096 <= m * 32
            for kg in range(kgA, kgA + ln):
                key = (rt, i, kg)
                assert key not in seen
                seen.add(key)
            cgs.append(cg)
        assert sorted(set(cgs)) == list(range(cgs[0], cgs[-1] + 1))
    assert len(seen) == RT * n * KG


@pytest.mark.parametrize("m,d,n", SHAPES)
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_reduction_reads_inside_workspace(m, d, n, b):
    C, RT, KG, NCB, segs, grid = geometry(m, d, n, b)
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
    import numpy as np
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
