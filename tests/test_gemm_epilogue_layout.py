"""Host replay of the fused GEMM's staged epilogue (csrc/nf4_gemm.cu, unsplit tiles).

For each 128-row accumulator, warp w of the 16 dequantizing warps stages TMEM lanes
32 (w mod 4).. and columns 64 (w / 4).. in shared memory, 16-byte chunk j of row r at
r * row_bytes + 16 (j ^ (r mod 8)); then warp w writes rows w, w + 16, .. of y, lane l taking
chunks l, l + 32, ..  This replays that index arithmetic on the CPU and checks that every
element of a tile inside M x N is written exactly once, from its own accumulator entry, for
f32 and 16-bit outputs and ragged edges; that staging stays inside the 128 KB it may use; and
that the eight lanes of each 16-byte shared-memory access phase hit eight different bank
groups on both sides.  The split-K sum's row slices and chunks are replayed the same way.
"""
import pytest

BN, DEQ_WARPS = 256, 16


def replay(M, N, m0, n0, f32_out):
    esz = 4 if f32_out else 2
    row_bytes, per = BN * esz, 16 // esz
    chunks = row_bytes // 16
    halves = 2 if m0 + 128 < M else 1
    written = {}
    for hh in range(halves):
        stage = {}
        for warp in range(DEQ_WARPS):
            q, cq = warp & 3, warp >> 2
            for c in range(2):
                cbase = 64 * cq + 32 * c
                for i in range(32 // per):
                    j = cbase // per + i
                    groups = []
                    for lane in range(32):
                        rr = 32 * q + lane
                        off = rr * row_bytes + ((j ^ (rr & 7)) << 4)
                        assert off % 16 == 0 and off + 16 <= 128 * 1024
                        assert off not in stage
                        stage[off] = [(128 * hh + rr, cbase + per * i + e) for e in range(per)]
                        groups.append((off // 16) % 8)
                    for ph in range(4):  # a 16-byte warp access runs in 4 phases of 8 lanes
                        assert len(set(groups[8 * ph:8 * ph + 8])) == 8
        for warp in range(DEQ_WARPS):
            for k in range(128 // DEQ_WARPS):
                r2 = warp + DEQ_WARPS * k
                m = m0 + 128 * hh + r2
                if m >= M:
                    break
                for base in range(0, chunks, 32):
                    groups = []
                    for lane in range(32):
                        j = base + lane
                        off = r2 * row_bytes + ((j ^ (r2 & 7)) << 4)
                        groups.append((off // 16) % 8)
                        col = n0 + j * per
                        for e in range(per):
                            if col + e < N:
                                key = (m, col + e)
                                assert key not in written
                                trow, tcol = stage[off][e]
                                assert (m0 + trow, n0 + tcol) == key
                                written[key] = True
                    for ph in range(4):
                        assert len(set(groups[8 * ph:8 * ph + 8])) == 8
    want = {(m, c) for m in range(m0, min(M, m0 + 256)) for c in range(n0, min(N, n0 + 256))}
    assert set(written) == want


@pytest.mark.parametrize("f32_out", [True, False])
@pytest.mark.parametrize("M,N,m0,n0", [(4096, 11008, 256, 10752), (300, 1001, 256, 768),
                                       (600, 300, 512, 256), (129, 257, 0, 256), (1, 1, 0, 0),
                                       (256, 256, 0, 0), (130, 129, 0, 0)])
def test_staged_epilogue_writes_each_element_once(M, N, m0, n0, f32_out):
    replay(M, N, m0, n0, f32_out)


def replay_split(M, N, m0, n0, S):
    """Split K: after the first cluster barrier, CTA z of the S CTAs of a tile adds rows
    [rows z / S, rows (z + 1) / S) of each staged 128-row accumulator (binary32, 1024-byte
    rows, chunk j of row r at 16 (j ^ (r mod 8))); thread e of 576 takes (row lo + e / nch,
    chunk e mod nch), 4 columns a chunk."""
    threads = 576
    cols = min(BN, N - n0)
    nch = (cols + 3) // 4
    written = {}
    for hh in range(2 if m0 + 128 < M else 1):
        rows = min(128, M - (m0 + 128 * hh))
        for z in range(S):
            lo, hi = rows * z // S, rows * (z + 1) // S
            for t in range(threads):
                for e in range(t, (hi - lo) * nch, threads):
                    r, j = lo + e // nch, e % nch
                    off = r * BN * 4 + ((j ^ (r & 7)) << 4)
                    assert off + 16 <= 128 * 1024
                    for k in range(4):
                        if 4 * j + k < cols:
                            key = (m0 + 128 * hh + r, n0 + 4 * j + k)
                            assert key not in written
                            written[key] = z
    want = {(m, c) for m in range(m0, min(M, m0 + 256)) for c in range(n0, min(N, n0 + 256))}
    assert set(written) == want


@pytest.mark.parametrize("S", [2, 3, 4, 7, 8])
@pytest.mark.parametrize("M,N,m0,n0", [(128, 11008, 0, 10752), (7, 1023, 0, 768),
                                       (300, 512, 256, 256), (200, 10240, 0, 0)])
def test_split_k_sum_covers_each_output_once(M, N, m0, n0, S):
    replay_split(M, N, m0, n0, S)
