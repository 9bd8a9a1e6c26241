"""Index arithmetic of the pair GEMM's staged epilogue stores and of the register-held row
quantiser's launch, checked on the host (CPU only): the formulas below are the kernels' own."""
import itertools

import pytest


def stage_write(lane, q):          # 16-byte slot a lane writes piece q of its row to
    return lane * 4 + (q ^ ((lane >> 1) & 3))


def stage_read(lane, j):           # (row, piece, slot) a lane reads for store instruction j
    r, q = 8 * j + (lane >> 2), lane & 3
    return r, q, r * 4 + (q ^ ((r >> 1) & 3))


def test_staging_is_a_permutation_and_reads_what_was_written():
    written = {stage_write(l, q): (l, q) for l in range(32) for q in range(4)}
    assert sorted(written) == list(range(128))          # 2 KB, every slot once
    seen = set()
    for j, l in itertools.product(range(4), range(32)):
        r, q, slot = stage_read(l, j)
        assert written[slot] == (r, q)                  # row r's piece q, as lane r wrote it
        seen.add((r, q))
    assert len(seen) == 128                             # every row piece stored exactly once


def test_staging_has_no_bank_conflicts():
    # a warp's 16-byte shared accesses go 8 lanes at a time; 8 slots of 16 bytes span the 32 banks
    for q in range(4):
        for phase in range(4):
            groups = {stage_write(l, q) % 8 for l in range(8 * phase, 8 * phase + 8)}
            assert len(groups) == 8
    for j in range(4):
        for phase in range(4):
            groups = {stage_read(l, j)[2] % 8 for l in range(8 * phase, 8 * phase + 8)}
            assert len(groups) == 8


def test_store_instruction_writes_whole_sectors():
    # store j: lanes 4m..4m+3 write the four 16-byte pieces of one row's 64 bytes
    for j in range(4):
        rows = {}
        for l in range(32):
            r, q, _ = stage_read(l, j)
            rows.setdefault(r, set()).add(q)
        assert len(rows) == 8 and all(v == {0, 1, 2, 3} for v in rows.values())


def quant_variant(K):
    """(threads per row, 16-byte chunks per thread) the layer picks for rows of K elements,
    or None for the two-pass fallback."""
    chunks = K // 8
    for tpr, c in ((32, 2), (32, 4), (32, 8), (128, 4), (128, 8), (256, 8)):
        if chunks <= tpr * c:
            return tpr, c
    return None


@pytest.mark.parametrize("K", [128, 256, 512, 768, 1024, 1536, 2048, 3072, 4096, 6144, 7168, 9216, 14336, 16384])
@pytest.mark.parametrize("rows", [1, 7, 8, 9, 255, 131072])
def test_register_quantiser_covers_every_row_and_chunk_in_bounds(K, rows):
    v = quant_variant(K)
    assert v is not None
    tpr, maxc = v
    chunks = K // 8
    rpc = 256 // tpr
    grid = (rows * tpr + 255) // 256
    assert grid * rpc >= rows                           # every row has a row group
    # within a row, threads tid < tpr take chunks tid + i tpr, i < maxc: each chunk once, none past
    covered = sorted(t + i * tpr for t in range(tpr) for i in range(maxc) if t + i * tpr < chunks)
    assert covered == list(range(chunks))
    assert (grid - 1) * rpc + (rpc - 1) < rows + rpc     # rows past the end are masked, not read
