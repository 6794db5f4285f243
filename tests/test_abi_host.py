"""The C-ABI library on the host: it loads, exports every symbol include/*.h
declares, sizes workspaces, and rejects invalid arguments before touching the GPU.
No compute call is made here (CPU only)."""

import ctypes
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "long_context_block_b200", "libmisa_b200.so")


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    from long_context_block_b200 import _binding
    return _binding


def test_exports_every_declared_symbol(lib):
    names = lib.declared_symbols()
    assert {"misa_pool_keys", "misa_route_heads", "misa_score_topk", "dsa_score_topk",
            "misa_dagger_rerank", "misa_score_topk_noalloc", "misa_testing_score_simt",
            "misa_testing_score_rows_wait_expiry"} <= set(names)
    cdll = ctypes.CDLL(LIB)
    for n in names:
        assert hasattr(cdll, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(names) <= exported


def test_workspace_sizes(lib):
    ws = lib.misa_workspace_size
    # route, one query per sequence: the 256-byte header only (the cluster router sums its
    # partial energies in distributed shared memory)
    assert ws(1, 32, 1, 64, 128, 32768, 64, 8, 2048, 8192) == 256
    # score + top-k: header + rows * L fp32 scores + tensor-core scratch (gathered q rows
    # padded to 16 heads, their weights, per-row tile offsets), each 256-aligned
    a256 = lambda x: (x + 255) // 256 * 256
    tc = lambda rows, n: a256(rows * n * 256) + a256(rows * n * 4) + a256((rows + 1) * 4)
    # rows of 8192+ scores (at most 1024 rows) add the histogram top-k scratch: per row a
    # 4096-bin score histogram, 16 group counts and ceil(k / 1024) group buffers of 8192 pairs
    hp = lambda rows, k: (a256(rows * 4096 * 4) + a256(rows * 16 * 4)
                          + a256(rows * (-(-k // 1024)) * 8192 * 8))
    assert ws(2, 32, 1, 64, 128, 32768, 64, 8, 2048, 8192) == 256 + 32 * 32768 * 4 + tc(32, 16) + hp(32, 2048)
    assert ws(3, 32, 1, 64, 128, 32768, 64, 8, 2048, 8192) == 256 + 32 * 32768 * 4 + tc(32, 64) + hp(32, 2048)
    assert ws(2, 16, 1, 64, 128, 131072, 64, 8, 8192, 8192) == \
        256 + 16 * 131072 * 4 + tc(16, 16) + hp(16, 8192)
    # 16 queries of one sequence share key tiles: one unit of 16 queries x 8 slots
    assert ws(2, 1, 16, 64, 128, 2048, 64, 8, 256, 512) == 256 + 16 * 2048 * 4 + tc(1, 128)
    # re-rank: sorted candidate ids, their scores, per-row counts, tensor-core scratch
    # (every row in the decode form with all 64 heads)
    assert ws(4, 16, 1, 64, 128, 131072, 64, 8, 2048, 8192) == \
        256 + 2 * 16 * 8192 * 4 + 256 + tc(16, 64)
    # invalid sizes report 0
    assert ws(1, 0, 1, 64, 128, 1024, 64, 8, 16, 16) == 0
    assert ws(1, 1, 1, 64, 128, 1024, 64, 65, 16, 16) == 0
    assert ws(2, 1, 1, 64, 64, 1024, 64, 8, 16, 16) == 0
    assert ws(4, 1, 1, 64, 128, 1024, 64, 8, 32, 16) == 0
    assert ws(9, 1, 1, 64, 128, 1024, 64, 8, 16, 16) == 0


def test_workspace_sizes_of_query_blocks(lib):
    """A sequence with T >= 2 queries is scored in units of QB queries (QB = the next power of
    two >= T, at most 256 / HS, at least 32 columns), HS = routed heads rounded up to a power
    of two >= 8: the scorer scratch holds units x QB x HS gathered rows."""
    ws = lib.misa_workspace_size
    a256 = lambda x: (x + 255) // 256 * 256
    tc = lambda units, n: a256(units * n * 256) + a256(units * n * 4) + a256((units + 1) * 4)
    L = 4096   # below the histogram path's 8192, so no histogram scratch
    for T, h, units, n in ((2, 8, 1, 32),     # QB = 4 (32 columns at HS = 8)
                           (3, 8, 1, 32),
                           (5, 8, 1, 64),     # QB = 8
                           (16, 8, 1, 128),
                           (40, 8, 2, 256),   # full width: QB = 32
                           (2, 16, 1, 32),    # HS = 16, QB = 2
                           (9, 16, 1, 256)):  # QB = 16
        assert ws(2, 1, T, 64, 128, L, 64, h, 256, 512) == 256 + T * L * 4 + tc(units, n), (T, h)
    # several sequences: units per sequence times nseq
    assert ws(2, 3, 4, 64, 128, L, 64, 8, 256, 512) == 256 + 12 * L * 4 + tc(3, 32)
    # dense DSA (all 64 heads, HS = 64): 4 queries fill a 256-column unit
    assert ws(3, 1, 4, 64, 128, L, 64, 8, 256, 512) == 256 + 4 * L * 4 + tc(1, 256)


def test_invalid_arguments_rejected_on_host(lib):
    c = lib.library()
    null = None
    # null pointers -> INVALID_ARG (1), before any CUDA call
    assert c.misa_pool_keys(null, 1, 1024, 128, 64, null, null) == 1
    # d != 128 -> UNSUPPORTED (2)
    assert c.misa_pool_keys(null, 1, 1024, 64, 64, null, null) == 2
    # B < 1
    assert c.misa_pool_keys(null, 1, 1024, 128, 0, null, null) == 1
    # refresh range outside [0, L] or reversed
    assert c.misa_pool_keys_range(null, 1, 1024, 128, 64, 10, 5, null, null) == 1
    assert c.misa_pool_keys_range(null, 1, 1024, 128, 64, -1, 5, null, null) == 1
    assert c.misa_pool_keys_range(null, 1, 1024, 128, 64, 0, 1025, null, null) == 1
    # h > H
    assert c.misa_route_heads(null, null, null, null, null, 1, 1, 8, 128, 1024, 64, 9, null,
                              null, null, 0, null) == 1
    # h > H routed heads; h = 17 .. H is valid (so the null pointers are what is rejected)
    assert c.misa_score_topk(null, null, null, null, null, 1, 1, 64, 128, 1024, 65, 16, null,
                             null, null, null, 0, null) == 1
    assert c.misa_score_topk(null, null, null, null, null, 1, 1, 64, 128, 1024, 64, 16, null,
                             null, null, null, 0, null) == 1
    assert c.misa_score_rows(null, null, null, null, null, 1, 1, 64, 128, 1024, 65, null, null,
                             0, null) == 1
    assert c.misa_score_topk_noalloc(null, null, null, null, null, 1, 1, 64, 128, 1024, 65, 16,
                                     null, null, null, null) == 1
    # test-only entry points: bad wait bound, skip index, gather pair, output stride
    assert c.misa_testing_score_rows_wait_expiry(null, null, null, null, null, 1, 1, 8, 128, 1024,
                                                 8, null, null, 0, 10, -1, null) == 1
    assert c.misa_testing_score_rows_wait_expiry(null, null, null, null, null, 1, 1, 8, 128, 1024,
                                                 8, null, null, 0, 100000, -2, null) == 1
    assert c.misa_testing_score_simt(null, null, null, null, null, null, null, 1, 1, 8, 128,
                                     1024, 8, 512, null, null, 0, null) == 1
    # topk < 1, topk > 16384
    assert c.dsa_score_topk(null, null, null, null, 1, 1, 64, 128, 1024, 0, null, null, null,
                            null, 0, null) == 1
    assert c.dsa_score_topk(null, null, null, null, 1, 1, 64, 128, 1024, 16385, null, null,
                            null, null, 0, null) == 2
    # k' < k
    assert c.misa_dagger_rerank(null, null, null, null, null, 1, 1, 64, 128, 1024, 8, 16, null,
                                null, null, 0, null) == 1
    assert c.misa_check_device_status(null, null) == 1


def test_status_strings(lib):
    c = lib.library()
    for code in range(0, 8):
        assert c.misa_status_string(code)
    assert c.misa_status_string(99) == b"unknown status"
