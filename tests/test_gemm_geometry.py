"""Launch geometry of the 8/4-bit expert GEMM and the fused vocabulary/update GEMM, checked
on the CPU at every bf16 workload shape before their first run.

The host's choices (token rows per tile, shared-memory stages, TMEM columns, work-item
bound) and the tensor maps' coordinates are replayed and checked against the limits they
must respect: at least two pipeline stages inside the 227 KB of shared memory, at most
512 TMEM columns, TMA x coordinates and global strides on 16-byte multiples, every box
starting inside its tensor, and work lists and record buffers inside their workspace
reservations.
"""
import numpy as np
import pytest

from block_diffusion_lm_masked_b200 import configs as CF

SMEM_GEMM = 200 * 1024
SMEM_MAX = 227 * 1024
ITEM_ROWS_LOWP = 64
BF16_CONFIGS = [n for n, c in CF.CONFIGS.items() if c["dtype"] == "bf16"]


def pow2_cols(need):
    c = 32
    while c < need:
        c <<= 1
    return c


def lowp_stage(fmt, n_max, terms, n_a):
    a = 128 * 64 // 2 if fmt == "nv4" else 128 * 64
    s = 128 * 4 if fmt == "nv4" else 128 * 2
    return ((terms * n_max * 128 + n_a * (a + s)) + 1023) & ~1023, a, s


@pytest.mark.parametrize("fmt", ["mx8", "nv4"])
@pytest.mark.parametrize("name", BF16_CONFIGS)
def test_lowp_gemm_geometry(name, fmt):
    c = CF.CONFIGS[name]
    H, F, E, k = c["hidden"], c["expert_ffn"], c["n_experts"], c["top_k"]
    V = c["vocab"]
    # gate/up and down (two-term tokens), and the dense vocabulary projection (one term)
    for dual_a, K, rows, terms, n_max in ((1, H, F, 2, ITEM_ROWS_LOWP), (0, F, H, 2, ITEM_ROWS_LOWP),
                                          (0, H, V, 1, 128)):
        # host checks of launch_tc_gemm_lowp
        assert K % 64 == 0 and 16 <= n_max <= (64 if dual_a else 128) and n_max % 16 == 0
        stage, a_bytes, s_bytes = lowp_stage(fmt, n_max, terms, 1 + dual_a)
        assert SMEM_GEMM >= 2 * stage
        stages = min(SMEM_GEMM // stage, 8)
        assert stages >= 2 and stages * stage <= SMEM_GEMM and SMEM_GEMM + 1024 <= SMEM_MAX
        # TMEM: two accumulators of n_max columns per weight matrix, four decoded stages
        acc_cols = n_max * (1 + dual_a)
        need = 2 * acc_cols + 4 * 32 * (1 + dual_a)
        assert pow2_cols(need) <= 512
        # code and scale tensor maps: strides and inner boxes on 16-byte multiples, every
        # weight tile's box starting inside its tensor
        row_bytes = K // 2 if fmt == "nv4" else K
        assert row_bytes % 16 == 0 and (rows * row_bytes) % 16 == 0
        m_tiles = -(-rows // 128)
        for m in range(m_tiles):
            for kb in range(K // 64):
                ax = kb * 32 if fmt == "nv4" else kb * 64
                assert ax % 16 == 0 and ax < row_bytes and m * 128 < rows
                if fmt == "nv4":
                    assert rows % 4 == 0 and m * 32 < rows // 4                      # (16, rows / 4, E * K / 64)
                else:
                    assert (m * 256) % 16 == 0 and m * 256 < rows * 2 and kb < K // 64  # (rows * 2, K / 64, E)
        # token operand: x = k-block column (bf16), rows of the permuted token matrix
        assert (64 * 2) % 16 == 0 and (K * 2) % 16 == 0


@pytest.mark.parametrize("name", BF16_CONFIGS)
def test_work_items_fit_their_reservation(name):
    """Tiles of 64 rows over each expert's segment: at most n k / 64 + E items (the grid's
    bound) and within the workspace's T k / 64 + E + 1, for skewed and uniform routings."""
    c = CF.CONFIGS[name]
    E, k = c["n_experts"], c["top_k"]
    rng = np.random.default_rng(3)
    for n in (1, 7, 64, c["canvas"], 4 * c["canvas"]):
        for skew in (0.0, 1.0, 3.0):
            p = np.exp(-skew * np.arange(E) / E)
            p /= p.sum()
            counts = np.zeros(E, dtype=np.int64)
            for _ in range(n):
                counts[rng.choice(E, size=k, replace=False, p=p)] += 1
            items = int(sum(-(-int(x) // ITEM_ROWS_LOWP) for x in counts))
            assert items <= n * k // ITEM_ROWS_LOWP + E
            assert items <= n * k // ITEM_ROWS_LOWP + E + 1      # the buffer, with T = n


@pytest.mark.parametrize("name", BF16_CONFIGS)
@pytest.mark.parametrize("C", [1, 17, 256, 300, 1024])
def test_fused_vocab_update_geometry(name, C):
    c = CF.CONFIGS[name]
    H, V = c["hidden"], c["vocab"]
    n_max = ((C + 15) & ~15) if C < 256 else 256
    assert H % 64 == 0 and 16 <= n_max <= 256 and n_max % 16 == 0
    stage = 128 * 64 * 2 + n_max * 128
    assert SMEM_GEMM >= stage
    stages = min(SMEM_GEMM // stage, 8)
    assert stages >= 2 and SMEM_GEMM + 1024 <= SMEM_MAX
    assert pow2_cols(2 * n_max) <= 512
    m_tiles = -(-V // 128)
    # the (token, id tile) records: rows of at most n_max tokens, all inside the
    # workspace's min(T, 1024) x m_tiles reservation (the entry refuses C > 1024)
    reserved = min(C, 1024) * m_tiles
    for row0 in range(0, C, n_max):
        rows = min(n_max, C - row0)
        n_pad = (rows + 15) & ~15
        assert n_pad <= n_max
        assert ((row0 + rows - 1) * m_tiles + m_tiles - 1) < reserved
        r = 0
        while r + 64 <= n_pad:                           # 64-row token boxes start inside the tensor
            assert row0 + r < C
            r += 64
        while r < n_pad:
            assert row0 + r < C
            r += 16


@pytest.mark.parametrize("name", BF16_CONFIGS)
def test_dense_lowp_tiles_are_weight_tile_major(name):
    """Dense mode (the vocabulary projection): tile t takes weight tile t / chunks and token
    chunk t % chunks, so the CTAs of one wave cover whole weight tiles with all their token
    chunks; every (weight tile, chunk) pair is taken exactly once."""
    c = CF.CONFIGS[name]
    V, C = c["vocab"], c["canvas"]
    for n in (C, 4 * C, 37):
        chunk = ((n + 15) & ~15) if n <= 64 else 128          # the host's token chunk
        chunks, m_tiles = -(-n // chunk), -(-V // 128)
        seen = set()
        for t in range(chunks * m_tiles):
            m, row0 = t // chunks, (t % chunks) * chunk
            assert m < m_tiles and row0 < n
            seen.add((m, row0))
        assert len(seen) == chunks * m_tiles
        # one wave of 148 CTAs reads about 148 / chunks distinct weight tiles
        assert len({t // chunks for t in range(min(148, chunks * m_tiles))}) == -(-min(148, chunks * m_tiles) // chunks)
