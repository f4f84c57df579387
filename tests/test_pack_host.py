"""Host layout helpers: canonical 18-byte Q4_0 blocks (GGUF order) <-> the
library's 144-byte super-blocks.  Checked on the CPU against a reader of the
canonical block written here from the format's definition, and by round trips."""
import numpy as np
import pytest

import oracle
from bit_weight_streaming_dequant_b200 import q4dec


def _canonical_blocks(seed, rows, K):
    """Random canonical blocks: finite fp16 scales (including negative, zero and
    subnormal values) and random nibble bytes."""
    rng = np.random.default_rng(seed)
    nb = rows * K // 32
    d = rng.standard_normal(nb).astype(np.float16)
    d[::7] = np.float16(0.0)
    d[3::11] = np.float16(3e-6)          # subnormal
    blocks = np.empty((nb, 18), dtype=np.uint8)
    blocks[:, :2] = d.view(np.uint8).reshape(nb, 2)
    blocks[:, 2:] = rng.integers(0, 256, size=(nb, 16), dtype=np.uint8)
    return blocks.reshape(-1)


def _canonical_dequant(blocks, rows, K):
    """w[r][k] from canonical blocks: d = fp16 (bytes 0-1, little endian);
    byte 2 + j holds element j (low nibble) and j + 16 (high nibble)."""
    b = blocks.reshape(rows, K // 32, 18)
    d = b[:, :, :2].copy().view(np.float16).astype(np.float64)[..., 0]
    w = np.empty((rows, K // 32, 32), dtype=np.float64)
    for j in range(16):
        w[:, :, j] = d * ((b[:, :, 2 + j] & 0x0F).astype(np.float64) - 8.0)
        w[:, :, j + 16] = d * ((b[:, :, 2 + j] >> 4).astype(np.float64) - 8.0)
    return w.reshape(rows, K)


@pytest.mark.parametrize("N,K", [(1, 256), (3, 512), (17, 1024), (64, 256)])
def test_weight_packing_matches_the_canonical_reading(N, K):
    blocks = _canonical_blocks(N * 7 + K, N, K)
    W = q4dec.pack_q4_0_weights(blocks, N, K)
    assert W.size == N * K // 256 * 144
    np.testing.assert_array_equal(oracle.dequant_weights(W, N, K), _canonical_dequant(blocks, N, K))
    np.testing.assert_array_equal(q4dec.unpack_q4_0_weights(W, N, K), blocks)


@pytest.mark.parametrize("rows,K", [(1, 256), (5, 256), (9, 768)])
def test_row_packing_matches_the_canonical_reading(rows, K):
    blocks = _canonical_blocks(rows * 3 + K, rows, K)
    R = q4dec.pack_q4_0_rows(blocks, rows, K)
    np.testing.assert_array_equal(oracle.dequant(R, rows, K), _canonical_dequant(blocks, rows, K))
    np.testing.assert_array_equal(q4dec.unpack_q4_0_rows(R, rows, K), blocks)


def test_weight_layout_is_column_major_by_super_block():
    # row n, super-block s lands at (s * N + n) * 144
    N, K = 4, 512
    blocks = _canonical_blocks(5, N, K)
    W = q4dec.pack_q4_0_weights(blocks, N, K)
    R = q4dec.pack_q4_0_rows(blocks, N, K)
    for n in range(N):
        for s in range(K // 256):
            assert np.array_equal(W[(s * N + n) * 144:(s * N + n + 1) * 144],
                                  R[(n * (K // 256) + s) * 144:(n * (K // 256) + s + 1) * 144])


def test_pack_rejects_bad_arguments():
    L = q4dec.lib()
    buf = np.zeros(4096, dtype=np.uint8)
    p = buf.ctypes.data
    for fn in ("q4d_pack_q4_0_weights", "q4d_unpack_q4_0_weights", "q4d_pack_q4_0_rows",
               "q4d_unpack_q4_0_rows"):
        f = getattr(L, fn)
        assert f(None, p, 1, 256) == 1
        assert f(p, None, 1, 256) == 1
        assert f(p, p + 2048, 0, 256) == 1
        assert f(p, p + 2048, 1, 100) == 2
        assert f(p, p + 2048, 1, 0) == 2
