"""The banded layout of T diag(beta) and P in the tensor-core prefill's records (host-side
restatement of the layout the kernel file documents; no GPU).

Both matrices are lower triangular (64 x 64). The chain multiplies by each as the B operand
(N x K = 64 x 64, K-major) of four K steps of 16; step s only needs rows 16 s .. 63 of columns
16 s .. 16 s + 15, so a record keeps exactly those "bands": band s in the unswizzled K-major
core-matrix layout (8 rows x 16 bytes per core matrix, 128 bytes from the first to the second
core matrix of the step, 256 bytes from one 8-row group to the next), bands back to back.
Step s then issues N = 64 - 16 s into accumulator columns 16 s .. 63.

These tests check that arithmetic against its definition: the chunk index is a bijection onto
the 320 chunks of the record, the writer's walk over chunk indices inverts it, reading a band
through the descriptor strides returns the matrix block, and the banded K steps give the
same product as the full 64 x 64 operand.
"""
import numpy as np

N_CHUNKS = 320  # 16-byte chunks of one banded matrix (5,120 bytes)


def band_start(s):
    """First chunk of band s (0, 128, 224, 288; 320 past the last)."""
    return 16 * s * (9 - s)


def tri_chunk(i, c):
    """Chunk holding row i, columns 8 c .. 8 c + 7 (requires c // 2 <= i // 16)."""
    s = c >> 1
    return band_start(s) + ((i - 16 * s) >> 3) * 16 + (c & 1) * 8 + (i & 7)


def writer_decode(o):
    """(row, chunk column) that chunk index o holds, as the record writer walks them."""
    sb = int(o >= band_start(1)) + int(o >= band_start(2)) + int(o >= band_start(3))
    rest = o - band_start(sb)
    return 16 * sb + (rest >> 4) * 8 + (rest & 7), 2 * sb + ((rest >> 3) & 1)


def stored_chunks():
    return [(i, c) for i in range(64) for c in range(8) if c // 2 <= i // 16]


def pack(M):
    """The banded image of lower-triangular M as 2-byte element slots."""
    img = np.full(N_CHUNKS * 8, np.nan)
    for i, c in stored_chunks():
        o = tri_chunk(i, c)
        img[8 * o:8 * o + 8] = M[i, 8 * c:8 * c + 8]
    return img


def descriptor_read(img, s, lbo=128, sbo=256):
    """B operand of K step s (rows 16 s .. 63, 16 columns) as the tensor core reads it
    from a K-major, unswizzled descriptor starting at band s."""
    n_rows = 64 - 16 * s
    B = np.empty((n_rows, 16))
    base = 16 * band_start(s)  # bytes
    for n in range(n_rows):
        for k in range(16):
            byte = base + (n // 8) * sbo + (k // 8) * lbo + (n % 8) * 16 + (k % 8) * 2
            B[n, k] = img[byte // 2]
    return B


def lower_random(rng):
    M = np.tril(rng.standard_normal((64, 64)))
    np.fill_diagonal(M, 1.0 + rng.random(64))
    return M


def test_band_sizes():
    assert [band_start(s) for s in range(5)] == [0, 128, 224, 288, 320]
    # band s: (64 - 16 s) rows x 2 chunks; 5,120 bytes per matrix, 11,520 per record with
    # the 1,280 bytes of per-token factors
    assert all(band_start(s + 1) - band_start(s) == 2 * (64 - 16 * s) for s in range(4))
    assert 2 * 16 * N_CHUNKS + 1280 == 11520


def test_chunk_index_is_a_bijection():
    idx = [tri_chunk(i, c) for i, c in stored_chunks()]
    assert sorted(idx) == list(range(N_CHUNKS))


def test_writer_walk_inverts_the_index():
    for o in range(N_CHUNKS):
        i, c = writer_decode(o)
        assert c // 2 <= i // 16
        assert tri_chunk(i, c) == o


def test_eight_rows_of_a_chunk_column_are_contiguous():
    # the 8 rows of an 8-row group at one chunk column occupy consecutive chunks (one
    # 128-byte core matrix): conflict-free 16-byte accesses by 8 consecutive threads
    for i0 in range(0, 64, 8):
        for c in range(8):
            if c // 2 <= i0 // 16:
                o = [tri_chunk(i0 + r, c) for r in range(8)]
                assert o == list(range(o[0], o[0] + 8)) and o[0] % 8 == 0


def test_descriptor_reads_the_blocks():
    rng = np.random.default_rng(0)
    M = lower_random(rng)
    img = pack(M)
    assert not np.isnan(img).any()
    for s in range(4):
        np.testing.assert_array_equal(descriptor_read(img, s), M[16 * s:, 16 * s:16 * s + 16])


def test_banded_k_steps_give_the_full_product():
    # D = X M^T (X: 128 value rows x 64 tokens), accumulated over the four K steps with step
    # s writing only columns 16 s .. 63 (the first, N = 64, initialising all of them)
    rng = np.random.default_rng(1)
    M = lower_random(rng)
    X = rng.standard_normal((128, 64))
    img = pack(M)
    D = np.full((128, 64), np.nan)
    for s in range(4):
        B = descriptor_read(img, s)
        part = X[:, 16 * s:16 * s + 16] @ B.T
        if s == 0:
            D[:, :] = part
        else:
            D[:, 16 * s:] += part
    np.testing.assert_allclose(D, X @ M.T, rtol=1e-12, atol=1e-12)


def test_a_nonzero_above_the_bands_would_be_missed():
    # the layout relies on the zeros above the diagonal 16-blocks: a matrix with an entry
    # there gives a different product (so the test above is not vacuous)
    rng = np.random.default_rng(2)
    M = lower_random(rng)
    M[3, 40] = 1.0
    X = rng.standard_normal((128, 64))
    img = pack(M)
    D = X[:, :16] @ descriptor_read(img, 0).T
    for s in range(1, 4):
        D[:, 16 * s:] += X[:, 16 * s:16 * s + 16] @ descriptor_read(img, s).T
    assert not np.allclose(D, X @ M.T)
