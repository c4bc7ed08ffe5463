"""The schedule of the device-side triangular inverse (csrc/w4_linalg.cu,
inverse_factor), replayed on the CPU with numpy products in place of the
GEMM launches: level b joins diagonal blocks 2p (size b) and 2p + 1 (size
cs <= b, smaller only for the last block) as
    [A 0; B C]^-1 = [A^-1 0; -C^-1 B A^-1, C^-1],
an unpaired last block carries over, and the pairs of a level are split into
the full ones (one batched launch) and the partial last one.  The replay uses
the same element offsets, batch strides and k-range cuts (k_from_n: the
triangular B operand starts at the tile's column; k_to_m: the triangular A
operand ends at the tile's row) and must give numpy's inverse for every
block count, powers of two or not.  No GPU."""
import numpy as np
import pytest

NB = 64


def gemm(A, lda, B, ldb, C, ldc, M, N, K, alpha, sA, sB, sC, batch, k_from_n=False,
         k_to_m=False, A0=0, B0=0, C0=0, bnc=True):
    """C(m, n) = alpha * sum_k A(m, k) B(n, k) on flat arrays, A k-contiguous,
    B n-contiguous (B(n, k) = B[k * ldb + n]), whole matrices (tile cuts are
    exact zeros of the triangular operands, so they are applied per element)."""
    for z in range(batch):
        a = A[A0 + z * sA:]
        b = B[B0 + z * sB:]
        for m in range(M):
            for n in range(N):
                k0 = n if k_from_n else 0
                k1 = min(K, m + 1) if k_to_m else K
                acc = 0.0
                for k in range(k0, k1):
                    acc += a[m * lda + k] * b[k * ldb + n]
                C[C0 + z * sC + m * ldc + n] = alpha * acc


def invert_by_schedule(L):
    n = L.shape[0]
    P = L.reshape(-1).copy()                      # L, row-major
    Linv = np.zeros(n * n)
    for kb in range(n // NB):                     # the inverted diagonal blocks
        blk = np.linalg.inv(L[kb * NB:(kb + 1) * NB, kb * NB:(kb + 1) * NB])
        for i in range(NB):
            Linv[(kb * NB + i) * n + kb * NB:(kb * NB + i) * n + (kb + 1) * NB] = blk[i]
    Y = np.zeros(n * n // 4)
    b = NB
    while b < n:
        nblk = (n + b - 1) // b
        npair = nblk // 2
        last_cs = n - (2 * npair - 1) * b
        full = npair if last_cs >= b else npair - 1
        for part in range(2):
            p0 = 0 if part == 0 else full
            cnt = full if part == 0 else npair - full
            if cnt <= 0:
                continue
            cs = b if part == 0 else last_cs
            off = p0 * (2 * b * n + 2 * b)
            stride = 2 * b * n + 2 * b
            # Y_p = B_p A_p^-1 (cs x b), A_p^-1 lower: k from the column
            gemm(P, n, Linv, n, Y, b, cs, b, b, 1.0, stride, stride, b * b, cnt,
                 k_from_n=True, A0=off + b * n, B0=off, C0=0)
            # Linv[(2p+1)b.., 2pb..] = -C_p^-1 Y_p, C_p^-1 lower: k up to the row
            gemm(Linv, n, Y, b, Linv, n, cs, b, cs, -1.0, stride, b * b, stride, cnt,
                 k_to_m=True, A0=off + b * n + b, B0=0, C0=off + b * n)
        b *= 2
    return Linv.reshape(n, n)


@pytest.mark.parametrize("blocks", [2, 3, 5, 6])
def test_schedule_inverts_every_block_count(blocks):
    n = blocks * NB
    rng = np.random.default_rng(blocks)
    L = np.tril(rng.uniform(-0.2, 0.2, (n, n)))
    L[np.diag_indices(n)] = rng.uniform(1.0, 2.0, n)
    got = invert_by_schedule(L)
    assert np.allclose(np.triu(got, 1), 0.0)
    np.testing.assert_allclose(got, np.linalg.inv(L), rtol=0, atol=1e-10)
