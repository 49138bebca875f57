"""The router's transposed lane butterfly (route.cu, tree_sum) restated in
numpy float32: for N accumulators per lane, each of the levels 16, 8, 4, 2, 1
keeps half of the live values on each lane and adds the partner's copy of
that half, and lane l ends with accumulator l >> (5 - log2 N).  Every sum it
forms has the same two operands as the plain xor butterfly of that
accumulator, so the result must be bit-identical, including for values of
very different magnitudes (where a different order would round differently)."""
import numpy as np
import pytest


def plain_butterfly(vals):
    s = vals.astype(np.float32).copy()
    for m in (16, 8, 4, 2, 1):
        s = np.array([np.float32(s[l] + s[l ^ m]) for l in range(32)], dtype=np.float32)
    return s


def transposed_butterfly(acc):
    n_acc = acc.shape[1]
    a = [list(acc[l].astype(np.float32)) for l in range(32)]
    for lvl in range(5):
        m = 16 >> lvl
        n = n_acc >> lvl
        if n > 1:
            send = [[a[l][i] if (l & m) else a[l][i + n // 2] for i in range(n // 2)] for l in range(32)]
            keep = [[a[l][i + n // 2] if (l & m) else a[l][i] for i in range(n // 2)] for l in range(32)]
            a = [[np.float32(keep[l][i] + send[l ^ m][i]) for i in range(n // 2)] for l in range(32)]
        else:
            a = [[np.float32(a[l][0] + a[l ^ m][0])] for l in range(32)]
    return np.array([a[l][0] for l in range(32)], dtype=np.float32)


@pytest.mark.parametrize("n_acc", [1, 2, 4, 8, 16, 32])
def test_transposed_butterfly_is_bit_identical(n_acc):
    rng = np.random.default_rng(n_acc)
    shift = 5 - int(np.log2(n_acc))
    for _ in range(10):
        acc = (rng.standard_normal((32, n_acc)) *
               np.exp(rng.uniform(-20, 20, (32, n_acc)))).astype(np.float32)
        out = transposed_butterfly(acc)
        for lane in range(32):
            ref = plain_butterfly(acc[:, lane >> shift])[0]
            assert out[lane].tobytes() == ref.tobytes()


def test_a_left_to_right_sum_differs():
    """The test can tell orders apart: a left-to-right sum of the same values
    differs from the butterfly on some inputs."""
    rng = np.random.default_rng(7)
    differs = 0
    for _ in range(50):
        v = (rng.standard_normal(32) * np.exp(rng.uniform(-20, 20, 32))).astype(np.float32)
        seq = np.float32(0)
        for x in v:
            seq = np.float32(seq + x)
        differs += int(seq.tobytes() != plain_butterfly(v)[0].tobytes())
    assert differs > 0
