"""The parity tests' reconstruction of a GPU kept set (rtp_check.gpu_kept),
checked on the CPU against fp32 selections made the way the kernels make them:
fp32 scores, cut key = tie key, keep s32 > t or (s32 == t and j <= jtie)."""
import numpy as np
import torch

from rtp_check import bits, f64, gpu_kept


def to_bits(x):
    return bits(torch.tensor(np.asarray(x, np.float32)).bfloat16())


def fp32_selection(q16, k16, count, rng):
    """A kept set of `count` keys under fp32 scores summed in a random order."""
    perm = rng.permutation(16)
    q = f64(q16).astype(np.float32)[perm]
    k = f64(k16).astype(np.float32)[:, perm]
    s = np.zeros(k.shape[0], np.float32)
    for d in range(16):
        s = (s + k[:, d] * q[d]).astype(np.float32)
    j = np.arange(s.size)
    order = np.lexsort((j, -s))
    c = int(order[count - 1])
    t = s[c]
    kept = (s > t) | ((s == t) & (j <= c))
    return kept, float(t), c


def test_gpu_kept_matches_fp32_selection():
    rng = np.random.default_rng(5)
    n_forced = n_amb = 0
    for trial in range(300):
        n = int(rng.integers(1, 3000))
        # coarse values make many exact and near ties
        k16 = to_bits(np.round(rng.normal(size=(n, 16)) * 4) / 4)
        if trial % 2:  # repeated key rows: exact ties that only the index orders
            k16 = k16[rng.integers(0, n // 8 + 1, n)]
        q16 = to_bits(rng.normal(size=16))
        count = int(rng.integers(1, n + 1))
        kept, t, c = fp32_selection(q16, k16, count, rng)
        assert kept.sum() == count
        mask, amb = gpu_kept(q16, k16, n - 1, t, c, count, 0.9)
        assert mask.sum() == count
        if amb is None:
            n_forced += 1
            assert np.array_equal(mask, kept)
        else:  # the two sets differ only inside the undecided keys
            n_amb += 1
            assert not np.any((mask ^ kept) & ~amb)
    assert n_forced > 100 and n_amb > 20
