"""Range-encoded Skip-List on the GPU vs the oracle, bit-exact (needs a B200)."""

import numpy as np
import pytest
import torch

import oracle
from temporal_block_sparse_b200 import lite_attn as la

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(autouse=True)
def _clean_state():
    la.load()
    yield
    assert la.lite_get_device_status() == 0


def _random_mask(B, H, N, d, density, seed, banded=False):
    _, T, W = la.lite_mask_geometry(N, d)
    rng = np.random.default_rng(seed)
    skip = rng.random((B, H, T, T)) >= density
    if banded:  # live bands around the diagonal plus a few far tiles: few long runs
        i = np.arange(T)[:, None]
        j = np.arange(T)[None, :]
        skip = np.abs(i - j) > (3 + (i % 5))
        skip = np.broadcast_to(skip, (B, H, T, T)).copy()
        skip &= rng.random((B, H, T, T)) > 0.02
    bits = np.zeros((B, H, T, W * 32), dtype=bool)
    bits[..., :T] = skip
    words = np.packbits(bits.reshape(B, H, T, W, 32), axis=-1, bitorder="little").view(np.uint32)[..., 0]
    return words, T


@pytest.mark.parametrize("B,H,N,d,density,banded", [
    (1, 1, 64, 64, 0.5, False),       # T = 1
    (1, 2, 1024, 64, 0.5, False),     # T = 16
    (2, 3, 2100, 64, 0.3, False),     # T = 33: two words, ragged
    (1, 4, 32760, 128, 0.1, False),   # T = 256
    (1, 2, 75600, 128, 0.0, True),    # T = 591, banded runs
    (2, 2, 75600, 128, 1.0, False),   # all live
    (1, 2, 75600, 128, 0.0, False),   # all skipped
])
def test_ranges_bit_exact(B, H, N, d, density, banded):
    words, T = _random_mask(B, H, N, d, density, seed=N + H, banded=banded)
    mask = torch.from_numpy(words.view(np.int32)).cuda()
    ranges, nruns = la.lite_mask_to_ranges(mask, B, H, N, d)
    want_r, want_n = oracle.mask_to_ranges(words, T)
    got_n = nruns.cpu().numpy()
    np.testing.assert_array_equal(got_n, want_n)
    got_r = ranges.cpu().numpy()
    for idx in np.ndindex(B, H, T):
        n = 2 * int(want_n[idx])
        np.testing.assert_array_equal(got_r[idx][:n], want_r[idx][:n])


def test_ranges_without_mask_is_one_run():
    ranges, nruns = la.lite_mask_to_ranges(None, 1, 2, 5000, 128)
    _, T, _ = la.lite_mask_geometry(5000, 128)
    assert (nruns == 1).all()
    assert (ranges[..., 0] == T - 1).all() and (ranges[..., 1] == -1).all()
