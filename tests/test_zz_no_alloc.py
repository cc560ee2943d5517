"""nv_philox4x32_10_noalloc, the entry point for callers that cannot
allocate device memory (a framework's caching allocator holds the device, or
a loop cannot afford cudaMalloc's synchronisation): through the C ABI, its
output equals the allocating nv_philox4x32_10's, bit for bit (integer
results), on two calls in a row, which share and reuse its fixed staging
array.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

from oracle import nvium_oracle as O

pytestmark = pytest.mark.gpu

nv = pytest.importorskip("exact_early_exit_b200")


def _noalloc(seed, ctr):
    out = np.zeros_like(ctr)
    st = nv.lib().nv_philox4x32_10_noalloc(ctypes.c_uint64(seed), ctr.ctypes.data, ctr.shape[0], out.ctypes.data,
                                           None)
    assert st == nv.NV_OK, nv.lib().nv_last_error()
    return out


def test_noalloc_matches_the_allocating_entry_point_on_two_calls():
    rng = np.random.default_rng(7)
    # first call fills most of the array, the second a smaller prefix: the
    # second must not see anything left over from the first
    for seed, n in ((0xDEADBEEF12345678, nv.NV_PHILOX_NOALLOC_MAX), (1234, 4099)):
        ctr = rng.integers(0, 2**32, size=(n, 4), dtype=np.uint64).astype(np.uint32)
        ref = nv.philox4x32_10(seed, ctr)
        got = _noalloc(seed, ctr)
        np.testing.assert_array_equal(got, ref)
        # and against the CPU oracle's Philox4x32-10 (pinned to the published
        # known-answer vectors) on a sample of the counters
        idx = rng.choice(n, size=512, replace=False)
        c = ctr[idx].astype(np.uint64)
        want = O.philox4x32_10([c[:, 0], c[:, 1], c[:, 2], c[:, 3]],
                               (np.uint64(seed & 0xFFFFFFFF), np.uint64(seed >> 32)))
        np.testing.assert_array_equal(got[idx], np.stack(want, axis=1).astype(np.uint32))


def test_noalloc_rejects_more_than_its_limit():
    n = nv.NV_PHILOX_NOALLOC_MAX + 1
    ctr = np.zeros((n, 4), np.uint32)
    out = np.zeros_like(ctr)
    st = nv.lib().nv_philox4x32_10_noalloc(ctypes.c_uint64(1), ctr.ctypes.data, n, out.ctypes.data, None)
    assert st == nv.NV_ERR_INVALID_ARG
    assert b"NV_PHILOX_NOALLOC_MAX" in nv.lib().nv_last_error()
