"""The allocation-free sort entry point (gs_sort_keys32_noalloc).

It exists for callers that cannot allocate device memory when they need a
sort (a plugin inside a host application whose allocator owns the device, a
latency-critical loop that must not risk an allocation's implicit device
synchronisation): its scratch is an array inside the library instead of a
caller workspace.  This test calls it through the C ABI several times in a
row on different data and sizes, with the default passes and with the
onesweep look-back (which clears a larger part of the shared array), and
checks each result against numpy's stable argsort of the keys' sorted bits
and against gs_sort_keys32 with a normal workspace (integer results:
exact).  It also checks that sizes above the stated maximum and the
bounded-wait test hook are refused.  It lives in a file of its own,
collected last, and passes both alone in a fresh process and after the rest
of the suite.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def b():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    from gaussian_splatting_differentiable_dgs_b200 import binding
    return binding


def _workspace_sort(b, keys, lo, hi):
    n = len(keys)
    kin = torch.as_tensor(keys.view(np.int32)).cuda()
    kout = torch.empty_like(kin)
    vals = torch.empty(n, dtype=torch.int32, device="cuda")
    ws = torch.empty(b.gs_sort_workspace_size(n, 4, lo, hi), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.gs_sort_keys32(kin, kout, vals, n, lo, hi, b.GS_SORT_IOTA, ws, st)
    assert b.gs_check(st) == 0
    return kout.cpu().numpy().view(np.uint32), vals.cpu().numpy()


def test_noalloc_sort_matches_stable_argsort(b):
    L = b.lib()
    rng = np.random.default_rng(11)
    cases = [(b.SORT_NOALLOC_MAX_N, 0, 32, 0), (100_003, 3, 27, 0),
             (b.SORT_NOALLOC_MAX_N, 0, 32, b.GS_SORT_ONESWEEP), (4097, 8, 24, 0),
             (77_777, 0, 32, b.GS_SORT_ONESWEEP)]
    for n, lo, hi, extra in cases:  # calls in a row: different sizes, data and passes
        keys = rng.integers(0, 1 << 32, n, dtype=np.uint64).astype(np.uint32)
        keys[::5] = keys[1]  # ties: the sort must be stable
        digit = (keys.astype(np.uint64) >> np.uint64(lo)) & np.uint64((1 << (hi - lo)) - 1)
        order = np.argsort(digit, kind="stable").astype(np.int32)
        kin = torch.as_tensor(keys.view(np.int32)).cuda()
        kout = torch.full_like(kin, -1)
        vals = torch.full((n,), -1, dtype=torch.int32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        stream = torch.cuda.current_stream().cuda_stream
        rc = L.gs_sort_keys32_noalloc(kin.data_ptr(), kout.data_ptr(), vals.data_ptr(), n, lo,
                                      hi, b.GS_SORT_IOTA | extra, st.data_ptr(), stream)
        assert rc == b.GS_OK
        assert b.gs_check(st) == 0
        got_v = vals.cpu().numpy()
        got_k = kout.cpu().numpy().view(np.uint32)
        assert (got_v == order).all(), (n, lo, hi, extra)
        assert (got_k == keys[order]).all()
        ref_k, ref_v = _workspace_sort(b, keys, lo, hi)
        assert (got_k == ref_k).all() and (got_v == ref_v).all()


def test_noalloc_sort_rejects_sizes_above_the_maximum_and_the_test_hook(b):
    L = b.lib()
    n = b.SORT_NOALLOC_MAX_N + 1
    rc = L.gs_sort_keys32_noalloc(None, None, None, n, 0, 32, b.GS_SORT_IOTA, None, None)
    assert rc == b.GS_ERR_CAPACITY
    assert L.gs_sort_keys32_noalloc(None, None, None, -1, 0, 32, 0, None, None) == b.GS_ERR_ARG
    stall = b.GS_SORT_IOTA | b.GS_SORT_TEST_STALL
    assert L.gs_sort_keys32_noalloc(None, None, None, 16, 0, 32, stall, None, None) == b.GS_ERR_ARG
