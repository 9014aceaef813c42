"""The device generator draws the same bits as the host generator."""
import numpy as np
import pytest

import kvattn_synth as ks
from tests import kvattn_testutil as U

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def test_device_normal_matches_host():
    t = torch.empty(1 << 20, dtype=torch.bfloat16, device="cuda")
    ks.device_normal_bf16(9, 3, t, offset=12345)
    host = ks.normal_bf16(9, 3, 12345, 1 << 20)
    # Box-Muller's log/cos may differ in the last fp64 bit between libraries;
    # after rounding to bf16 that changes essentially nothing
    assert (U.to_host(t) != host).mean() < 1e-5


def test_device_cache_fill_matches_host():
    sp = np.array([0, 5, 17], np.int32)
    c = torch.empty((3, 20, 2, 128), dtype=torch.bfloat16, device="cuda")
    ks.device_cache_fill(4, 7, c, torch.from_numpy(sp).cuda())
    host = ks.cache_fill(4, 7, 3, 20, 2, 128, sp)
    assert (U.to_host(c) != host).mean() < 1e-5
    assert np.all(U.to_host(c)[0] == 0)
