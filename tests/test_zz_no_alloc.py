"""mpe_route_noalloc: the bucketing step for callers that cannot allocate device
memory while they route (a serving engine with a fixed GPU memory plan, or code
running while another component owns the allocator). Its working memory is a
file-scope device array inside the library instead of context scratch.

Called through the C ABI and compared with mpe_route, the existing entry point,
on consecutive calls that reuse the shared array (results must be identical:
this is integer work), and, in a fresh process before any context exists, at
the largest expert count with the oracle's bucketing. Collected last so that a
failure here comes after every other test has run.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

mpe = pytest.importorskip("mixed_precision_expert_b200")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_expert_b200.build import build
    build()
    assert torch.cuda.is_available()


def _noalloc(L, ids, E):
    T, k = ids.shape
    n = T * k
    perm = torch.full((max(n, 1),), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((max(n, 1),), -7, dtype=torch.int32, device="cuda")
    offs = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = L.mpe_route_noalloc(ids.data_ptr(), T, k, E, perm.data_ptr(), offs.data_ptr(),
                             inv.data_ptr(), stream)
    assert rc == 0, L.mpe_last_error_global()
    torch.cuda.synchronize()
    return perm[:n].cpu().numpy(), offs.cpu().numpy(), inv[:n].cpu().numpy()


def test_route_noalloc_matches_route_on_consecutive_calls():
    L = mpe.lib()
    E = 128
    ctx = mpe.Context(E, 128, 128)
    rng = np.random.default_rng(2024)
    # two multi-chunk calls in a row (the shared histograms are reused), then a
    # single-chunk call
    cases = [(8192, 8), (5000, 3), (300, 3)]
    for T, k in cases:
        ids_np = rng.integers(0, E, size=(T, k)).astype(np.int32)
        ids_np[0, 0] = E + 5  # a dropped id
        ids = torch.from_numpy(ids_np).cuda()
        perm, offs, inv = _noalloc(L, ids, E)
        rp, ro, ri = ctx.route(ids)
        torch.cuda.synchronize()
        assert np.array_equal(offs, ro.cpu().numpy())
        nvalid = int(offs[-1])
        assert np.array_equal(perm[:nvalid], rp.cpu().numpy()[:nvalid])
        assert np.array_equal(inv, ri.cpu().numpy())
        assert inv[0] == -1
    # an empty batch writes only the offsets (all zero)
    empty = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    _, offs, _ = _noalloc(L, empty, E)
    assert np.all(offs == 0)


def test_route_noalloc_rejects_sizes_beyond_its_maximum():
    L = mpe.lib()
    ids = torch.zeros((65537, 1), dtype=torch.int32, device="cuda")
    buf = torch.zeros(65537, dtype=torch.int32, device="cuda")
    offs = torch.zeros(9, dtype=torch.int32, device="cuda")
    rc = L.mpe_route_noalloc(ids.data_ptr(), 65537, 1, 8, buf.data_ptr(), offs.data_ptr(),
                             buf.data_ptr(), None)
    assert rc == -1
    assert b"65536" in L.mpe_last_error_global()


# Runs in a fresh interpreter: no mpe.Context is created before the calls, so
# the entry point's own set-up (the array's address, the shared-memory limit
# that the single-chunk kernel needs at 1,024 experts) is what makes them work.
_FRESH = r"""
import sys
import numpy as np
import torch
sys.path[:0] = [sys.argv[1], sys.argv[2]]
import mixed_precision_expert_b200 as mpe
from oracle import route as orr
L = mpe.lib()
E = mpe.MAX_EXPERTS
rng = np.random.default_rng(77)
stream = torch.cuda.current_stream().cuda_stream
for T, k in ((128, 8), (1000, 1), (300, 3)):   # single-chunk calls, T*k <= 1024
    ids_np = rng.integers(0, E, size=(T, k)).astype(np.int32)
    ids_np[rng.integers(0, T), 0] = -3             # a dropped id
    ids = torch.from_numpy(ids_np).cuda()
    n = T * k
    perm = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    offs = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    rc = L.mpe_route_noalloc(ids.data_ptr(), T, k, E, perm.data_ptr(), offs.data_ptr(),
                             inv.data_ptr(), stream)
    assert rc == 0, L.mpe_last_error_global()
    torch.cuda.synchronize()
    rp, ro, ri = orr.route(ids_np, E)
    assert np.array_equal(offs.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy()[:int(ro[-1])], rp)
    assert np.array_equal(inv.cpu().numpy(), ri)
    ctx = mpe.Context(E, 128, 128)
    p2, o2, i2 = ctx.route(ids)
    assert np.array_equal(o2.cpu().numpy(), ro) and np.array_equal(i2.cpu().numpy(), ri)
    ctx.close()
print("FRESH-OK")
"""


def test_route_noalloc_first_call_in_fresh_process_at_max_experts():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    tests = os.path.join(root, "tests")
    r = subprocess.run([sys.executable, "-c", _FRESH, root, tests], capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and "FRESH-OK" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
