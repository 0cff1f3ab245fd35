"""The allocation-free ridge-fit entry point (sparsepr_ridge_fit_static) against the regular
one (needs a B200).

It exists for callers that cannot allocate device memory when they fit the correction; the
test feeds it the probe rows of a regular call (plan / attention / fit_apply) and checks that
it returns that call's fitted map exactly (both paths sum the same probe rows in the same
order and share the solve and projection kernels), on three different calls in a row: the
static scratch keeps the previous call's contents, and the third call has fewer heads and
fewer probe rows than the one before it, so rows left over from that call would show.  This file is
collected last so that a run stopping at the first failure has run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

from free_block_sparse_02_b200 import build, configs, gen
from free_block_sparse_02_b200 import _lib as S

pytestmark = pytest.mark.gpu


def _entry():
    build.build()
    f = S.load().sparsepr_ridge_fit_static
    vp = ctypes.c_void_p
    f.restype = ctypes.c_int32
    f.argtypes = [vp, vp, vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_double, vp, vp, vp]
    return f


def _regular_call(w, variant):
    op = S.SparsePR(w)
    Q, K, V = gen.make_qkv(w, variant=variant)
    op(Q.cuda(), K.cuda(), V.cuda(), out_dtype=torch.float32)
    op.sync()
    probes = op.query(S.Q_PROBES)
    osp = op.query(S.Q_OSP)
    osp_p = np.stack([osp[h][probes[h]] for h in range(osp.shape[0])])
    return osp_p, op.query(S.Q_ODENSE), op.query(S.Q_PROBE_W), op.query(S.Q_FIT)


CASES = [
    (configs.scaled_down(configs.workload(1), heads=2, grid=(4, 16, 32), s=64, n_kgroups=16, n_qgroups=16,
                         P=48, km_iters=6), 0),
    (configs.scaled_down(configs.workload(2), heads=3, grid=(3, 10, 20), s=96, n_kgroups=16, n_qgroups=12,
                         P=40, km_iters=6), 1),
    (configs.scaled_down(configs.workload(2), heads=1, grid=(3, 10, 20), s=96, n_kgroups=16, n_qgroups=12,
                         P=24, km_iters=6), 2),
]


def test_static_ridge_fit_matches_fit_apply_on_consecutive_calls():
    f = _entry()
    stream = torch.cuda.current_stream().cuda_stream
    for w, variant in CASES:
        osp_p, od, pw, A_ref = _regular_call(w, variant)
        H, P, d = osp_p.shape
        t_osp = torch.from_numpy(np.ascontiguousarray(osp_p)).cuda()
        t_od = torch.from_numpy(np.ascontiguousarray(od)).cuda()
        t_w = torch.from_numpy(np.ascontiguousarray(pw)).cuda()
        A = torch.full((H, d + 1, d), float("nan"), dtype=torch.float64, device="cuda")
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        rc = f(t_osp.data_ptr(), t_od.data_ptr(), t_w.data_ptr(), H, P, d, w.lam, A.data_ptr(),
               status.data_ptr(), stream)
        assert rc == 0
        torch.cuda.synchronize()
        assert status.item() == 0
        got = A.cpu().numpy()
        assert np.isfinite(got).all()
        assert np.array_equal(got, A_ref), f"max difference {np.abs(got - A_ref).max():.3e}"


def test_static_ridge_fit_rejects_sizes_beyond_its_scratch():
    f = _entry()
    t = torch.zeros(1, dtype=torch.float64, device="cuda")
    p = t.data_ptr()
    assert f(p, p, p, 17, 8, 64, -1.0, p, None, None) == 4        # more heads than the scratch holds
    assert f(p, p, p, 2, 5000, 64, -1.0, p, None, None) == 4      # more probes than the scratch holds
    assert f(p, p, p, 2, 8, 96, -1.0, p, None, None) == 2         # unsupported head dimension
    assert f(None, None, None, 2, 8, 64, -1.0, p, None, None) == 1
