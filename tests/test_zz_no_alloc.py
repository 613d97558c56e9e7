"""The no-allocation entry point, cta_certified_topk_attn_noalloc.

Callers that cannot call cudaMalloc (during CUDA-graph capture, inside
runtimes that own all device memory, under a fixed memory budget) use this
entry point: the library's own fixed 32 MiB device array replaces the
workspace.  The GPU test calls it through the C ABI twice in a row, on two
different problems, and checks each result against the ordinary entry point
with the parity tolerances of tests/parity.py.  This file is collected last
on purpose and needs nothing from the other test files' state.
"""
import ctypes

import numpy as np
import pytest
import torch

import certified_top_sparse_b200 as cta
from certified_top_sparse_b200 import _lib
from certified_top_sparse_b200 import workloads as W
from parity import check_out


def _problems():
    # two shapes with different workspace layouts inside the shared scratch
    a = W.decode32k(batch=1, n_heads=8, n_kv_heads=2, n=20000, d=128, seed=77)
    b = W.tiny(n=9000, d=64, n_heads=6, seed=78)
    return [(a, 0.01), (b, 0.1)]


def _alloc_outputs(prob, dev):
    rows = (prob.batch, prob.n_heads, prob.m)
    return dict(out=torch.empty(prob.q.shape, dtype=prob.q.dtype, device=dev),
                k_out=torch.empty(rows, dtype=torch.int32, device=dev),
                idx_out=torch.full((*rows, prob.n), -1, dtype=torch.int32, device=dev),
                tv_out=torch.empty(rows, dtype=torch.float32, device=dev),
                err_out=torch.empty(rows, dtype=torch.float32, device=dev),
                kl_out=torch.empty(rows, dtype=torch.float32, device=dev))


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    dev = torch.device("cuda")
    lib = cta.load()
    for prob, eps in _problems():
        q, K, V = prob.q.to(dev), prob.K.to(dev), prob.V.to(dev)
        ref = cta.cta_certified_topk_attn(q, K, V, eps)
        o = _alloc_outputs(prob, dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        opts = _lib.make_opts(batch=prob.batch, m=prob.m, dtype=_lib._dtype_code(q),
                              stream=torch.cuda.current_stream().cuda_stream,
                              err_out=o["err_out"], kl_out=o["kl_out"], status_dev=status)
        rc = lib.cta_certified_topk_attn_noalloc(
            _lib._ptr(q), _lib._ptr(K), _lib._ptr(V), prob.n, prob.d, prob.n_heads,
            prob.n_kv_heads, eps, _lib._ptr(o["out"]), _lib._ptr(o["k_out"]),
            _lib._ptr(o["idx_out"]), _lib._ptr(o["tv_out"]), ctypes.byref(opts))
        assert rc == 0, cta.cta_status_string(rc)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        rows = prob.rows
        k_ref = ref["k"].reshape(-1).cpu().numpy()
        k_new = o["k_out"].reshape(-1).cpu().numpy()
        assert np.array_equal(k_new, k_ref)
        idx_ref = ref["idx"].reshape(rows, -1).cpu().numpy()
        idx_new = o["idx_out"].reshape(rows, -1).cpu().numpy()
        for r in range(rows):
            assert np.array_equal(idx_new[r, : k_new[r]], idx_ref[r, : k_ref[r]])
        for key, name in (("tv", "tv_out"), ("kl", "kl_out")):
            a = o[name].reshape(-1).double().cpu().numpy()
            b = ref[key].reshape(-1).double().cpu().numpy()
            assert np.all(np.abs(a - b) <= 1e-6)
        ea = o["err_out"].reshape(-1).double().cpu().numpy()
        eb = ref["err"].reshape(-1).double().cpu().numpy()
        assert np.all(np.abs(ea - eb) <= 1e-4 * eb + 1e-7)
        check_out(o["out"].float().reshape(rows, -1).cpu().numpy().astype(np.float64),
                  ref["out"].float().reshape(rows, -1).cpu().numpy().astype(np.float64),
                  prob.q.dtype)


def test_noalloc_rejects_oversized_problem_before_launch():
    """A problem whose scratch exceeds the fixed array is refused with its own
    status code; the check runs on the host before any device work."""
    lib = cta.load()
    n, d, h, kv = 1 << 20, 128, 32, 8
    assert cta.cta_workspace_size(n, d, h, kv) > cta.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)
    opts = _lib.make_opts()
    rc = lib.cta_certified_topk_attn_noalloc(fake, fake, fake, n, d, h, kv, 0.01, fake, fake, fake,
                                             fake, ctypes.byref(opts))
    assert rc == cta.CTA_ERR_TOO_LARGE
    assert "32 MiB" in cta.cta_status_string(rc)
