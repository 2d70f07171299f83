"""The library's failure paths on the GPU, driven without a fault or a hang
(fm.h "failure-path test hooks"):
  * a scoring launch whose query operand is withheld: its bounded wait runs
    out, the launch ends, fm_sync_status reports FM_ERR_DEVICE, and the next
    launch on the same context is correct again;
  * a device allocation made to fail at every position inside fm_create and
    fm_level2_create: FM_ERR_OOM, no handle, and nothing left allocated."""
import ctypes

import numpy as np
import pytest
import torch

from gen import synthetic as G
from tests import helpers as H

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from learned_kv_chunk_b200 import fm  # noqa: E402  (loads libfm.so; raises if missing)

DEV = torch.device("cuda", 0)
N_CREATE_ALLOCS = 16   # device allocations fm_create makes
N_LEVEL2_ALLOCS = 8    # device allocations fm_level2_create makes


@pytest.fixture(scope="module")
def weights():
    return G.make_weights(4545, 3)


def test_stalled_launch_reports_device_error_and_context_recovers(weights):
    case = H.make_case(2, 1000, [1000, 777], seed=41, weights=weights)
    r = fm.Retriever(weights, device=0, max_batch=4)
    lib = fm.lib()
    try:
        keys = [k.to(DEV) for k in case.comp_k]
        q, w = r.fm_query_prep(case.hidden.to(DEV), case.positions.to(DEV))
        nv = case.n_valid.to(DEV)
        good, _, _ = r.fm_score_fused(keys, q, w, n_valid=nv, N=case.N)
        good = good.clone()
        r.fm_sync_status()
        assert lib.fm_debug_stall_next_score(r.handle, 0) == fm.FM_ERR_INVALID_ARG
        assert lib.fm_debug_stall_next_score(r.handle, ctypes.c_uint64(1_000_000)) == fm.FM_OK
        ens = torch.full_like(good, -1.0)
        r.fm_score_fused(keys, q, w, n_valid=nv, N=case.N, ens=ens)  # the launch itself succeeds
        st = lib.fm_sync_status(r.handle, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == fm.FM_ERR_DEVICE
        r.fm_sync_status()  # the record was cleared
        again, _, _ = r.fm_score_fused(keys, q, w, n_valid=nv, N=case.N)
        torch.cuda.synchronize()
        r.fm_sync_status()
        assert torch.equal(again, good)
    finally:
        r.close()


def _create(weights, max_batch=4):
    cfg = fm.fm_config_default()
    cfg.max_batch = max_batch
    lw = (fm.fm_layer_weights * 3)()
    keep = []
    for l, wd in enumerate(weights):
        ts = [wd[k].contiguous() for k in ("wq_a", "q_norm", "wq_b", "weights_proj")]
        keep.extend(ts)
        lw[l].wq_a, lw[l].q_norm, lw[l].wq_b, lw[l].weights_proj = [t.data_ptr() for t in ts]
    h = ctypes.c_void_p()
    st = fm.lib().fm_create(ctypes.byref(cfg), lw, 0, ctypes.byref(h))
    return st, h


def test_create_fails_cleanly_at_every_allocation(weights):
    lib = fm.lib()
    torch.cuda.synchronize()
    live0 = lib.fm_debug_live_allocations()
    try:
        for n in range(1, N_CREATE_ALLOCS + 1):
            lib.fm_debug_fail_alloc(n)
            st, h = _create(weights)
            assert st == fm.FM_ERR_OOM, (n, st)
            assert not h.value
            assert lib.fm_debug_live_allocations() == live0, n
        lib.fm_debug_fail_alloc(N_CREATE_ALLOCS + 1)  # past the last one: create succeeds
        st, h = _create(weights)
        assert st == fm.FM_OK and h.value
        assert lib.fm_debug_live_allocations() == live0 + N_CREATE_ALLOCS
        assert lib.fm_destroy(h) == fm.FM_OK
        assert lib.fm_debug_live_allocations() == live0
    finally:
        lib.fm_debug_fail_alloc(0)


def test_level2_create_fails_cleanly_at_every_allocation(weights):
    lib = fm.lib()
    B, R = 2, 256
    r = fm.Retriever(weights, device=0, max_batch=B)
    try:
        keys = G.make_keys(46, [R] * B, R, 3, None, device=DEV)
        ids = torch.arange(R, dtype=torch.int32, device=DEV).repeat(B, 1).contiguous()
        count = torch.full((B,), R, dtype=torch.int32, device=DEV)
        live0 = lib.fm_debug_live_allocations()
        for n in range(1, N_LEVEL2_ALLOCS + 1):
            lib.fm_debug_fail_alloc(n)
            with pytest.raises(fm.FMError) as exc:
                fm.Level2Step(r, keys, ids, count, k=64)
            assert exc.value.status == fm.FM_ERR_OOM, n
            assert lib.fm_debug_live_allocations() == live0, n
        lib.fm_debug_fail_alloc(0)
        step = fm.Level2Step(r, keys, ids, count, k=64)
        assert lib.fm_debug_live_allocations() == live0 + N_LEVEL2_ALLOCS
        step.close()
        assert lib.fm_debug_live_allocations() == live0
        r.fm_sync_status()
    finally:
        lib.fm_debug_fail_alloc(0)
        r.close()
