"""Failure detection on the GPU without a GPU fault: a bounded wait that nothing satisfies ends
after its time limit with a status the host reads, and the context keeps working."""
import time

import pytest
import torch

import long_context_attention_rkv_b200 as rkv
import synth
from gpu_harness import DeviceRun, check_compress, check_decode, check_refs, unit_rows

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_with_timeout_status_and_context_stays_usable():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    rkv.rkv_selftest_wait_timeout(err)
    torch.cuda.synchronize()
    took = time.perf_counter() - t0
    assert int(err.item()) == rkv.STATUS_CODE["RKV_ERR_TIMEOUT"]
    assert 1.5 < took < 60.0, f"the wait gave up after {took:.2f} s (limit 2 s)"
    # the same context then runs the whole path against the oracle
    wl = synth.WORKLOADS["tiny"]
    lengths = wl.lengths()
    K, V = synth.gen_layer(wl, 0, lengths)
    run = DeviceRun(wl, K, V, lengths)
    for b, n in enumerate(lengths):
        for h in range(wl.n_kv_heads):
            g = run.unit(b, h)
            Xk, Xv = unit_rows(wl, K, V, b, h, n)
            check_refs(wl, g, Xk, Xv)
            check_compress(wl, g, Xk, Xv)
    check_decode(run, synth.gen_query(wl, 0, 0))
    assert run.layer.device_error() == 0
