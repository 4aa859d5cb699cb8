"""Failure handling on the GPU without a fault: a wait that nothing satisfies gives up
after its limit and reports through the device error word, the context stays usable,
and a decode grid that sees the timeout bit stops early with NaN output."""
import time

import numpy as np
import pytest
import torch

from paged_kv_cache_324_b200 import binding as B
from paged_kv_cache_324_b200 import workload as wl
from tests import harness as H
from tests.parity import attention_close

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    err = torch.zeros(1, dtype=torch.int32, device="cuda:0")
    t0 = time.perf_counter()
    B.selftest_bounded_wait(err, 20_000)          # 20 ms
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(err.item()) & B.DEVERR_TIMEOUT
    assert 0.015 < dt < 5.0
    # the context is still usable: a small decode step matches the oracle afterwards
    w = wl.make("tiny")
    g = H.gpu_step(w, keep_pools=False)
    o = H.oracle_step(w)
    assert g["err"] == 0
    assert attention_close(g["out"], o["out"], w.kv_dtype, w.q_dtype)[0]


def test_decode_stops_early_after_a_timeout_in_the_same_error_word():
    w = wl.make("tiny")
    dev = torch.device("cuda:0")
    kp = H.to_dev_bits(w.initial_pool("k"), w.kv_dtype, dev)
    vp = H.to_dev_bits(w.initial_pool("v"), w.kv_dtype, dev)
    q = H.to_dev_bits(w.q, w.q_dtype, dev)
    out = torch.zeros_like(q)
    err = torch.full((1,), B.DEVERR_TIMEOUT, dtype=torch.int32, device=dev)
    B.paged_attn_decode(out, q, kp, vp, torch.from_numpy(w.block_tables).to(dev),
                        torch.from_numpy(w.context_lens).to(dev), float(w.scale),
                        max_context_len=w.max_context_len, device_error=err)
    torch.cuda.synchronize()
    assert np.isnan(H.out_f64(out)).all()


def test_selftest_rejects_bad_arguments():
    err = torch.zeros(1, dtype=torch.int32, device="cuda:0")
    with pytest.raises(B.PagedKVError):
        B.selftest_bounded_wait(err, 0)
