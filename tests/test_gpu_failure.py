"""Failure detection on the GPU without a fault: a device-side wait that can
never complete gives up after the library's bound, records LL_ERR_TIMEOUT in
the device error word, and leaves the context usable."""
import time

import numpy as np
import pytest
import torch

import sink_window_attention_b200 as swa
import swa_workloads as W
from oracle import rope as orope
from oracle.stream import StreamOracle
from tests.conftest import assert_parity

pytestmark = pytest.mark.gpu

K_ERR_WAIT_TIMEOUT = 1  # the device error word's timeout bit


def test_bounded_waits_report_timeout_and_context_survives():
    from sink_window_attention_b200 import build
    build.build()
    assert swa.device_error() == 0
    t0 = time.time()
    code = swa.selftest_bounded_waits()
    dt = time.time() - t0
    assert code & K_ERR_WAIT_TIMEOUT, code
    assert 0.2 < dt < 60.0, dt  # two waits of about a second of SM clocks each
    assert swa.device_error() == 0  # read and cleared
    # the context still runs the library: one small stream step against the oracle
    w = W.replace(W.TINY, dtype="bf16", name="after_timeout")
    rope = swa.Rope(pairs=w.pairs, grid_h=w.grid_h, grid_w=w.grid_w, theta0=w.theta0)
    om = orope.head_frequencies(w.H, w.pairs, w.theta0)
    so = StreamOracle(w.H, w.D, w.grid_h, w.grid_w, om, w.pairs, w.t_offset)
    cache = swa.KVCache(1, w.H, w.D, w.N, "bf16")
    for f in range(3):
        q, k, v = W.qkv_frames(w, 0, f, 1)
        out = swa.append_and_attend(cache, k.cuda(), v.cuda(), q.cuda(), f, rope)
        so.append(f, k[0].double().numpy(), v[0].double().numpy())
    torch.cuda.synchronize()
    ref = so.attend(q[0].double().numpy(), 2)
    assert_parity(out[0].double().cpu().numpy(), ref, what="after timeout")
    assert swa.device_error() == 0
