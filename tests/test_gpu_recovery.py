"""Failure detection on the GPU without a GPU fault: a test hook makes one CTA skip a
barrier arrival, the kernel's bounded waits run out (about 0.2 s), the kernel unwinds
(in-flight copies drained, TMEM freed) and the status word reports DSA_ERR_TIMEOUT.
The context must stay usable: the next call is correct."""

import time

import numpy as np
import pytest
import torch

from sparse_attention_long_03_b200 import dsa
from sparse_attention_long_03_b200 import workloads as W

from dsa_testutil import DeviceWorkload, bf16_to_f64

pytestmark = pytest.mark.gpu

TIMEOUT = 6


def _tiny():
    cfg, cache, qs = W.make("tiny")
    return DeviceWorkload(cfg, cache, qs)


def test_indexer_timeout_is_reported_and_recovered():
    w = _tiny()
    ref = w.indexer()
    assert dsa.dsa_read_device_status() == 0
    dsa.dsa_debug_inject(1)
    t0 = time.time()
    w.indexer()
    st = dsa.dsa_read_device_status()
    assert st == TIMEOUT
    assert time.time() - t0 < 10.0
    again = w.indexer()
    assert dsa.dsa_read_device_status() == 0
    for t in range(w.host_q.n_tokens):  # entries past a token's position are not written
        n = int(w.host_q.tok_pos[t]) + 1
        assert torch.equal(again[t, :n], ref[t, :n])


def test_attention_timeout_is_reported_and_recovered():
    w = _tiny()
    out0, lse0, idx = w.forward()
    assert dsa.dsa_read_device_status() == 0
    dsa.dsa_debug_inject(2)
    w.attention(idx)
    assert dsa.dsa_read_device_status() == TIMEOUT
    out1, lse1 = w.attention(idx)
    assert dsa.dsa_read_device_status() == 0
    assert torch.equal(out1, out0) and torch.equal(lse1, lse0)


def test_injection_can_be_cleared():
    w = _tiny()
    dsa.dsa_debug_inject(1)
    dsa.dsa_debug_inject(0)
    w.indexer()
    assert dsa.dsa_read_device_status() == 0
