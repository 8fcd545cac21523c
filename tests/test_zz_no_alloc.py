"""The indexer entry point for callers that cannot allocate device memory
(dsa_indexer_logits_noalloc) gives the same logits as the allocating entry point, on two
calls in a row, and rejects calls larger than its fixed scratch.

This file is collected last on purpose: it checks an addition that leaves every other
path unchanged, so a run that stops at the first failure has run all else before it."""

import ctypes

import numpy as np
import pytest
import torch

from sparse_attention_long_03_b200 import dsa
from sparse_attention_long_03_b200 import workloads as W

from dsa_testutil import LOGIT_RTOL, DeviceWorkload, logit_error

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "decode_32k"])
def test_noalloc_indexer_matches_allocating_entry_point(name):
    cfg, cache, qs = W.make(name, with_kv=False, with_q=False)
    w = DeviceWorkload(cfg, cache, qs)
    ref = w.indexer().cpu().numpy()
    assert dsa.dsa_read_device_status() == 0
    for _ in range(2):  # the shared scratch keeps the previous call's contents
        got = torch.full_like(torch.from_numpy(ref), float("nan")).cuda()
        dsa.dsa_indexer_logits_noalloc(w.cache, w.queries, w.q8, w.q_scale, w.w, got)
        assert dsa.dsa_read_device_status() == 0
        got = got.cpu().numpy()
        for t in range(qs.n_tokens):
            n = int(qs.tok_pos[t]) + 1
            g, r = got[t, :n].astype(np.float64), ref[t, :n].astype(np.float64)
            assert np.isfinite(g).all()
            assert logit_error(g, r) <= LOGIT_RTOL


def test_noalloc_rejects_more_tokens_than_its_scratch():
    L = dsa.lib()
    q = dsa.Queries(12289, 16, 16, 100)
    c = dsa.PagedCache(16, 16, 16, 16, 1, 8, 8, 64, 128, 576)
    st = L.dsa_indexer_logits_noalloc(ctypes.byref(c), ctypes.byref(q), 16, 16, 16, 64, 16,
                                      128, None)
    assert st == 3  # DSA_ERR_WORKSPACE, nothing launched
