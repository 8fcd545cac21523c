"""GPU parity of each stage and of the fused path against the CPU oracle, on the tiny,
decode-32K and decode-128K workloads (every query token checked in full), plus edge
cases.  All calls go through the C ABI (libdsa.so)."""

import functools

import numpy as np
import pytest
import torch

from oracle import dsa_ref as R
from sparse_attention_long_03_b200 import dsa
from sparse_attention_long_03_b200 import workloads as W

from dsa_testutil import (ATTN_MAX_ABS, ATTN_MEAN_REL, LOGIT_RTOL, LSE_ABS, DeviceWorkload,
                          attn_errors, bf16_to_f64, check_topk_band, logit_error,
                          oracle_attention, oracle_logits)

pytestmark = pytest.mark.gpu

DECODE = ["tiny", "decode_32k", "decode_128k"]


@functools.lru_cache(maxsize=None)
def workload(name):
    cfg, cache, qs = W.make(name)
    return DeviceWorkload(cfg, cache, qs)


@functools.lru_cache(maxsize=None)
def staged(name):
    """GPU logits, GPU top-k on them, GPU attention on that selection (host copies)."""
    w = workload(name)
    logits = w.indexer()
    idx = w.topk(logits)
    out, lse = w.attention(idx)
    torch.cuda.synchronize()
    assert dsa.dsa_read_device_status() == 0
    return logits.cpu().numpy(), idx.cpu().numpy(), bf16_to_f64(out), lse.cpu().numpy()


@functools.lru_cache(maxsize=None)
def oracle_rows(name):
    w = workload(name)
    return [oracle_logits(w, t) for t in range(w.host_q.n_tokens)]


@pytest.mark.parametrize("name", DECODE)
def test_indexer_logits(name):
    w = workload(name)
    logits, _, _, _ = staged(name)
    for t, r in enumerate(oracle_rows(name)):
        g = logits[t, :r.shape[0]].astype(np.float64)
        assert np.isfinite(g).all(), f"token {t}: non-finite logits"
        err = logit_error(g, r)
        assert err <= LOGIT_RTOL, f"token {t}: logit error {err:.3e}"


@pytest.mark.parametrize("name", DECODE)
def test_topk_exact_on_gpu_logits(name):
    """The selection step alone is integer work: on the GPU's own fp32 logits it must
    reproduce the oracle's set exactly (ties to the smaller position)."""
    w = workload(name)
    logits, idx, _, _ = staged(name)
    k = w.cfg.topk
    for t in range(w.host_q.n_tokens):
        n = int(w.host_q.tok_pos[t]) + 1
        ref = R.topk_select(logits[t, :n].astype(np.float64), k)
        got = idx[t][idx[t] >= 0]
        assert (idx[t][min(k, n):] == -1).all()
        assert np.array_equal(np.sort(got), ref), f"token {t}"


@pytest.mark.parametrize("name", DECODE)
def test_topk_band_against_oracle_logits(name):
    w = workload(name)
    _, idx, _, _ = staged(name)
    for t, r in enumerate(oracle_rows(name)):
        ok, msg = check_topk_band(idx[t], r, w.cfg.topk)
        assert ok, f"token {t}: {msg}"


@pytest.mark.parametrize("name", DECODE)
def test_attention_on_gpu_selection(name):
    w = workload(name)
    _, idx, out, lse = staged(name)
    for t in range(w.host_q.n_tokens):
        sel = idx[t][idx[t] >= 0]
        ro, rl = oracle_attention(w, t, sel)
        mx, mr = attn_errors(out[t], ro)
        assert mx <= ATTN_MAX_ABS and mr <= ATTN_MEAN_REL, f"token {t}: max {mx:.2e} rel {mr:.2e}"
        assert np.abs(lse[t] - rl).max() <= LSE_ABS


@pytest.mark.parametrize("name", DECODE)
def test_fused_forward_matches_stages(name):
    """dsa_forward runs the same kernels: identical selection and output."""
    w = workload(name)
    _, idx_s, out_s, lse_s = staged(name)
    out, lse, idx = w.forward()
    torch.cuda.synchronize()
    assert dsa.dsa_read_device_status() == 0
    assert np.array_equal(idx.cpu().numpy(), idx_s)
    assert np.array_equal(bf16_to_f64(out), out_s)
    assert np.array_equal(lse.cpu().numpy(), lse_s)


def test_planted_keys_selected_on_gpu():
    w = workload("decode_128k")
    _, idx, _, _ = staged("decode_128k")
    for t in range(w.host_q.n_tokens):
        b = int(w.host_q.tok_seq[t])
        planted = W.planted_positions(w.cfg, b, int(w.host_cache.seq_lens[b]))
        assert np.isin(planted, idx[t]).all()


# ------------------------------------------------------------------------------ edge cases

def _topk_rows(rows, k, max_pos=None):
    """Run dsa_topk on explicit fp32 rows (one query token per row)."""
    T = len(rows)
    n_max = max(r.shape[0] for r in rows)
    max_pos = max_pos if max_pos is not None else n_max - 1
    ld = max_pos + 1
    logits = torch.full((T, ld), float("nan"))
    for t, r in enumerate(rows):
        logits[t, :r.shape[0]] = torch.from_numpy(r.astype(np.float32))
    logits = logits.cuda()
    tok_pos = torch.tensor([r.shape[0] - 1 for r in rows], dtype=torch.int32, device="cuda")
    tok_seq = torch.zeros(T, dtype=torch.int32, device="cuda")
    q = dsa.make_queries(tok_seq, tok_pos, max_pos)
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(logits, q, k, idx)
    return idx.cpu().numpy()


@pytest.mark.parametrize("long_rows", [False, True])
def test_topk_edge_cases(long_rows):
    rng = np.random.default_rng(11)
    k = 2048
    rows = [
        np.array([1.0]),                                   # single position
        rng.standard_normal(k),                            # exactly k
        rng.standard_normal(k + 1),                        # one too many
        np.full(5000, 0.25),                               # all equal: first k positions
        rng.integers(-3, 4, size=9000).astype(np.float64),  # heavy ties
        -np.abs(rng.standard_normal(7000)) - 1.0,          # all negative
        np.concatenate([np.zeros(3000), -np.zeros(3000)]),  # +0 and -0 are equal
        rng.standard_normal(30000) * 1e-30,                # tiny magnitudes
    ]
    if long_rows:  # rows longer than the shared-memory row cache
        rows += [rng.standard_normal(70000), rng.integers(0, 3, size=50000).astype(np.float64)]
    max_pos = 100000 if long_rows else None
    idx = _topk_rows(rows, k, max_pos)
    for t, r in enumerate(rows):
        rr = r.astype(np.float32).astype(np.float64)
        ref = R.topk_select(rr, k)
        got = idx[t][idx[t] >= 0]
        assert np.array_equal(np.sort(got), ref), f"row {t}"
        assert (idx[t][min(k, r.shape[0]):] == -1).all()


def test_attention_empty_and_ragged_selection():
    """Rows with fewer than k valid entries (-1 padding), a single entry, and none."""
    w = workload("decode_32k")
    T, k = w.host_q.n_tokens, w.cfg.topk
    rng = np.random.default_rng(12)
    idx = np.full((T, k), -1, np.int32)
    counts = [1, 2, 63, 64, 65, 1000, 2047, 0]
    for t, c in enumerate(counts):
        pos = int(w.host_q.tok_pos[t])
        sel = np.sort(rng.choice(pos + 1, size=c, replace=False))
        slots = np.sort(rng.choice(k, size=c, replace=False))  # scattered among -1 slots
        idx[t, slots] = sel
    out, lse = w.attention(torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    assert dsa.dsa_read_device_status() == 0
    out, lse = bf16_to_f64(out), lse.cpu().numpy()
    for t, c in enumerate(counts):
        sel = idx[t][idx[t] >= 0]
        if c == 0:
            assert (out[t] == 0).all() and np.isneginf(lse[t]).all()
            continue
        ro, rl = oracle_attention(w, t, sel)
        mx, mr = attn_errors(out[t], ro)
        assert mx <= ATTN_MAX_ABS and mr <= ATTN_MEAN_REL, f"count {c}: {mx:.2e} {mr:.2e}"
        assert np.abs(lse[t] - rl).max() <= LSE_ABS


def test_bad_block_table_entry_is_reported_not_faulted():
    cfg, cache, qs = W.make("tiny")
    cache.block_table = cache.block_table.copy()
    cache.block_table[0, 3] = 10 ** 6  # far outside the cache
    w = DeviceWorkload(cfg, cache, qs)
    logits = w.indexer()
    assert dsa.dsa_read_device_status() == 5  # DSA_ERR_BAD_INDEX, and the word is cleared
    lg = logits.cpu().numpy()
    for t in range(qs.n_tokens):
        n = int(qs.tok_pos[t]) + 1
        assert np.isnan(lg[t, 192:256]).all()  # logical block 3 = positions 192..255
        assert np.isfinite(lg[t, :192]).all() and np.isfinite(lg[t, 256:n]).all()
    assert dsa.dsa_read_device_status() == 0  # the context is still usable


def test_bad_selected_index_is_reported():
    w = workload("tiny")
    idx = torch.zeros((w.host_q.n_tokens, w.cfg.topk), dtype=torch.int32, device="cuda")
    idx[0, 0] = 100000  # beyond the token's position
    w.attention(idx)
    assert dsa.dsa_read_device_status() == 5
    assert dsa.dsa_read_device_status() == 0


def test_launch_count_moves():
    w = workload("tiny")
    n0 = dsa.dsa_launch_count()
    w.forward()
    torch.cuda.synchronize()
    assert dsa.dsa_launch_count() - n0 >= 3
