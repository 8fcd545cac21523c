"""Out-of-bounds writes on the GPU, the stand-in for a memory checker: every buffer an
entry point writes (outputs and workspaces) is a view into a larger allocation whose guard
regions hold a byte pattern (dsa_testutil.Guarded); after the call the guards must be
unchanged and the device status clean.  Covered: the three stages and the fused forward on
the tiny and decode-32K workloads and on a prefill sample (every 7th causal row of the 16K
sequence: the batch plan, the row-wise top-k and the split-free attention), the
allocation-free indexer, the cache append and the context-parallel kernels.

Collected after the parity files: a failure here stops (-x) only what follows it."""

import numpy as np
import pytest
import torch

from sparse_attention_long_03_b200 import dsa
from sparse_attention_long_03_b200 import workloads as W

from dsa_testutil import DeviceWorkload, Guarded
from test_gpu_append import _case

pytestmark = pytest.mark.gpu

CASES = ["tiny", "decode_32k", "prefill_sample"]
DEV = "cuda"


def _workload(name):
    if name == "prefill_sample":
        cfg = W.CONFIGS["prefill_16k"]
        qs = W.prefill_queries(cfg, positions=np.arange(0, 16384, 7))
        cache = W.make_cache(cfg)
    else:
        cfg, cache, qs = W.make(name)
    return DeviceWorkload(cfg, cache, qs, device=DEV)


def _clean(*guarded):
    torch.cuda.synchronize()
    assert dsa.dsa_read_device_status() == 0
    for g in guarded:
        assert g.intact()


def _ws(nbytes, dev):
    return Guarded((max(256, int(nbytes)),), torch.uint8, dev)


@pytest.mark.parametrize("name", CASES)
def test_stages_write_only_their_outputs(name):
    w = _workload(name)
    T, H, k, dv = w.host_q.n_tokens, w.cfg.n_heads, w.cfg.topk, w.cfg.d_v
    dev, L = w.k8.device, dsa.lib()
    logits = Guarded((T, w.ld), torch.float32, dev, fill=float("nan"))
    ws_i = _ws(L.dsa_indexer_workspace_size(T), dev)
    dsa.dsa_indexer_logits(w.cache, w.queries, w.q8, w.q_scale, w.w, logits.t, ws_i.t)
    _clean(logits, ws_i)
    idx = Guarded((T, k), torch.int32, dev, fill=-7)
    ws_t = _ws(L.dsa_topk_workspace_size(T, w.max_pos, k), dev)
    dsa.dsa_topk(logits.t, w.queries, k, idx.t, ws_t.t)
    _clean(idx, ws_t)
    out = Guarded((T, H, dv), torch.int16, dev, fill=0)
    lse = Guarded((T, H), torch.float32, dev, fill=0.0)
    ws_a = _ws(L.dsa_attn_workspace_size(T, H, dv, k), dev)
    dsa.dsa_sparse_mla_attn(w.cache, w.queries, w.q, dv, w.cfg.scale, idx.t, out.t, lse.t,
                            ws_a.t)
    _clean(out, lse, ws_a)
    if T <= 12288:
        logits2 = Guarded((T, w.ld), torch.float32, dev, fill=float("nan"))
        dsa.dsa_indexer_logits_noalloc(w.cache, w.queries, w.q8, w.q_scale, w.w, logits2.t)
        _clean(logits2)


@pytest.mark.parametrize("name", CASES)
def test_forward_writes_only_its_outputs(name):
    w = _workload(name)
    T, H, k, dv = w.host_q.n_tokens, w.cfg.n_heads, w.cfg.topk, w.cfg.d_v
    dev = w.k8.device
    for with_idx in (True, False):
        out = Guarded((T, H, dv), torch.int16, dev, fill=0)
        lse = Guarded((T, H), torch.float32, dev, fill=0.0)
        idx = Guarded((T, k), torch.int32, dev, fill=-7) if with_idx else None
        ws = _ws(dsa.forward_workspace_size(T, w.max_pos, k, H, dv), dev)
        dsa.dsa_forward(w.cache, w.queries, w.q8, w.q_scale, w.w, w.q, dv, w.cfg.scale, k,
                        out.t, lse.t, idx.t if with_idx else None, ws.t)
        _clean(out, lse, ws, *([idx] if with_idx else []))


def test_cache_append_writes_only_the_caches():
    rng = np.random.default_rng(5)
    k8, ks, kv, bt, tok_seq, tok_pos, k_in, kv_in = _case(rng, 128, 576, bad=False)
    dev = torch.device(DEV)
    g8 = Guarded(k8.shape, torch.uint8, dev)
    g8.t.copy_(torch.from_numpy(k8))
    gs = Guarded(ks.shape, torch.float32, dev)
    gs.t.copy_(torch.from_numpy(ks))
    gkv = Guarded(kv.shape, torch.int16, dev)
    gkv.t.copy_(torch.from_numpy(kv.view(np.int16)))
    dbt = torch.from_numpy(bt).to(dev)
    cache = dsa.make_cache(g8.t, gs.t, gkv.t, dbt)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    dsa.dsa_cache_append(cache, g8.t, gs.t, gkv.t, t(tok_seq), t(tok_pos), t(k_in),
                         t(kv_in.view(np.int16)))
    _clean(g8, gs, gkv)


def test_context_parallel_kernels_write_only_their_outputs():
    w = _workload("decode_32k")
    T, H, k, dv = w.host_q.n_tokens, w.cfg.n_heads, w.cfg.topk, w.cfg.d_v
    dev = w.k8.device
    logits = w.indexer()
    idx = w.topk(logits)
    vals = Guarded((T, k), torch.float32, dev)
    poss = Guarded((T, k), torch.int32, dev)
    dsa.dsa_cp_candidates(logits, idx, 1000, vals.t, poss.t)
    _clean(vals, poss)
    # two parts: the same candidates, the second part's positions moved past the first's
    pv = torch.stack([vals.t, vals.t]).contiguous()
    pp = torch.stack([poss.t, torch.where(poss.t >= 0, poss.t + 40000, poss.t)]).contiguous()
    sel = Guarded((T, k), torch.int32, dev, fill=-7)
    sel_local = Guarded((T, k), torch.int32, dev, fill=-7)
    ws = _ws(dsa.lib().dsa_cp_merge_workspace_size(T, 2, k), dev)
    dsa.dsa_cp_merge_topk(pv, pp, k, sel.t, 0, 40000, sel_local.t, ws.t)
    _clean(sel, sel_local, ws)
    o_parts = torch.zeros((2, T, H, dv), dtype=torch.int16, device=dev)
    l_parts = torch.zeros((2, T, H), dtype=torch.float32, device=dev)
    out = Guarded((T, H, dv), torch.int16, dev, fill=0)
    lse = Guarded((T, H), torch.float32, dev, fill=0.0)
    dsa.dsa_cp_attn_merge(o_parts, l_parts, out.t, lse.t)
    _clean(out, lse)
