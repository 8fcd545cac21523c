"""The Python binding checks what the C entry points cannot see behind a raw pointer (the
element type and the extents of every tensor) before anything reaches the library, so a
wrong tensor raises on the host instead of letting a kernel read or write past its end.

CPU only: the tensors here live on the host, so a call whose arguments all pass the checks
stops at the next one ("CUDA tensors only") — no device pointer is ever formed.  The
bound-call object (ForwardCall) is checked against dsa_forward with a recording stand-in for
the library: it must hand the C entry point the same arguments."""

import ctypes

import pytest
import torch

from sparse_attention_long_03_b200 import dsa

T, HI, DI, H, DKV, DV, K, MAXPOS = 4, 64, 128, 128, 576, 512, 2048, 4095


def _cache():
    return dsa.PagedCache(None, None, None, None, 4, 64, 256, 64, DI, DKV)


def _queries():
    return dsa.Queries(T, None, None, MAXPOS)


def _indexer_args():
    return dict(q8=torch.zeros(T, HI, DI, dtype=torch.uint8), q_scale=torch.ones(T),
                w=torch.zeros(T, HI), logits=torch.zeros(T, MAXPOS + 1))


def _attn_args():
    return dict(q=torch.zeros(T, H, DKV, dtype=torch.bfloat16),
                idx=torch.zeros(T, K, dtype=torch.int32),
                out=torch.zeros(T, H, DV, dtype=torch.int16), lse=torch.zeros(T, H))


def _expect(msg, fn, *a, **kw):
    with pytest.raises(ValueError, match=msg):
        fn(*a, **kw)


def test_indexer_arguments():
    c, q = _cache(), _queries()
    a = _indexer_args()
    _expect("CUDA tensors only", dsa.dsa_indexer_logits, c, q, **a)  # all checks passed
    bad = [("q8", torch.zeros(T, HI, DI, dtype=torch.int8), "q8: dtype"),
           ("q8", torch.zeros(T, HI, 64, dtype=torch.uint8), "q8: shape"),
           ("q8", torch.zeros(T + 1, HI, DI, dtype=torch.uint8), "q8: shape"),
           ("q_scale", torch.ones(T, dtype=torch.float64), "q_scale: dtype"),
           ("w", torch.zeros(T, HI // 2), "w: shape"),
           ("logits", torch.zeros(T, MAXPOS), "logits: 4095 columns"),
           ("logits", torch.zeros(T, MAXPOS + 1, dtype=torch.float16), "logits: dtype")]
    for name, t, msg in bad:
        _expect(msg, dsa.dsa_indexer_logits, c, q, **{**a, name: t})
        _expect(msg, dsa.dsa_indexer_logits_noalloc, c, q, **{**a, name: t})
    # FP8 may also come typed as e4m3
    _expect("CUDA tensors only", dsa.dsa_indexer_logits, c, q,
            **{**a, "q8": torch.zeros(T, HI, DI, dtype=torch.float8_e4m3fn)})


def test_topk_arguments():
    q = _queries()
    logits, idx = torch.zeros(T, MAXPOS + 1), torch.zeros(T, K, dtype=torch.int32)
    _expect("CUDA tensors only", dsa.dsa_topk, logits, q, K, idx)
    _expect("idx: shape", dsa.dsa_topk, logits, q, K, torch.zeros(T, K - 1, dtype=torch.int32))
    _expect("idx: dtype", dsa.dsa_topk, logits, q, K, torch.zeros(T, K, dtype=torch.int64))
    _expect("logits: 2048 columns", dsa.dsa_topk, torch.zeros(T, 2048), q, K, idx)


def test_attention_arguments():
    c, q = _cache(), _queries()
    a = _attn_args()
    f = dsa.dsa_sparse_mla_attn
    _expect("CUDA tensors only", f, c, q, a["q"], DV, 0.07, a["idx"], a["out"], a["lse"])
    _expect("CUDA tensors only", f, c, q, a["q"], DV, 0.07, a["idx"], a["out"])  # lse optional
    _expect("q: shape", f, c, q, torch.zeros(T, H, 512, dtype=torch.int16), DV, 0.07, a["idx"],
            a["out"])
    _expect("q: dtype", f, c, q, torch.zeros(T, H, DKV), DV, 0.07, a["idx"], a["out"])
    _expect("out: shape", f, c, q, a["q"], DV, 0.07, a["idx"],
            torch.zeros(T, H, 256, dtype=torch.int16))
    _expect("out: shape", f, c, q, a["q"], DV, 0.07, a["idx"],
            torch.zeros(T, H // 2, DV, dtype=torch.int16))
    _expect("lse: shape", f, c, q, a["q"], DV, 0.07, a["idx"], a["out"], torch.zeros(T, H, 1))
    _expect("idx: shape", f, c, q, a["q"], DV, 0.07, torch.zeros(T + 1, K, dtype=torch.int32),
            a["out"])


def test_forward_arguments():
    c, q = _cache(), _queries()
    i, a = _indexer_args(), _attn_args()

    def fwd(**over):
        x = {**i, **a, **over}
        return dsa.dsa_forward(c, q, x["q8"], x["q_scale"], x["w"], x["q"], DV, 0.07, K,
                               x["out"], x["lse"], x["idx"])

    _expect("CUDA tensors only", fwd)
    _expect("CUDA tensors only", fwd, idx=None)  # idx_out optional
    _expect("q8: shape", fwd, q8=torch.zeros(T, HI, 32, dtype=torch.uint8))
    _expect("w: shape", fwd, w=torch.zeros(T, HI + 1))
    _expect("idx: shape", fwd, idx=torch.zeros(T, K // 2, dtype=torch.int32))
    _expect("out: dtype", fwd, out=torch.zeros(T, H, DV))


def test_cache_and_queries_descriptors():
    rows = 256 * 64
    k8, ks = torch.zeros(rows, DI, dtype=torch.uint8), torch.zeros(rows)
    kv, bt = torch.zeros(rows, DKV, dtype=torch.int16), torch.zeros(4, 64, dtype=torch.int32)
    _expect("CUDA tensors only", dsa.make_cache, k8, ks, kv, bt)
    _expect("CUDA tensors only", dsa.make_cache, k8, ks, None, bt)  # keys only
    _expect("CUDA tensors only", dsa.make_cache, None, None, kv, bt)  # latent rows only
    _expect("k_scale: shape", dsa.make_cache, k8, torch.zeros(rows - 1), kv, bt)
    _expect("kv: shape", dsa.make_cache, k8, ks, kv[:-64], bt)
    _expect("block_table: dtype", dsa.make_cache, k8, ks, kv, bt.long())
    _expect("k8: dtype", dsa.make_cache, k8.short(), ks, kv, bt)
    seq, pos = torch.zeros(T, dtype=torch.int32), torch.zeros(T, dtype=torch.int32)
    _expect("CUDA tensors only", dsa.make_queries, seq, pos, 7)
    _expect("tok_pos: shape", dsa.make_queries, seq, pos[:-1], 7)
    _expect("tok_seq: dtype", dsa.make_queries, seq.long(), pos, 7)


def test_append_arguments():
    c, n, rows = _cache(), 5, 256 * 64
    k8, ks = torch.zeros(rows, DI, dtype=torch.uint8), torch.zeros(rows)
    kv = torch.zeros(rows, DKV, dtype=torch.int16)
    seq, pos = torch.zeros(n, dtype=torch.int32), torch.zeros(n, dtype=torch.int32)
    k_in, kv_in = torch.zeros(n, DI), torch.zeros(n, DKV, dtype=torch.int16)
    f = dsa.dsa_cache_append
    _expect("CUDA tensors only", f, c, k8, ks, kv, seq, pos, k_in, kv_in)
    _expect("CUDA tensors only", f, c, k8, ks, None, seq, pos, k_in)
    _expect("k8: 16320 rows", f, c, k8[:-64], ks[:-64], kv, seq, pos, k_in, kv_in)
    _expect("k_in: shape", f, c, k8, ks, kv, seq, pos, torch.zeros(n, 64), kv_in)
    _expect("k_in: dtype", f, c, k8, ks, kv, seq, pos, k_in.half(), kv_in)
    _expect("kv_in: shape", f, c, k8, ks, kv, seq, pos, k_in, kv_in[:, :512])
    _expect("tok_pos: shape", f, c, k8, ks, kv, seq, pos[:-1], k_in, kv_in)


def test_context_parallel_arguments():
    G = 2
    logits = torch.zeros(T, MAXPOS + 1)
    idx = torch.zeros(T, K, dtype=torch.int32)
    vals, poss = torch.zeros(T, K), torch.zeros(T, K, dtype=torch.int32)
    _expect("CUDA tensors only", dsa.dsa_cp_candidates, logits, idx, 0, vals, poss)
    _expect("values: shape", dsa.dsa_cp_candidates, logits, idx, 0, vals[:, :-1], poss)
    _expect("positions: dtype", dsa.dsa_cp_candidates, logits, idx, 0, vals, poss.long())

    gv, gp = torch.zeros(G, T, K), torch.zeros(G, T, K, dtype=torch.int32)
    out_idx = torch.zeros(T, K, dtype=torch.int32)
    _expect("CUDA tensors only", dsa.dsa_cp_merge_topk, gv, gp, K, out_idx)
    _expect("values: shape", dsa.dsa_cp_merge_topk, gv, gp, K // 2, out_idx)  # k != row length
    _expect("positions: shape", dsa.dsa_cp_merge_topk, gv, gp[:1], K, out_idx)
    _expect("idx_local: shape", dsa.dsa_cp_merge_topk, gv, gp, K, out_idx, 0, 64,
            torch.zeros(T, 1, dtype=torch.int32))

    o = torch.zeros(G, T, H, DV, dtype=torch.int16)
    lp, out, lse = torch.zeros(G, T, H), torch.zeros(T, H, DV, dtype=torch.int16), torch.zeros(T, H)
    _expect("CUDA tensors only", dsa.dsa_cp_attn_merge, o, lp, out, lse)
    _expect("lse_parts: shape", dsa.dsa_cp_attn_merge, o, lp[:, :, :-1], out, lse)
    _expect("out: shape", dsa.dsa_cp_attn_merge, o, lp, out[:-1], lse)
    _expect("o_parts: dtype", dsa.dsa_cp_attn_merge, o.float(), lp, out, lse)


class _RecordingLib:
    """Stands in for libdsa: records each call's arguments and returns DSA_OK."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            return 1 << 20 if name.endswith("workspace_size") else 0
        return fn


def _norm(a):
    if hasattr(a, "_obj"):  # ctypes.byref
        return ("ref", id(a._obj))
    if isinstance(a, ctypes.c_void_p):
        return ("ptr", a.value)
    return a


def test_forward_call_marshals_like_dsa_forward(monkeypatch):
    """ForwardCall passes the C entry point exactly what dsa_forward passes, and each call
    of the bound object is one call of the entry point."""
    fake = _RecordingLib()
    monkeypatch.setattr(dsa, "_LIB", fake)
    monkeypatch.setattr(dsa, "_ptr", lambda t: None if t is None else ctypes.c_void_p(t.data_ptr()))
    monkeypatch.setattr(dsa, "_stream", lambda s=None: ctypes.c_void_p(1234))
    c, q = _cache(), _queries()
    i, a = _indexer_args(), _attn_args()
    ws = torch.empty(1 << 20, dtype=torch.uint8)
    argv = (c, q, i["q8"], i["q_scale"], i["w"], a["q"], DV, 0.07, K, a["out"], a["lse"], a["idx"],
            ws)
    dsa.dsa_forward(*argv)
    direct = [x for x in fake.calls if x[0] == "dsa_forward"]
    fc = dsa.ForwardCall(*argv)
    n0 = len(fake.calls)
    fc()
    fc()
    bound = [x for x in fake.calls[n0:] if x[0] == "dsa_forward"]
    assert len(direct) == 1 and len(bound) == 2 and len(fake.calls) - n0 == 2
    want = [_norm(x) for x in direct[0][1]]
    for _, args in bound:
        assert [_norm(x) for x in args] == want
    assert len(want) == 17


def test_forward_call_checks_its_arguments():
    c, q = _cache(), _queries()
    i, a = _indexer_args(), _attn_args()
    with pytest.raises(ValueError, match="out: shape"):
        dsa.ForwardCall(c, q, i["q8"], i["q_scale"], i["w"], a["q"], DV, 0.07, K,
                        torch.zeros(T, H, DV // 2, dtype=torch.int16))
    with pytest.raises(ValueError, match="CUDA tensors only"):
        dsa.ForwardCall(c, q, i["q8"], i["q_scale"], i["w"], a["q"], DV, 0.07, K, a["out"])
