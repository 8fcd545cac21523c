"""Shared helpers of the GPU parity tests: device upload of a workload and the
comparison rules against the oracle.

Tolerances (the workload definition's parity bar):
  * indexer logits: relative error <= 1e-3 per entry, with the denominator floored at
    1e-3 * max|row| (sums of ReLU terms with signed weights cross zero, where a plain
    relative error is undefined);
  * top-k on the GPU's own logits: the exact oracle set (bit-exact index work);
  * top-k inside the fused path (GPU logits vs oracle logits): sets equal except for
    positions whose oracle logit lies within 1e-3*|I_k| of the k-th value I_k;
  * attention on the GPU-selected set: max |g-r| <= 1e-2 and
    sum|g-r| / sum|r| <= 2e-3 (outputs are BF16); LSE within 2e-3 absolute.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import dsa_ref as R
from sparse_attention_long_03_b200 import dsa

LOGIT_RTOL = 1e-3
TOPK_BAND = 1e-3
ATTN_MAX_ABS = 1e-2
ATTN_MEAN_REL = 2e-3
LSE_ABS = 2e-3


class DeviceWorkload:
    """Device copies of a host workload plus the C-ABI descriptors."""

    def __init__(self, cfg, cache, qs, device="cuda"):
        self.cfg = cfg
        self.host_cache = cache
        self.host_q = qs
        d = device
        self.k8 = torch.from_numpy(cache.k8).to(d)
        self.k_scale = torch.from_numpy(cache.k_scale).to(d)
        self.kv = torch.from_numpy(cache.kv.view(np.int16)).to(d) if cache.kv is not None else None
        self.block_table = torch.from_numpy(cache.block_table).to(d)
        self.cache = dsa.make_cache(self.k8, self.k_scale, self.kv, self.block_table)
        self.set_queries(qs)

    def set_queries(self, qs):
        d = self.k8.device
        self.host_q = qs
        self.tok_seq = torch.from_numpy(qs.tok_seq).to(d)
        self.tok_pos = torch.from_numpy(qs.tok_pos).to(d)
        self.q8 = torch.from_numpy(qs.q8).to(d)
        self.q_scale = torch.from_numpy(qs.q_scale).to(d)
        self.w = torch.from_numpy(qs.w).to(d)
        self.q = torch.from_numpy(qs.q.view(np.int16)).to(d) if qs.q is not None else None
        self.max_pos = int(qs.tok_pos.max()) if qs.n_tokens else 0
        self.queries = dsa.make_queries(self.tok_seq, self.tok_pos, self.max_pos)
        self.ld = ((self.max_pos + 1 + 127) // 128) * 128

    # -- stages through the C ABI
    def indexer(self):
        logits = torch.full((self.host_q.n_tokens, self.ld), float("nan"), device=self.k8.device)
        dsa.dsa_indexer_logits(self.cache, self.queries, self.q8, self.q_scale, self.w, logits)
        return logits

    def topk(self, logits, k=None):
        k = k or self.cfg.topk
        idx = torch.full((self.host_q.n_tokens, k), -7, dtype=torch.int32, device=self.k8.device)
        dsa.dsa_topk(logits, self.queries, k, idx)
        return idx

    def attention(self, idx, with_lse=True):
        T, H = self.host_q.n_tokens, self.cfg.n_heads
        out = torch.zeros((T, H, self.cfg.d_v), dtype=torch.int16, device=self.k8.device)
        lse = torch.zeros((T, H), dtype=torch.float32, device=self.k8.device) if with_lse else None
        dsa.dsa_sparse_mla_attn(self.cache, self.queries, self.q, self.cfg.d_v, self.cfg.scale,
                                idx, out, lse)
        return out, lse

    def forward(self, with_idx=True):
        T, H = self.host_q.n_tokens, self.cfg.n_heads
        out = torch.zeros((T, H, self.cfg.d_v), dtype=torch.int16, device=self.k8.device)
        lse = torch.zeros((T, H), dtype=torch.float32, device=self.k8.device)
        idx = (torch.full((T, self.cfg.topk), -7, dtype=torch.int32, device=self.k8.device)
               if with_idx else None)
        dsa.dsa_forward(self.cache, self.queries, self.q8, self.q_scale, self.w, self.q,
                        self.cfg.d_v, self.cfg.scale, self.cfg.topk, out, lse, idx)
        return out, lse, idx


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.bfloat16).to(torch.float64).cpu().numpy()


def oracle_logits(w: DeviceWorkload, t: int) -> np.ndarray:
    c, q = w.host_cache, w.host_q
    return R.indexer_logits_row(c.k8, c.k_scale, c.block_table, int(q.tok_seq[t]),
                                int(q.tok_pos[t]), q.q8[t], q.q_scale[t], q.w[t])


def logit_error(g: np.ndarray, r: np.ndarray) -> float:
    floor = 1e-3 * np.abs(r).max() if r.size else 1.0
    den = np.maximum(np.abs(r), max(floor, 1e-30))
    return float(np.max(np.abs(g - r) / den)) if r.size else 0.0


def check_topk_band(g_idx: np.ndarray, r_logits: np.ndarray, k: int):
    """The fused-path selection rule; returns (ok, message)."""
    n = r_logits.shape[0]
    n_sel = min(k, n)
    G = g_idx[g_idx >= 0]
    if G.size != n_sel or (g_idx[n_sel:] != -1).any():
        return False, f"size {G.size} != {n_sel} or bad padding"
    if np.unique(G).size != G.size:
        return False, "duplicates"
    if G.min() < 0 or G.max() >= n:
        return False, "out of range"
    vk = R.kth_value(r_logits, k)
    b = TOPK_BAND * abs(vk)
    must = np.nonzero(r_logits > vk + b)[0]
    if not np.isin(must, G).all():
        return False, f"missing {np.setdiff1d(must, G)[:8]}"
    if not (r_logits[G] >= vk - b).all():
        return False, "selected below the band"
    return True, ""


def attn_errors(g: np.ndarray, r: np.ndarray):
    d = np.abs(g - r)
    return float(d.max()), float(d.sum() / max(np.abs(r).sum(), 1e-30))


def oracle_attention(w: DeviceWorkload, t: int, sel: np.ndarray):
    c, q = w.host_cache, w.host_q
    return R.sparse_mla_attn_token(c.kv, c.block_table, int(q.tok_seq[t]), q.q[t], sel,
                                   w.cfg.scale, w.cfg.d_v)


# ------------------------------------------------------------------------------ guard regions

GUARD_BYTES = 4096   # a multiple of 256: the interior keeps the allocation's alignment
GUARD_BYTE = 0xA5


class Guarded:
    """A tensor of `shape` and `dtype` placed inside one larger byte allocation, with
    GUARD_BYTES of a fixed byte pattern before it and at least that many after it.  A
    kernel that writes past either end of the tensor changes a guard byte; intact() says
    whether the guards still hold the pattern.  This stands in for a memory checker."""

    def __init__(self, shape, dtype, device, fill=None):
        shape = tuple(int(s) for s in shape)
        elem = torch.empty((), dtype=dtype).element_size()
        self.nbytes = int(np.prod(shape, dtype=np.int64)) * elem
        padded = (self.nbytes + 255) // 256 * 256
        self.buf = torch.full((GUARD_BYTES + padded + GUARD_BYTES,), GUARD_BYTE,
                              dtype=torch.uint8, device=device)
        self.t = self.buf[GUARD_BYTES:GUARD_BYTES + self.nbytes].view(dtype).view(shape)
        if fill is not None:
            self.t.fill_(fill)

    def intact(self) -> bool:
        head = self.buf[:GUARD_BYTES]
        tail = self.buf[GUARD_BYTES + self.nbytes:]
        return bool((head == GUARD_BYTE).all().item() and (tail == GUARD_BYTE).all().item())
